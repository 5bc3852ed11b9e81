// Sequential part of the gate-aware backward of Gated Delta Rule-2 on the
// sm_100a tensor cores (bf16 I/O, d_k = d_v = 128, chunk 64): the reverse
// state pass, dv, dw and dS0, after the forward has left its chunk records
// (T, P among them), chunk states and Delta in the workspace.  The chunk-
// parallel gradients dq, dk, db, dg follow in tc_bwd_grad.cu.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B): only the state gradient crosses chunk borders.  Per chunk
// (chunk-start frame, tc_common.cuh; dS' = dL/dS_{c+1} entering the chunk
// from the right):
//   dDelta = P^T dO + Kb dS',           dU = T^T dDelta,   dw = dU.v, dv = dU.w
//   dS_c  = diag(gamma) dS' + Qb^T dO - W^T dDelta                 (carried left)
// In a mild chunk's frame (frame factor s, see REC_* in common.cuh) the record
// holds Kx = Kb s / gamma, Qb / s and W / s, so the kernel feeds r dS' with
// r = gamma / s, starts tensor memory at (gamma / s) dS' and reads dS_c / s.

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

// ============================================================ state kernel
namespace tbs {
constexpr int kCompute = 256;            // warps 0..7: readouts, dU outputs, the next dX
constexpr int kThreads = kCompute + 64;  // warp 8 issues the products; warp 9 the copies
constexpr uint32_t STG = 0;                   // two chunk records, REC_BYTES each
constexpr uint32_t RAW_DO = 2 * REC_BYTES;    // dO half, bf16 [64 pos][64]
constexpr uint32_t OP_DO = RAW_DO + 8192;     // dO fp16      [64 pos][64 v]  MN-major B
constexpr uint32_t OP_DS = OP_DO + 8192;      // dX fp16      [128 key][64 v] MN-major B
constexpr uint32_t OP_DD = OP_DS + 16384;     // dDelta fp16  [64 pos][64 v]  MN-major B
constexpr uint32_t VV = OP_DD + 8192;         // v half bf16 [64][64], 128-B swizzled; dv in place
constexpr uint32_t VW = VV + 8192;            // w half: f32 as two [64][32] 128-B swizzled boxes, or
                                              // bf16 as one [64][64]; dw in place
constexpr uint32_t NDU = VW + 16384;          // -dU fp16 [64 pos][64 v] (the workspace layout)
constexpr uint32_t MISC = NDU + 8192;         // mbarriers; TMEM slot
constexpr uint32_t SMEM_BYTES = MISC + 128 + 1024;
constexpr uint32_t TM_DS = 0, TM_DD = 64, TM_DU = 128;  // 256 columns allocated
constexpr uint32_t ID_MM64 = idesc_f16(64, 64, true, true);
constexpr uint32_t ID_KM64 = idesc_f16(64, 64, false, true);
constexpr uint32_t ID_MM128x64 = idesc_f16(128, 64, true, true);
constexpr long long kWait = 2000000000LL;
constexpr float kRange = 6.0e4f;
static_assert(MISC % 1024 == 0, "alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace tbs

// One CTA per (b, h, half of d_v), walking the chunks in reverse.  Entering
// chunk c, the compute warps put diag(gamma / s) dS' in tensor memory and
// r dS' as an fp16 operand (s, r of the chunk's frame: s = r = 1 in the
// chunk-start frame).  Per chunk, from the chunk's record (Qb, Kx, -W, T, P,
// gamma, s):
//   (1) dDelta = P^T dO + Kb dS'  (committed alone),  then dS += Qb^T dO
//   (2) dS += (-W)^T dDelta  (committed alone),       then dU = T^T dDelta
// after which tensor memory holds dS_c / s, the dS' of chunk c - 1 once
// multiplied by s.  dU is read
// while the next chunk's first products run: dv = dU.w and dw = dU.v are
// formed in place of the v and w tiles (128-B swizzled TMA tiles) and leave
// by TMA stores; -dU and dS' go to the workspace for the gradient kernel.  Warps 0..7 read
// the accumulators and form the operands and outputs; warp 8 issues the
// products (an issuing thread is held for about as long as the products
// run); warp 9 requests every copy, so that neither delays the readouts.
template <bool GB, bool ACT>  // w and dw as bf16 (else float32); ACT: gate logits (GateAct)
__global__ void __launch_bounds__(tbs::kThreads, 1)
tc_bwd_state_kernel(const __grid_constant__ CUtensorMap mdo, const __grid_constant__ CUtensorMap mv,
                    const __grid_constant__ CUtensorMap mw, const __grid_constant__ CUtensorMap mdv,
                    const __grid_constant__ CUtensorMap mdw, const float *__restrict__ dST,
                    float *__restrict__ dS0, void *__restrict__ dv_out, void *__restrict__ dw_out,
                    unsigned char *__restrict__ ws, TcWs lay, SegPass sp, unsigned int *status, Dims d) {
    using namespace tbs;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    // 0, 1 records of stages 0, 1; 2 dO; 3 (unused); 4 v and w;
    // 5 dDelta ready; 6 dS ready; 7 dU ready
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 64);
    float big = 0.f;  // range check: operand magnitude

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, n = blockIdx.z;
    // this CTA's task (SegPass in common.cuh): a real run of segment sg, or in
    // the first pass of a split sequence a run from a zero exit gradient (R_s)
    int vh, sg = 0, mode = 0;  // mode 0 real, 1 from zero
    {
        const int x = blockIdx.x;
        if (sp.P == 1) { vh = x; }
        else if (sp.phase == 2) { sg = x >> 1; vh = x & 1; }
        else if (x < 2) { sg = sp.P - 1; vh = x; }
        else { mode = 1; sg = 1 + ((x - 2) >> 1); vh = (x - 2) & 1; }
    }
    const int v0 = vh * 64;
    // sequence n: tokens bos .. bos + T - 1 of batch row bb, chunks NC; a
    // segment narrows these to its own chunks
    const Seq sq = seq_of(d, n);
    int NC = sq.nc, T = sq.len, bos = sq.bos;
    const int bb = sq.brow;
    const size_t bhx = (size_t)n * d.H + h;
    size_t tile0 = (size_t)tile_of(d, sq, h, 0);  // workspace tile of the run's first chunk
    if (sp.P > 1) {
        const int L = seg_len(NC, sp.P), cb = sg * L;
        NC = min(L, NC - cb);
        T = min(T - 64 * cb, 64 * NC);
        bos += 64 * cb;
        tile0 += cb;
    }
    // the exit gradient (null: zero) and where the entry gradient goes (null:
    // nowhere); only real runs write dv, dw, -dU and dS'
    const bool real = mode == 0;
    const GateAct ga = ACT ? gate_act(d.act) : GateAct{false, 1.f};  // logits in: w activated on load, dw by the chain rule
    const float *ext = !real ? nullptr
                     : (sp.P == 1 || sg == sp.P - 1) ? (dST ? dST + st_off(d, n, h) : nullptr)
                     : seg_buf(sp, bhx, sg, SEG_ENTRY);
    float *fin = !real ? seg_buf(sp, bhx, sg, SEG_ZERO)
               : (sp.P == 1 || sg == 0) ? (dS0 ? dS0 + st_off(d, n, h) : nullptr)
               : (sp.phase == 1 ? seg_buf(sp, bhx, sp.P - 2, SEG_ENTRY) : nullptr);
    const bool compute = tid < kCompute, issuer = tid == kCompute, copier = tid == kCompute + 32;
    const bool copy_warp = warp == kCompute / 32 + 1;
    const int quarter = warp & 3, half = (warp >> 2) & 1;
    const int key = quarter * 32 + lane;
    const unsigned char *recs = ws + lay.rec + tile0 * (size_t)REC_BYTES;
    if (NC <= 0) {  // an empty sequence: dS0 = dS_T
        if (fin && tid < 256) {
            const size_t so = (size_t)(tid >> 1) * 128 + v0 + 32 * (tid & 1);
            for (int j = 0; j < 32; ++j) fin[so + j] = ext ? ext[so + j] : 0.f;
        }
        return;
    }

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    int issued[5] = {0, 0, 0, 0, 0};  // loads requested per barrier (the copier)
    int groups[3] = {0, 0, 0};        // commits to barriers 5, 6, 7 (the issuer)
    auto load_rec = [&](int cc) {
        const int s = cc & 1;
        mbar_expect_tx(&bars[s], REC_BYTES);
        bulk_load(sm + STG + s * REC_BYTES, recs + (size_t)cc * REC_BYTES, REC_BYTES, &bars[s]);
        ++issued[s];
    };
    auto load_do = [&](int cc) {
        mbar_expect_tx(&bars[2], 8192);
        tma_load_4d(sm + RAW_DO, &mdo, v0, h, bos + cc * 64, bb, &bars[2]);
        ++issued[2];
    };
    auto load_vw = [&](int cc) {
        mbar_expect_tx(&bars[4], 8192 + (GB ? 8192 : 16384));
        tma_load_4d(sm + VV, &mv, v0, h, bos + cc * 64, bb, &bars[4]);
        tma_load_4d(sm + VW, &mw, v0, h, bos + cc * 64, bb, &bars[4]);
        if (!GB) tma_load_4d(sm + VW + 8192, &mw, v0 + 32, h, bos + cc * 64, bb, &bars[4]);
        ++issued[4];
    };
    // the frame factor s of chunk cc (1 for the chunk-start frame)
    auto rec_s = [&](int cc) {
        const float sv = reinterpret_cast<const float *>(sm + STG + (cc & 1) * REC_BYTES + REC_FAC)[128 + key];
        return sv < 0.f ? 1.f : sv;
    };
    // dO of chunk cc in RAW_DO -> fp16 operand (each thread 16 values); rows
    // past the sequence's end (a packed layout's next sequence) count as zero
    auto convert_do = [&](int cc) {
        const int r = tid >> 2, cg = tid & 3;
        uint4 d0 = *reinterpret_cast<const uint4 *>(sm + RAW_DO + r * 128 + cg * 32);
        uint4 d1 = *reinterpret_cast<const uint4 *>(sm + RAW_DO + r * 128 + cg * 32 + 16);
        if (r >= T - 64 * cc) d0 = d1 = make_uint4(0u, 0u, 0u, 0u);
        const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(&d0);
        const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&d1);
        float x[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[2 * e] = __low2float(a[e]);
            x[2 * e + 1] = __high2float(a[e]);
            x[8 + 2 * e] = __low2float(b2[e]);
            x[8 + 2 * e + 1] = __high2float(b2[e]);
        }
        st_h8(sm + OP_DO + sw128_chunk(r, 2 * cg, 64), x);
        st_h8(sm + OP_DO + sw128_chunk(r, 2 * cg + 1, 64), x + 8);
        big = absmax8(x, big);
        big = absmax8(x + 8, big);
    };
    // dS' of the next chunk cc to process: diag(gamma / s) dS' into TMEM (the
    // products add the rest of dS_c / s to it), r dS' as the fp16 operand
    // (this thread's row, 32 columns); r = 1, or gamma / s for a mild chunk
    auto put_ds = [&](const float *x, int cc) {
        const float *fac = reinterpret_cast<const float *>(sm + STG + (cc & 1) * REC_BYTES + REC_FAC);
        const float gam = fac[key], sv = fac[128 + key];
        const float g_s = sv < 0.f ? gam : gam / sv, r = sv < 0.f ? 1.f : gam / sv;
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = g_s * x[j];
        tmem_st16(taddr(tm + TM_DS, quarter * 32, 32 * half), y);
        tmem_st16(taddr(tm + TM_DS, quarter * 32, 32 * half + 16), y + 16);
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = r * x[j];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            st_h8(sm + OP_DS + sw128_chunk(key, 4 * half + jj, 128), y + 8 * jj);
            big = absmax8(y + 8 * jj, big);
        }
    };
    // dU of chunk cc (TMEM) -> dv, dw in place of v, w; -dU staged (compute
    // threads; the copier stores them after the next barrier: store_du)
    auto flush_du = [&](int cc, uint32_t vw_par, uint32_t du_par) {
        bool fine = mbar_wait(&bars[7], du_par, kWait);
        fine = mbar_wait(&bars[4], vw_par, kWait) && fine;
        fence_after_sync();
        float du[16];
        tmem_ld16x256x4(taddr(tm + TM_DU, quarter * 32, 32 * half), du);
        tmem_wait_ld();
        {
            // 16x256b: rows quarter * 16 + t/4 and + 8, column pairs 32 * half +
            // 8 jb + 2 (t % 4); dv, dw in place of v, w and -dU, pair by pair
            const int rA = quarter * 16 + (lane >> 2), cp0 = 32 * half + 2 * (lane & 3);
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int rr = rA + 8 * (p & 1), jb = p >> 1, c = cp0 + 8 * jb;
                const float u0 = du[4 * jb + 2 * (p & 1)], u1 = du[4 * jb + 2 * (p & 1) + 1];
                unsigned char *pv = sm + VV + sw128_off(rr, c, 64);
                unsigned char *pw = sm + VW + (GB ? sw128_off(rr, c, 64)
                                                  : (c >> 5) * 8192 + sw128_chunk(rr, (c & 31) >> 2, 64) + (c & 3) * 4);
                const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(pv));
                const float2 wx = gld2<GB>(pw);  // w, or its logit
                const float2 wf = act_w2(ga, wx);
                *reinterpret_cast<uint32_t *>(pv) = pack_bf16(u0 * wf.x, u1 * wf.y);
                // dw = dU v, times dw/dx for logits
                gst2<GB>(pw, u0 * vf.x * ga.dw(wx.x), u1 * vf.y * ga.dw(wx.y));
                *reinterpret_cast<uint32_t *>(sm + NDU + sw128_off(rr, c, 64)) = pack_f16(-u0, -u1);
                big = fmaxf(big, fmaxf(fabsf(u0), fabsf(u1)));
            }
        }
        fence_proxy_async();
        return fine;
    };
    // the copy warp: dv, dw and -dU of chunk cc out, then the v, w tiles of
    // chunk cc - 1.  A chunk that ends inside a packed layout (rows past its
    // sequence's end belong to the next sequence) leaves row by row from the
    // whole warp instead of by TMA stores, which would write all 64 rows.
    auto store_du = [&](int cc) {
        const int L = T - 64 * cc;
        if (!real) {
            // a run from a zero exit gradient keeps only its entry gradient
        } else if (d.cu && L < 64) {
            __nv_bfloat16 *dvp = reinterpret_cast<__nv_bfloat16 *>(dv_out);
            for (int i = lane; i < L * 8; i += 32) {  // dv: 8 chunks of 8 bf16 per row
                const int r = i >> 3, j = i & 7;
                const size_t row = tok(d, bb, bos + 64 * cc + r, h, 128) + v0;
                *reinterpret_cast<uint4 *>(dvp + row + 8 * j) =
                    *reinterpret_cast<const uint4 *>(sm + VV + sw128_chunk(r, j, 64));
                if constexpr (GB) {
                    *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(dw_out) + row + 8 * j) =
                        *reinterpret_cast<const uint4 *>(sm + VW + sw128_chunk(r, j, 64));
                } else {  // two [64][32] float32 boxes: 4 floats per 16-byte chunk
                    for (int x = 0; x < 2; ++x)
                        *reinterpret_cast<uint4 *>(reinterpret_cast<float *>(dw_out) + row + 32 * x + 4 * j) =
                            *reinterpret_cast<const uint4 *>(sm + VW + x * 8192 + sw128_chunk(r, j, 64));
                }
            }
            fence_proxy_async();
            __syncwarp();
        } else if (lane == 0) {
            tma_store_4d(&mdv, sm + VV, v0, h, bos + cc * 64, bb);
            tma_store_4d(&mdw, sm + VW, v0, h, bos + cc * 64, bb);
            if (!GB) tma_store_4d(&mdw, sm + VW + 8192, v0 + 32, h, bos + cc * 64, bb);
        }
        if (lane == 0) {
            if (real) bulk_store(ws + lay.ckndU + ((tile0 + cc) * 2 + vh) * 8192, sm + NDU, 8192);
            bulk_commit();
            bulk_wait_read();  // VV, VW and NDU may be rewritten
            if (cc > 0) load_vw(cc - 1);
            if (cc > 1) {  // the v, w after those into L2, so that their copy takes the L2 latency
                tma_prefetch_4d(&mv, v0, h, bos + (cc - 2) * 64, bb);
                tma_prefetch_4d(&mw, v0, h, bos + (cc - 2) * 64, bb);
                if (!GB) tma_prefetch_4d(&mw, v0 + 32, h, bos + (cc - 2) * 64, bb);
            }
            if (cc > 3) tma_prefetch_4d(&mdo, v0, h, bos + (cc - 4) * 64, bb);  // dO two requests ahead
        }
    };

    if (copier) {
        load_rec(NC - 1);
        if (NC > 1) load_rec(NC - 2);
        load_do(NC - 1);
        load_vw(NC - 1);
    }
    // ---------------- prologue: dS' = dS_T (or zero) for the last chunk; dO
    bool ok = true;
    if (compute) {
        float x[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 t = ext ? *reinterpret_cast<const float4 *>(ext + (size_t)key * 128 + v0 + 32 * half + j)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            x[j] = t.x; x[j + 1] = t.y; x[j + 2] = t.z; x[j + 3] = t.w;
        }
        ok = mbar_wait(&bars[(NC - 1) & 1], 0, kWait);
        ok = mbar_wait(&bars[2], 0, kWait) && ok;
        put_ds(x, NC - 1);
        convert_do(NC - 1);
        tmem_wait_st();
    }
    fence_proxy_async();
    fence_before_sync();
    bool abort = __syncthreads_or(!ok);
    if (!abort && copier) {
        fence_after_sync();
        if (real) bulk_store(ws + lay.ckdS + ((tile0 + NC - 1) * 2 + vh) * 16384, sm + OP_DS, 16384);
        bulk_commit();
        if (NC > 1) load_do(NC - 2);
        bulk_wait_read();  // the dS' copy has left OP_DS
    }

    for (int i = 0; i < NC && !abort; ++i) {
        const int c = NC - 1 - i;
        const uint32_t par = i & 1;
        unsigned char *stg = sm + STG + (c & 1) * REC_BYTES;
        // ---------------- (1) dDelta products, then Qb^T dO
        if (!copier) ok = mbar_wait(&bars[c & 1], (i >> 1) & 1, kWait) && ok;  // record c
        if (issuer) {
            const uint32_t st = smem_addr(stg);
            // Qb is rows 64..127 of the [-W; Qb] tile: 64-key blocks 16 KB apart
            const uint64_t dP = desc_mnmajor(st + REC_P, 64, 0), dO = desc_mnmajor(smem_addr(sm + OP_DO), 64, 0),
                           dK = desc_kmajor(st + REC_KH, 64, 0), dX = desc_mnmajor(smem_addr(sm + OP_DS), 128, 0),
                           dQ = desc_mnmajor_lbo(st + REC_WQ + 8192, 16384, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_DD, kstep_mnmajor(dP, ks), kstep_mnmajor(dO, ks), ID_MM64, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_DD, kstep_kmajor(dK, 64, ks), kstep_mnmajor(dX, ks), ID_KM64, 1);
            mma_commit(&bars[5]);
            ++groups[0];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_DS, kstep_mnmajor(dQ, ks), kstep_mnmajor(dO, ks), ID_MM128x64, 1);
        }
        // the next chunk's dU, while these products run
        if (compute && c + 1 < NC) ok = flush_du(c + 1, (i - 1) & 1, (i - 1) & 1) && ok;
        // ---------------- dDelta to fp16, (2) products
        if (compute) {
            ok = mbar_wait(&bars[5], par, kWait) && ok;
            fence_after_sync();
            float dd[16];
            tmem_ld16x256x4(taddr(tm + TM_DD, quarter * 32, 32 * half), dd);
            tmem_wait_ld();
            const int rA = quarter * 16 + (lane >> 2), cp0 = 32 * half + 2 * (lane & 3);
#pragma unroll
            for (int p = 0; p < 8; ++p) {  // 16x256b pairs, as in the dU flush
                const int rr = rA + 8 * (p & 1), jb = p >> 1, c = cp0 + 8 * jb;
                const float x0 = dd[4 * jb + 2 * (p & 1)], x1 = dd[4 * jb + 2 * (p & 1) + 1];
                *reinterpret_cast<uint32_t *>(sm + OP_DD + sw128_off(rr, c, 64)) = pack_f16(x0, x1);
                big = fmaxf(big, fmaxf(fabsf(x0), fabsf(x1)));
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (copy_warp && c + 1 < NC) store_du(c + 1);
        if (issuer) {
            fence_after_sync();
            const uint32_t st = smem_addr(stg);
            const uint64_t dW = desc_mnmajor_lbo(st + REC_WQ, 16384, 0), dT = desc_mnmajor(st + REC_T, 64, 0),
                           dD = desc_mnmajor(smem_addr(sm + OP_DD), 64, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_DS, kstep_mnmajor(dW, ks), kstep_mnmajor(dD, ks), ID_MM128x64, 1);
            mma_commit(&bars[6]);
            ++groups[1];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_DU, kstep_mnmajor(dT, ks), kstep_mnmajor(dD, ks), ID_MM64, ks > 0);
            mma_commit(&bars[7]);
            ++groups[2];
        }
        // ---------------- dS_c: dS' of chunk c - 1; its dO
        if (compute) {
            ok = mbar_wait(&bars[6], par, kWait) && ok;
            if (c > 0) {
                ok = mbar_wait(&bars[(c - 1) & 1], ((i + 1) >> 1) & 1, kWait) && ok;  // record c-1
                ok = mbar_wait(&bars[2], (i + 1) & 1, kWait) && ok;                 // dO of chunk c-1
            }
            fence_after_sync();
            float sv[32];
            tmem_ld16(taddr(tm + TM_DS, quarter * 32, 32 * half), sv);
            tmem_ld16(taddr(tm + TM_DS, quarter * 32, 32 * half + 16), sv + 16);
            tmem_wait_ld();
            const float se = rec_s(c);  // tensor memory holds dS_c / s
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] *= se;
            if (c == 0) {
                if (fin) {
                    float *dst = fin + (size_t)key * 128 + v0 + 32 * half;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(dst + j) = make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
                }
            } else {
                put_ds(sv, c - 1);
                convert_do(c - 1);
                tmem_wait_st();
            }
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (c > 0) {
            if (copier) {
                fence_after_sync();
                if (real) bulk_store(ws + lay.ckdS + ((tile0 + c - 1) * 2 + vh) * 16384, sm + OP_DS, 16384);
                bulk_commit();
                if (c >= 2) {
                    load_do(c - 2);           // raw dO consumed
                    // this chunk's record is consumed once T^T dDelta has read T
                    if (!mbar_wait(&bars[7], par, kWait)) record_status(status, GDN2_ERR_TIMEOUT);
                    load_rec(c - 2);
                    // and the one after it into L2, so that its copy takes the L2 latency
                    if (c >= 3) bulk_prefetch_l2(recs + (size_t)(c - 3) * REC_BYTES, REC_BYTES);
                }
                bulk_wait_read();  // the dS' copy has left OP_DS before it is rewritten
            }
        }
    }
    if (!abort && compute) ok = flush_du(0, (NC - 1) & 1, (NC - 1) & 1);
    fence_before_sync();
    const bool bad = __syncthreads_or(abort || !ok);
    if (!bad && copy_warp) store_du(0);
    if (!(big <= kRange)) record_status(status, GDN2_ERR_RANGE);
    if (copier) bulk_wait_all();
    if (bad && copier) {
        record_status(status, GDN2_ERR_TIMEOUT);
        for (int k2 = 0; k2 < 5; ++k2)
            if (issued[k2] > 0) mbar_wait(&bars[k2], (issued[k2] - 1) & 1, kWait);
    }
    if (bad && issuer) {
        for (int k2 = 0; k2 < 3; ++k2)
            if (groups[k2] > 0) mbar_wait(&bars[5 + k2], (groups[k2] - 1) & 1, kWait);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

// ---------------------------------------------------------------- launcher
// the gradient kernel (tc_bwd_grad.cu), launched after the state pass on the same stream
cudaError_t tc_bwd_grad_launch(const void *q, const void *k, const void *g, const void *b,
                               const void *dO, void *dq, void *dk, void *dg, void *db, void *ws,
                               unsigned int *status, const Dims &d, cudaStream_t s);

// the link step between the passes (seg_link.cu)
cudaError_t seg_link_launch(const SegPass &sp, int nbh, bool backward, cudaStream_t s);

template <bool GB, bool ACT>
static cudaError_t tc_bwd_state_run(const void *v, const void *w, const void *dO, const float *dST,
                                    void *dv, void *dw, float *dS0, void *ws, unsigned int *status,
                                    const Dims &d, cudaStream_t s) {
    CUtensorMap mdo_half, mv, mw, mdv, mdw;
    if (!make_btHd_map(&mdo_half, dO, true, d.B, d.T, d.H, 128, 64, 64) ||
        !make_btHd_map(&mv, v, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mw, w, GB, d.B, d.T, d.H, 128, 64, gate_box_cols<GB>(), true) ||
        !make_btHd_map(&mdv, dv, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mdw, dw, GB, d.B, d.T, d.H, 128, 64, gate_box_cols<GB>(), true))
        return cudaErrorInvalidValue;
    const TcWs lay = tc_ws_layout(d);
    cudaError_t e = cudaFuncSetAttribute(tc_bwd_state_kernel<GB, ACT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tbs::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // a split sequence takes the maps M_s the split forward left in the workspace
    SegPass sp{1, 0, nullptr};
    if (lay.P > 1) sp = SegPass{lay.P, 1, reinterpret_cast<float *>(static_cast<char *>(ws) + lay.seg)};
    launch_begin(K_TC_BWD_STATE, s);
    tc_bwd_state_kernel<GB, ACT><<<dim3(sp.P > 1 ? 2 * (sp.P - 1) : 2, d.H, num_seqs(d)), tbs::kThreads,
                              tbs::SMEM_BYTES, s>>>(mdo_half, mv, mw, mdv, mdw, dST, dS0, dv, dw,
                                                    (unsigned char *)ws, lay, sp, status, d);
    launch_end(K_TC_BWD_STATE, s);
    if (sp.P > 1) {
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = seg_link_launch(sp, d.B * d.H, true, s)) != cudaSuccess) return e;
        sp.phase = 2;
        launch_begin(K_TC_BWD_STATE, s);
        tc_bwd_state_kernel<GB, ACT><<<dim3(2 * (sp.P - 1), d.H, d.B), tbs::kThreads, tbs::SMEM_BYTES, s>>>(
            mdo_half, mv, mw, mdv, mdw, dST, dS0, dv, dw, (unsigned char *)ws, lay, sp, status, d);
        launch_end(K_TC_BWD_STATE, s);
    }
    return cudaGetLastError();
}

cudaError_t tc_bwd_launch(const void *q, const void *k, const void *v, const void *g,
                          const void *b, const void *w, const void *dO, const float *dST,
                          void *dq, void *dk, void *dv, void *dg, void *db, void *dw,
                          float *dS0, void *ws, unsigned int *status, const Dims &d,
                          cudaStream_t s) {
    cudaError_t e =
        d.act ? (d.gb ? tc_bwd_state_run<true, true>(v, w, dO, dST, dv, dw, dS0, ws, status, d, s)
                      : tc_bwd_state_run<false, true>(v, w, dO, dST, dv, dw, dS0, ws, status, d, s))
              : (d.gb ? tc_bwd_state_run<true, false>(v, w, dO, dST, dv, dw, dS0, ws, status, d, s)
                      : tc_bwd_state_run<false, false>(v, w, dO, dST, dv, dw, dS0, ws, status, d, s));
    if (e != cudaSuccess) return e;
    return tc_bwd_grad_launch(q, k, g, b, dO, dq, dk, dg, db, ws, status, d, s);
}

}  // namespace gdn2
