// Gate-aware chunkwise backward of Gated Delta Rule-2 on the sm_100a tensor
// cores (bf16 I/O, d_k = d_v = 128, chunk 64), after the forward has left
// its chunk records (T, P among them), chunk states and Delta in the workspace.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B, D.6; digg thread 11/): the per-channel gates cannot be pulled
// out of the products that accumulate the gradient of the strictly-lower A,
// so they stay inside them: b enters dA and dKc through Kc in every channel
// sum below.
//
// Chunk equations (decay factors relative to the chunk's middle row m, see
// tc_common.cuh; dS = dL/dS_next entering the chunk from the right):
//   dS_m  = diag(e^(G_L-G_m)) dS
//   dDelta = P^T dO + Kh dS_m,         dU = T^T dDelta,   dw = dU.v, dv = dU.w
//   dS_c  = diag(e^G_m) (dS_m + Qb^T dO - W^T dDelta)             (carried left)
//   (W^T dDelta = Kc^T dU, since W = T Kc)
//   S_m   = diag(e^G_m) S_c
//   dP = lower-incl(dO Delta^T),       dA = -strictly-lower(dU Delta^T)
//   Y1 = dO S_m^T + dP Kh              dq  = Y1.E
//   Y2 = -dU S_m^T + dA Kh             dKc.e^G = Y2.E,  db = Y2.E.k
//   Y3 = Delta dS_m^T + dP^T Qb + dA^T Kc            dk = Y2.E.b + Y3/E
//   dG = dq.q + Y2.E.b.k - (Y3/E).k, plus rowsum(dS . S_next) on the last row
//   dg = reverse in-chunk cumsum of dG
// (E = e^(G - G_m); the chunk-end term rowsum(dS_next . S_next) is the
// derivative through the chunk's total decay, since S_next = e^G_L (...).)
//
// Two kernels:
//  * tc_bwd_state_kernel: one CTA per (b, h, half of d_v), walking the chunks
//    in reverse with dS in tensor memory and the chunk records double-
//    buffered; two tcgen05.mma round trips per chunk on the state's path
//    (dDelta; then dS), with dU and its outputs off that path.  Writes dw,
//    dv, dS0, and per chunk dS_m, -dU and the half-sums of the chunk-end
//    term to the workspace.
//  * tc_bwd_grad_kernel: persistent, one CTA per SM walking the (b, h, chunk)
//    tiles, all chunks in parallel, full d_v; five products, then three
//    accumulations, then dq, dk, db, dg.

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
constexpr uint32_t STG_S = OP_DD + 8192;      // checkpoint S_m fp16 [128 key][64 v]
constexpr uint32_t VV = STG_S + 16384;        // v half bf16 [64][64], 128-B swizzled; dv in place
constexpr uint32_t VW = VV + 8192;            // w half f32, two [64][32] 128-B swizzled boxes; dw in place
constexpr uint32_t NDU = VW + 16384;          // -dU fp16 [64 pos][64 v] (the workspace layout)
constexpr uint32_t MISC = NDU + 8192;         // sEnd [2][128] f32; mbarriers; TMEM slot
constexpr uint32_t SMEM_BYTES = MISC + 1024 + 128 + 1024;
constexpr uint32_t TM_DS = 0, TM_DD = 64, TM_DU = 128;  // 256 columns allocated
constexpr uint32_t ID_MM64 = idesc_f16(64, 64, true, true);
constexpr uint32_t ID_KM64 = idesc_f16(64, 64, false, true);
constexpr uint32_t ID_MM128x64 = idesc_f16(128, 64, true, true);
constexpr long long kWait = 2000000000LL;
constexpr float kRange = 6.0e4f;
static_assert(MISC % 1024 == 0, "alignment");
}  // namespace tbs

// One CTA per (b, h, half of d_v), walking the chunks in reverse with
// dX = diag(e^(G_L - G_m)) dS_next in tensor memory.  Per chunk, from the
// chunk's record (Qb, Kh, -W, T, P, factors):
//   (1) dDelta = P^T dO + Kh dX  (committed alone),  then dS_m = dX + Qb^T dO
//   (2) dS_m += (-W)^T dDelta  (committed alone),     then dU = T^T dDelta
// then dS_c = diag(e^G_m) dS_m and the previous chunk's dX = diag(e^(G_L -
// G_m)) dS_c.  dU is read while the next chunk's first products run: dv =
// dU.w and dw = dU.v are formed in place of the v and w tiles (128-B
// swizzled TMA tiles) and leave by TMA stores; -dU, dX and the chunk-end
// half-sums go to the workspace for the gradient kernel.  Warps 0..7 read
// the accumulators and form the operands and outputs; warp 8 issues the
// products (an issuing thread is held for about as long as the products
// run); warp 9 requests every copy, so that neither delays the readouts.
__global__ void __launch_bounds__(tbs::kThreads, 1)
tc_bwd_state_kernel(const __grid_constant__ CUtensorMap mdo, const __grid_constant__ CUtensorMap mv,
                    const __grid_constant__ CUtensorMap mw, const __grid_constant__ CUtensorMap mdv,
                    const __grid_constant__ CUtensorMap mdw, const float *__restrict__ dST,
                    float *__restrict__ dS0, unsigned char *__restrict__ ws, TcWs lay,
                    unsigned int *status, Dims d) {
    using namespace tbs;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *sEnd = reinterpret_cast<float *>(sm + MISC);  // [2][128]
    // 0, 1 records of stages 0, 1; 2 dO; 3 state checkpoint; 4 v and w;
    // 5 dDelta ready; 6 dS ready; 7 dU ready
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC + 1024);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 1024 + 64);
    float big = 0.f;  // range check: operand magnitude

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int vh = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, v0 = vh * 64;
    const int NC = d.NC, H = d.H;
    const bool compute = tid < kCompute, issuer = tid == kCompute, copier = tid == kCompute + 32;
    const int quarter = warp & 3, half = (warp >> 2) & 1;
    const int key = quarter * 32 + lane;
    const size_t bh = (size_t)bb * H + h;
    const unsigned char *recs = ws + lay.rec + bh * NC * (size_t)REC_BYTES;

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
        tma_load_4d(sm + RAW_DO, &mdo, v0, h, cc * 64, bb, &bars[2]);
        ++issued[2];
    };
    auto load_s = [&](int slot) {  // state checkpoint `slot` of this half
        mbar_expect_tx(&bars[3], 16384);
        bulk_load(sm + STG_S, ws + lay.ckS + ((bh * (NC + 1) + slot) * 2 + vh) * 16384, 16384, &bars[3]);
        ++issued[3];
    };
    auto load_vw = [&](int cc) {
        mbar_expect_tx(&bars[4], 8192 + 16384);
        tma_load_4d(sm + VV, &mv, v0, h, cc * 64, bb, &bars[4]);
        tma_load_4d(sm + VW, &mw, v0, h, cc * 64, bb, &bars[4]);
        tma_load_4d(sm + VW + 8192, &mw, v0 + 32, h, cc * 64, bb, &bars[4]);
        ++issued[4];
    };
    auto rec_fac = [&](int cc) {  // e^(G_L - G_m) of chunk cc (then e^G_m at +128)
        return reinterpret_cast<const float *>(sm + STG + (cc & 1) * REC_BYTES + REC_FAC);
    };
    // dO of the chunk in RAW_DO -> fp16 operand (each thread 16 values)
    auto convert_do = [&]() {
        const int r = tid >> 2, cg = tid & 3;
        const uint4 d0 = *reinterpret_cast<const uint4 *>(sm + RAW_DO + r * 128 + cg * 32);
        const uint4 d1 = *reinterpret_cast<const uint4 *>(sm + RAW_DO + r * 128 + cg * 32 + 16);
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
    // dX of chunk c into TMEM and the fp16 operand (this thread's row, 32 columns)
    auto put_dx = [&](float *x) {
        tmem_st16(taddr(tm + TM_DS, quarter * 32, 32 * half), x);
        tmem_st16(taddr(tm + TM_DS, quarter * 32, 32 * half + 16), x + 16);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            st_h8(sm + OP_DS + sw128_chunk(key, 4 * half + jj, 128), x + 8 * jj);
            big = absmax8(x + 8 * jj, big);
        }
    };
    // rowsum over this thread's 32 columns of x . S (S from STG_S)
    auto end_term = [&](const float *x) {
        float acc = 0.f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            float s8[8];
            ld_h8(sm + STG_S + sw128_chunk(key, 4 * half + jj, 128), s8);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc += x[8 * jj + e] * s8[e];
        }
        return acc;
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
                unsigned char *pw = sm + VW + (c >> 5) * 8192 + sw128_chunk(rr, (c & 31) >> 2, 64) + (c & 3) * 4;
                const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(pv));
                const float2 wf = *reinterpret_cast<const float2 *>(pw);
                *reinterpret_cast<uint32_t *>(pv) = pack_bf16(u0 * wf.x, u1 * wf.y);
                *reinterpret_cast<float2 *>(pw) = make_float2(u0 * vf.x, u1 * vf.y);
                *reinterpret_cast<uint32_t *>(sm + NDU + sw128_off(rr, c, 64)) = pack_f16(-u0, -u1);
                big = fmaxf(big, fmaxf(fabsf(u0), fabsf(u1)));
            }
        }
        fence_proxy_async();
        return fine;
    };
    // the copier: dv, dw and -dU of chunk cc out, then the v, w tiles of chunk cc - 1
    auto store_du = [&](int cc) {
        tma_store_4d(&mdv, sm + VV, v0, h, cc * 64, bb);
        tma_store_4d(&mdw, sm + VW, v0, h, cc * 64, bb);
        tma_store_4d(&mdw, sm + VW + 8192, v0 + 32, h, cc * 64, bb);
        bulk_store(ws + lay.ckndU + ((bh * NC + cc) * 2 + vh) * 8192, sm + NDU, 8192);
        bulk_commit();
        bulk_wait_read();  // VV, VW and NDU may be rewritten
        if (cc > 0) load_vw(cc - 1);
    };

    if (copier) {
        load_rec(NC - 1);
        if (NC > 1) load_rec(NC - 2);
        load_do(NC - 1);
        load_s(NC);
        load_vw(NC - 1);
    }
    // ---------------- prologue: dS_T (or zero), the last chunk's end term and dX; dO
    bool ok = true;
    if (compute) {
        float x[32];
        const size_t so = st_off(d, bb, h);
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 t = dST ? *reinterpret_cast<const float4 *>(dST + so + (size_t)key * 128 + v0 + 32 * half + j)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            x[j] = t.x; x[j + 1] = t.y; x[j + 2] = t.z; x[j + 3] = t.w;
        }
        ok = mbar_wait(&bars[3], 0, kWait);
        ok = mbar_wait(&bars[(NC - 1) & 1], 0, kWait) && ok;
        ok = mbar_wait(&bars[2], 0, kWait) && ok;
        sEnd[half * 128 + key] = end_term(x);  // the last checkpoint is S_T itself
        const float gam = rec_fac(NC - 1)[key];
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] *= gam;
        put_dx(x);
        convert_do();
        tmem_wait_st();
    }
    fence_proxy_async();
    fence_before_sync();
    bool abort = __syncthreads_or(!ok);
    if (!abort) {
        if (compute && half == 0)
            reinterpret_cast<float *>(ws + lay.ckEnd + ((bh * NC + NC - 1) * 2 + vh) * 512)[key] =
                sEnd[key] + sEnd[128 + key];
        if (copier) {
            fence_after_sync();
            bulk_store(ws + lay.ckdS + ((bh * NC + NC - 1) * 2 + vh) * 16384, sm + OP_DS, 16384);
            bulk_commit();
            if (NC > 1) {
                load_s(NC - 1);
                load_do(NC - 2);
            }
            bulk_wait_read();  // the dX copy has left OP_DS
        }
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
        if (copier && c + 1 < NC) store_du(c + 1);
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
        // ---------------- dS_c; the previous chunk's end term, dX and dO
        if (compute) {
        ok = mbar_wait(&bars[6], par, kWait) && ok;
        if (c > 0) {
            ok = mbar_wait(&bars[3], (i + 1) & 1, kWait) && ok;                 // S_m of chunk c
            ok = mbar_wait(&bars[(c - 1) & 1], ((i + 1) >> 1) & 1, kWait) && ok;  // record c-1
            ok = mbar_wait(&bars[2], (i + 1) & 1, kWait) && ok;                 // dO of chunk c-1
        }
        fence_after_sync();
        {
            float sv[32];
            tmem_ld16(taddr(tm + TM_DS, quarter * 32, 32 * half), sv);
            tmem_ld16(taddr(tm + TM_DS, quarter * 32, 32 * half + 16), sv + 16);
            tmem_wait_ld();
            const float e = reinterpret_cast<const float *>(stg + REC_FAC)[128 + key];
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] *= e;  // dS_c
            if (c == 0) {
                if (dS0) {
                    float *dst = dS0 + st_off(d, bb, h) + (size_t)key * 128 + v0 + 32 * half;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(dst + j) = make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
                }
            } else {
                // the checkpoint holds S_m = diag(e^G_m) S_c
                sEnd[half * 128 + key] = end_term(sv) / e;
                const float gam = rec_fac(c - 1)[key];
#pragma unroll
                for (int j = 0; j < 32; ++j) sv[j] *= gam;
                put_dx(sv);
                convert_do();
                tmem_wait_st();
            }
        }
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (c > 0) {
            if (compute && half == 0)
                reinterpret_cast<float *>(ws + lay.ckEnd + ((bh * NC + c - 1) * 2 + vh) * 512)[key] =
                    sEnd[key] + sEnd[128 + key];
            if (copier) {
                fence_after_sync();
                bulk_store(ws + lay.ckdS + ((bh * NC + c - 1) * 2 + vh) * 16384, sm + OP_DS, 16384);
                bulk_commit();
                load_s(c - 1);                // S_m of chunk c consumed
                if (c >= 2) {
                    load_do(c - 2);           // raw dO consumed
                    // this chunk's record is consumed once T^T dDelta has read T
                    if (!mbar_wait(&bars[7], par, kWait)) record_status(status, GDN2_ERR_TIMEOUT);
                    load_rec(c - 2);
                }
                bulk_wait_read();  // the dX copy has left OP_DS before it is rewritten
            }
        }
    }
    if (!abort && compute) ok = flush_du(0, (NC - 1) & 1, (NC - 1) & 1);
    fence_before_sync();
    const bool bad = __syncthreads_or(abort || !ok);
    if (!bad && copier) store_du(0);
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

// ============================================================ chunk kernel
namespace tbg {
constexpr int kCompute = 512;             // warps 0..15 form operands and outputs
constexpr int kThreads = kCompute + 32;   // warp 16 issues the copies and products
constexpr int kWarps = kCompute / 32;
constexpr uint32_t RQ = 0;        // q: two 128-B swizzled [64][64] bf16 boxes; Qb, then dq, in place
constexpr uint32_t RK = 16384;    // k (bf16); dk in place
constexpr uint32_t RB = 32768;    // b: four [64][32] f32 boxes; db in place
constexpr uint32_t RG = 65536;    // g (f32); G - G_m, then dG, then dg in place
constexpr uint32_t DN = 98304;    // [dO; -dU] [128][128] K-major (K-blocks of 16 KB)
constexpr uint32_t DL = 131072;   // Delta [64 pos][128 v] K-major
constexpr uint32_t SMT = 147456;  // S_m [128 key][128 v] K-major (then Kh, Kc)
constexpr uint32_t DXT = 180224;  // dX  [128 key][128 v] K-major (then [dP; dA])
constexpr uint32_t KH = SMT, KC = SMT + 16384, PA = DXT;  // after the first products
constexpr uint32_t TE = DXT + 16384, TEI = DL;              // E = e^(G - G_m), 1/E (fp16 [64][128])
constexpr uint32_t MISC = 212992; // sEnd [2][256]; sRef [128]; scan [16][128]; mbarriers; slot
constexpr uint32_t SMEM_BYTES = MISC + 2560 + 8192 + 128 + 1024;
constexpr uint32_t LOAD_A = 114688;  // dO, -dU, Delta, S_m, dX (the first products' operands)
constexpr uint32_t LOAD_B = 98304;   // raw q, k, b, g
constexpr uint32_t TM_Y1 = 0, TM_Y2 = 128, TM_Y3 = 256, TM_PA = 384;  // 512 columns
constexpr uint32_t ID_PA = idesc_f16(128, 64, false, false);
constexpr uint32_t ID_KK128 = idesc_f16(64, 128, false, false);
constexpr uint32_t ID_KM128 = idesc_f16(64, 128, false, true);
constexpr uint32_t ID_MM128 = idesc_f16(64, 128, true, true);
constexpr long long kWait = 2000000000LL;
constexpr float kRange = 6.0e4f;
}  // namespace tbg

// descriptor of K step kstep of a K-major operand whose 64-wide K-blocks lie
// blk bytes apart (d0 = its K step 0)
__device__ __forceinline__ uint64_t kstep_kmajor_blk(uint64_t d0, uint32_t blk, int kstep) {
    return d0 + (uint64_t)((((uint32_t)(kstep >> 2) * blk) + (kstep & 3) * 32) >> 4);
}

// Persistent: one CTA per SM walks the (b, h, chunk) tiles, full d_v.  Warp 16
// loads the tile (raw q, k, b, g, dO as 128-B swizzled TMA boxes; S_m, dX,
// Delta, -dU from the workspace) and issues the products; warps 0..15 form
// the operands and the outputs:
//   (1) [dP; dA] = [dO; -dU] Delta^T (M = 128), Y1 = dO S_m^T, Y2 = -dU S_m^T,
//       Y3 = Delta dX^T, while the decay factors Qb (in place of q), Kc, Kh
//       are formed
//   (2) Y1 += dP Kh, Y2 += dA Kh, Y3 += dP^T Qb + dA^T Kc (masked dP, dA)
// then, per (row, channel) straight from tensor memory: dq = Y1.E,
// db = Y2.E.k, dk = Y2.E.b + Y3/E, dG = Y1.Qb + Y2.Kc - Y3.Kh, written in
// place of q, k, b, g; dg is the reverse in-chunk cumsum of dG plus the
// chunk-end term, and the four tiles leave by TMA stores.  Sixteen compute
// warps (four rows each in the row-wise phases) hide the latency of the
// per-element work; E and 1/E are kept as fp16 tiles between the factor
// phase and the outputs.  The next tile's copies are requested as soon as
// their buffers are free: dO and -dU after the first products, Delta, S_m
// and dX after the outputs are formed, the raw tiles once the TMA stores have
// read them.
__global__ void __launch_bounds__(tbg::kThreads, 1)
tc_bwd_grad_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mb, const __grid_constant__ CUtensorMap mg,
                   const __grid_constant__ CUtensorMap mdo, const __grid_constant__ CUtensorMap mdq,
                   const __grid_constant__ CUtensorMap mdk, const __grid_constant__ CUtensorMap mdb,
                   const __grid_constant__ CUtensorMap mdg, unsigned char *__restrict__ ws, TcWs lay,
                   unsigned int *status, Dims d) {
    using namespace tbg;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    // chunk-end term per channel as the two d_v halves' partials [2][128],
    // double-buffered by tile parity (copied in with Delta, S_m, dX)
    float *sEnd2 = reinterpret_cast<float *>(sm + MISC);
    float *sRef = reinterpret_cast<float *>(sm + MISC + 2048);  // G of the middle row per channel
    float *scan = reinterpret_cast<float *>(sm + MISC + 2560);  // per-warp totals [16][128]
    // 0 first-product operands (two parts), 1, 2 products, 3 raw tiles, 4 dO
    // converted (one arrival per compute warp)
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC + 2560 + 8192);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 2560 + 8192 + 64);
    float big = 0.f, gbig = 0.f;  // range checks: operand magnitude, |G - G_m|

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NC = d.NC, H = d.H;
    const int ntiles = d.B * H * NC;
    const int quarter = warp & 3, cgrp = (warp >> 2) & 3;  // TMEM lane quarter; column group
    const bool compute = warp < kWarps, issuer = tid == kCompute;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (issuer) {
        mbar_init(&bars[0], 2);
        for (int i = 1; i < 4; ++i) mbar_init(&bars[i], 1);
        mbar_init(&bars[4], kWarps);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    // tile `it` = (b * H + h) * NC + c; copies requested by the issuer
    int issued[3] = {0, 0, 0};  // operand parts 1, 2 and raw tiles
    auto load_a1 = [&](int it) {  // dO (TMA) and -dU: [dO; -dU]
        const int c = it % NC, bhi = it / NC, h = bhi % H, bb = bhi / H;
        mbar_expect_tx(&bars[0], 32768);
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(sm + DN + x * 16384, &mdo, 64 * x, h, c * 64, bb, &bars[0]);
            bulk_load(sm + DN + x * 16384 + 8192, ws + lay.ckndU + ((size_t)it * 2 + x) * 8192, 8192, &bars[0]);
        }
        ++issued[0];
    };
    auto load_a2 = [&](int it, int pb) {  // Delta, S_m, dX and the chunk-end partials
        mbar_expect_tx(&bars[0], LOAD_A - 32768 + 1024);
        bulk_load(sEnd2 + 256 * pb, ws + lay.ckEnd + (size_t)it * 1024, 1024, &bars[0]);
        bulk_load(sm + DL, ws + lay.ckD + ((size_t)it * 2) * 8192, 16384, &bars[0]);
        bulk_load(sm + SMT, ws + lay.ckS + ((size_t)(it + it / NC) * 2) * 16384, 32768, &bars[0]);
        bulk_load(sm + DXT, ws + lay.ckdS + ((size_t)it * 2) * 16384, 32768, &bars[0]);
        ++issued[1];
    };
    auto load_b = [&](int it) {  // raw q, k, b, g
        const int c = it % NC, bhi = it / NC, h = bhi % H, bb = bhi / H;
        mbar_expect_tx(&bars[3], LOAD_B);
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(sm + RQ + x * 8192, &mq, 64 * x, h, c * 64, bb, &bars[3]);
            tma_load_4d(sm + RK + x * 8192, &mk, 64 * x, h, c * 64, bb, &bars[3]);
        }
        for (int x = 0; x < 4; ++x) {
            tma_load_4d(sm + RB + x * 8192, &mb, 32 * x, h, c * 64, bb, &bars[3]);
            tma_load_4d(sm + RG + x * 8192, &mg, 32 * x, h, c * 64, bb, &bars[3]);
        }
        ++issued[2];
    };
    if (issuer && (int)blockIdx.x < ntiles) {
        load_a1(blockIdx.x);
        load_a2(blockIdx.x, 0);
        load_b(blockIdx.x);
    }

    bool ok = true;
    for (int it = blockIdx.x, n = 0; it < ntiles; it += gridDim.x, ++n) {
        const int c = it % NC, bhi = it / NC, h = bhi % H, bb = bhi / H, c0 = c * 64;
        const uint32_t par = n & 1;
        const int nxt = it + (int)gridDim.x;
        const bool more = nxt < ntiles;
        ok = mbar_wait(&bars[0], par, kWait) && ok;

        // ---------------- dO to fp16; then, while the first products run, the
        // cumulative decay (rows 4w..4w+3, channels 4l..4l+3)
        if (compute) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {  // the dO rows of [dO; -dU], in place
                const int i = tid + kCompute * m;
                unsigned char *p = sm + DN + (i >> 9) * 16384 + (i & 511) * 16;
                uint4 raw = *reinterpret_cast<const uint4 *>(p);
                const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
                float x[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[2 * e] = __low2float(b2[e]);
                    x[2 * e + 1] = __high2float(b2[e]);
                }
                st_h8(p, x);
            }
            // the issuer waits for this, the compute warps go on to the decay
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[4]);
        }
        if (issuer) {
            ok = mbar_wait(&bars[4], par, kWait) && ok;
            fence_after_sync();
            const uint64_t dn = desc_kmajor(smem_addr(sm + DN), 128, 0), dl = desc_kmajor(smem_addr(sm + DL), 64, 0),
                           s = desc_kmajor(smem_addr(sm + SMT), 128, 0), dx = desc_kmajor(smem_addr(sm + DXT), 128, 0),
                           ado = desc_kmajor(smem_addr(sm + DN), 64, 0), andu = desc_kmajor(smem_addr(sm + DN + 8192), 64, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t b_s = kstep_kmajor(s, 128, ks), a_dl = kstep_kmajor(dl, 64, ks);
                mma_bf16(tm + TM_PA, kstep_kmajor(dn, 128, ks), a_dl, ID_PA, ks > 0);
                mma_bf16(tm + TM_Y1, kstep_kmajor_blk(ado, 16384, ks), b_s, ID_KK128, ks > 0);
                mma_bf16(tm + TM_Y2, kstep_kmajor_blk(andu, 16384, ks), b_s, ID_KK128, ks > 0);
                mma_bf16(tm + TM_Y3, a_dl, kstep_kmajor(dx, 128, ks), ID_KK128, ks > 0);
            }
            mma_commit(&bars[1]);
        }
        float G[4][4];
        if (compute) {
            ok = mbar_wait(&bars[3], par, kWait) && ok;
            float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 t = *reinterpret_cast<const float4 *>(sm + RG + sw128_chunk(4 * warp + m, lane, 64));
                run[0] += t.x; run[1] += t.y; run[2] += t.z; run[3] += t.w;
#pragma unroll
                for (int i = 0; i < 4; ++i) G[m][i] = run[i];
            }
            *reinterpret_cast<float4 *>(scan + warp * 128 + 4 * lane) = make_float4(run[0], run[1], run[2], run[3]);
            named_sync(1, kCompute);
            if (tid < 128) {  // per channel: exclusive prefix over the warps' totals, in place
                float acc = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < kWarps; ++w2) {
                    const float t = scan[w2 * 128 + tid];
                    scan[w2 * 128 + tid] = acc;
                    acc += t;
                    if (w2 == kWarps / 2 - 1) sRef[tid] = acc;  // rows 0..31: G of the middle row
                }
            }
            named_sync(1, kCompute);
        }
        // ---------------- decay factors while the products run: Qb in place of q;
        // Kh, Kc kept in registers until S_m is consumed
        uint2 khr[4], kcr[4], er[4], eir[4];
        if (compute) {
            const float4 pre4 = *reinterpret_cast<const float4 *>(scan + warp * 128 + 4 * lane);
            const float4 ref4 = *reinterpret_cast<const float4 *>(sRef + 4 * lane);
            const float pre[4] = {pre4.x, pre4.y, pre4.z, pre4.w}, ref[4] = {ref4.x, ref4.y, ref4.z, ref4.w};
            uint2 qr[4], kr[4];
            float4 bv[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {  // every input row before the first store
                const int r = 4 * warp + m;
                qr[m] = *reinterpret_cast<const uint2 *>(sm + RQ + sw128_chunk(r, lane >> 1, 64) + (lane & 1) * 8);
                kr[m] = *reinterpret_cast<const uint2 *>(sm + RK + sw128_chunk(r, lane >> 1, 64) + (lane & 1) * 8);
                bv[m] = *reinterpret_cast<const float4 *>(sm + RB + sw128_chunk(r, lane, 64));
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = 4 * warp + m;
                float Gv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    Gv[i] = G[m][i] + pre[i] - ref[i];
                    gbig = fmaxf(gbig, fabsf(Gv[i]));
                }
                const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qr[m]);
                const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kr[m]);
                const float qf[4] = {__low2float(q2[0]), __high2float(q2[0]), __low2float(q2[1]), __high2float(q2[1])};
                const float kf[4] = {__low2float(k2[0]), __high2float(k2[0]), __low2float(k2[1]), __high2float(k2[1])};
                const float bf[4] = {bv[m].x, bv[m].y, bv[m].z, bv[m].w};
                float qb[4], kc[4], kh[4], e[4], ei[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    e[i] = __expf(Gv[i]);
                    ei[i] = __expf(-Gv[i]);
                    qb[i] = qf[i] * e[i];
                    kc[i] = bf[i] * kf[i] * e[i];
                    kh[i] = kf[i] * ei[i];
                }
                st_h4(sm + RQ + sw128_chunk(r, lane >> 1, 64) + (lane & 1) * 8, qb[0], qb[1], qb[2], qb[3]);
                khr[m] = make_uint2(pack_f16(kh[0], kh[1]), pack_f16(kh[2], kh[3]));
                kcr[m] = make_uint2(pack_f16(kc[0], kc[1]), pack_f16(kc[2], kc[3]));
                er[m] = make_uint2(pack_f16(e[0], e[1]), pack_f16(e[2], e[3]));
                eir[m] = make_uint2(pack_f16(ei[0], ei[1]), pack_f16(ei[2], ei[3]));
#pragma unroll
                for (int i = 0; i < 4; ++i) big = fmaxf(big, fmaxf(fabsf(qb[i]), fmaxf(fabsf(kc[i]), fabsf(kh[i]))));
            }
            // ---------------- masked dP, dA; Kh, Kc into the space of S_m
            ok = mbar_wait(&bars[1], par, kWait) && ok;
            fence_after_sync();
            {
                // accumulator row quarter * 32 + lane: 0..63 dP, 64..127 dA; 16 columns from 16 * cgrp
                float row[16];
                tmem_ld16(taddr(tm + TM_PA, quarter * 32, 16 * cgrp), row);
                tmem_wait_ld();
                const int pr = quarter * 32 + lane, r = pr & 63;
                // dP keeps j <= r; dA = strictly-lower of (-dU) Delta^T
#pragma unroll
                for (int j = 0; j < 16; ++j) row[j] = (pr < 64 ? 16 * cgrp + j <= r : 16 * cgrp + j < r) ? row[j] : 0.f;
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    st_h8(sm + PA + sw128_chunk(pr, 2 * cgrp + jj, 128), row + 8 * jj);
                    big = absmax8(row + 8 * jj, big);
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t off = sw128_off(4 * warp + m, 4 * lane, 64);
                *reinterpret_cast<uint2 *>(sm + KH + off) = khr[m];
                *reinterpret_cast<uint2 *>(sm + KC + off) = kcr[m];
                *reinterpret_cast<uint2 *>(sm + TE + off) = er[m];
                *reinterpret_cast<uint2 *>(sm + TEI + off) = eir[m];
            }
        }
        if (issuer) {  // dO and -dU of the next tile, once the first products have read them
            ok = mbar_wait(&bars[1], par, kWait) && ok;
            if (more) load_a1(nxt);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (issuer) {
            fence_after_sync();
            const uint64_t kP = desc_kmajor(smem_addr(sm + PA), 128, 0), kA = desc_kmajor(smem_addr(sm + PA + 8192), 128, 0),
                           mP = desc_mnmajor(smem_addr(sm + PA), 64, 0), mA = desc_mnmajor(smem_addr(sm + PA + 8192), 64, 0),
                           qb = desc_mnmajor(smem_addr(sm + RQ), 64, 0), kc = desc_mnmajor(smem_addr(sm + KC), 64, 0),
                           kh = desc_mnmajor(smem_addr(sm + KH), 64, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t b_kh = kstep_mnmajor(kh, ks);
                mma_bf16(tm + TM_Y1, kstep_kmajor(kP, 128, ks), b_kh, ID_KM128, 1);
                mma_bf16(tm + TM_Y2, kstep_kmajor(kA, 128, ks), b_kh, ID_KM128, 1);
                mma_bf16(tm + TM_Y3, kstep_mnmajor(mP, ks), kstep_mnmajor(qb, ks), ID_MM128, 1);
                mma_bf16(tm + TM_Y3, kstep_mnmajor(mA, ks), kstep_mnmajor(kc, ks), ID_MM128, 1);
            }
            mma_commit(&bars[2]);
        }
        // ---------------- dq, dk, db, dG per (row, channel), from tensor memory.
        // The M = 64 accumulators hold row quarter * 16 + l in lane l < 16; the
        // 16x256b loads give each thread two rows x two column pairs of every
        // 16-channel group.
        if (compute) {
            ok = mbar_wait(&bars[2], par, kWait) && ok;
            fence_after_sync();
            // 16x256b loads: thread t holds rows q16 + t/4 and q16 + t/4 + 8, column
            // pairs 2 (t % 4) and 8 + 2 (t % 4) of each 16-column group
            const int rA = quarter * 16 + (lane >> 2), cp0 = 2 * (lane & 3);
#pragma unroll 1
            for (int g2 = 0; g2 < 2; ++g2) {
                const int ch0 = 32 * cgrp + 16 * g2;
                float y1[8], y2[8], y3[8];
                tmem_ld16x256x2(taddr(tm + TM_Y1 + ch0, quarter * 32, 0), y1);
                tmem_ld16x256x2(taddr(tm + TM_Y2 + ch0, quarter * 32, 0), y2);
                tmem_ld16x256x2(taddr(tm + TM_Y3 + ch0, quarter * 32, 0), y3);
                tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 4; ++p) {  // (row, column pair): p & 1 picks the row, p >> 1 the pair
                    const int rr = rA + 8 * (p & 1), c = ch0 + cp0 + 8 * (p >> 1);
                    const int ri = 2 * (p & 1) + 4 * (p >> 1);  // register index of the pair
                    const uint32_t o16 = sw128_off(rr, c, 64);
                    const uint32_t o32 = sw128_chunk(rr, c >> 2, 64) + (c & 3) * 4;
                    const float2 qb = __half22float2(*reinterpret_cast<const __half2 *>(sm + RQ + o16));
                    const float2 kc = __half22float2(*reinterpret_cast<const __half2 *>(sm + KC + o16));
                    const float2 kh = __half22float2(*reinterpret_cast<const __half2 *>(sm + KH + o16));
                    const float2 E = __half22float2(*reinterpret_cast<const __half2 *>(sm + TE + o16));
                    const float2 Ei = __half22float2(*reinterpret_cast<const __half2 *>(sm + TEI + o16));
                    const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + RK + o16));
                    const float2 bf = *reinterpret_cast<const float2 *>(sm + RB + o32);
                    const float a1[2] = {y1[ri], y1[ri + 1]}, a2[2] = {y2[ri], y2[ri + 1]}, a3[2] = {y3[ri], y3[ri + 1]};
                    const float qv[2] = {qb.x, qb.y}, kcv[2] = {kc.x, kc.y}, khv[2] = {kh.x, kh.y};
                    const float Ev[2] = {E.x, E.y}, Eiv[2] = {Ei.x, Ei.y}, kv[2] = {kf.x, kf.y}, bv[2] = {bf.x, bf.y};
                    float dq[2], dk[2], db[2], dG[2];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float dkc = a2[i] * Ev[i], dkh = a3[i] * Eiv[i];
                        dq[i] = a1[i] * Ev[i];
                        db[i] = dkc * kv[i];
                        dk[i] = dkc * bv[i] + dkh;
                        dG[i] = a1[i] * qv[i] + a2[i] * kcv[i] - a3[i] * khv[i];
                    }
                    *reinterpret_cast<uint32_t *>(sm + RQ + o16) = pack_bf16(dq[0], dq[1]);
                    *reinterpret_cast<uint32_t *>(sm + RK + o16) = pack_bf16(dk[0], dk[1]);
                    *reinterpret_cast<float2 *>(sm + RB + o32) = make_float2(db[0], db[1]);
                    *reinterpret_cast<float2 *>(sm + RG + o32) = make_float2(dG[0], dG[1]);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (issuer) {
            if (more) load_a2(nxt, (n + 1) & 1);  // Kh, Kc, E, 1/E, dP, dA are consumed
            for (int x = 0; x < 2; ++x) {
                tma_store_4d(&mdq, sm + RQ + x * 8192, 64 * x, h, c0, bb);
                tma_store_4d(&mdk, sm + RK + x * 8192, 64 * x, h, c0, bb);
            }
            for (int x = 0; x < 4; ++x) tma_store_4d(&mdb, sm + RB + x * 8192, 32 * x, h, c0, bb);
            bulk_commit();
        }
        // ---------------- dg: reverse in-chunk cumsum of dG with the chunk-end term
        if (compute) {
            float run[4] = {0.f, 0.f, 0.f, 0.f}, x[4][4];
#pragma unroll
            for (int m = 3; m >= 0; --m) {
                const float4 t = *reinterpret_cast<const float4 *>(sm + RG + sw128_chunk(4 * warp + m, lane, 64));
                run[0] += t.x; run[1] += t.y; run[2] += t.z; run[3] += t.w;
#pragma unroll
                for (int i = 0; i < 4; ++i) x[m][i] = run[i];
            }
            *reinterpret_cast<float4 *>(scan + warp * 128 + 4 * lane) = make_float4(run[0], run[1], run[2], run[3]);
            named_sync(1, kCompute);
            if (tid < 128) {  // per channel: the end term plus the later warps' totals, in place
                float acc = sEnd2[256 * par + tid] + sEnd2[256 * par + 128 + tid];
#pragma unroll
                for (int w2 = kWarps - 1; w2 >= 0; --w2) {
                    const float t = scan[w2 * 128 + tid];
                    scan[w2 * 128 + tid] = acc;
                    acc += t;
                }
            }
            named_sync(1, kCompute);
            const float4 a4 = *reinterpret_cast<const float4 *>(scan + warp * 128 + 4 * lane);
            const float after[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<float4 *>(sm + RG + sw128_chunk(4 * warp + m, lane, 64)) =
                    make_float4(x[m][0] + after[0], x[m][1] + after[1], x[m][2] + after[2], x[m][3] + after[3]);
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) break;
        if (issuer) {
            for (int x = 0; x < 4; ++x) tma_store_4d(&mdg, sm + RG + x * 8192, 32 * x, h, c0, bb);
            bulk_commit();
            bulk_wait_read();  // the tiles may be refilled
            if (more) load_b(nxt);
        }
    }
    if (issuer) bulk_wait_all();
    if (!(big <= kRange) || !(gbig <= 9.f)) record_status(status, GDN2_ERR_RANGE);
    if (!ok && issuer) {
        record_status(status, GDN2_ERR_TIMEOUT);
        // every copy landed and every issued product done before the shared
        // and tensor memory go away
        if (issued[0] > 0) mbar_wait(&bars[0], (issued[0] - 1) & 1, kWait);
        if (issued[2] > 0) mbar_wait(&bars[3], (issued[2] - 1) & 1, kWait);
        mbar_wait(&bars[1], 0, kWait);
        mbar_wait(&bars[1], 1, kWait);
        mbar_wait(&bars[2], 0, kWait);
        mbar_wait(&bars[2], 1, kWait);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------- launchers
cudaError_t tc_bwd_launch(const void *q, const void *k, const void *v, const float *g,
                          const float *b, const float *w, const void *dO, const float *dST,
                          void *dq, void *dk, void *dv, float *dg, float *db, float *dw,
                          float *dS0, void *ws, unsigned int *status, const Dims &d,
                          cudaStream_t s) {
    CUtensorMap mdo_half, mv, mw, mdv, mdw, mq, mk, mb, mg, mdo, mdq, mdk, mdb, mdg;
    if (!make_btHd_map(&mdo_half, dO, true, d.B, d.T, d.H, 128, 64, 64) ||
        !make_btHd_map(&mv, v, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mw, w, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mdv, dv, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mdw, dw, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mq, q, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mk, k, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mb, b, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mg, g, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mdo, dO, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mdq, dq, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mdk, dk, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mdb, db, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mdg, dg, false, d.B, d.T, d.H, 128, 64, 32, true))
        return cudaErrorInvalidValue;
    const TcWs lay = tc_ws_layout(d);
    cudaError_t e = cudaFuncSetAttribute(tc_bwd_state_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tbs::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tbg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    launch_begin(K_TC_BWD_STATE, s);
    tc_bwd_state_kernel<<<dim3(2, d.H, d.B), tbs::kThreads, tbs::SMEM_BYTES, s>>>(
        mdo_half, mv, mw, mdv, mdw, dST, dS0, (unsigned char *)ws, lay, status, d);
    launch_end(K_TC_BWD_STATE, s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    launch_begin(K_TC_BWD_GRAD, s);
    const long long ntiles = (long long)d.B * d.H * d.NC;
    const int grid = (int)(ntiles < sm_count() ? ntiles : sm_count());
    tc_bwd_grad_kernel<<<grid, tbg::kThreads, tbg::SMEM_BYTES, s>>>(
        mq, mk, mb, mg, mdo, mdq, mdk, mdb, mdg, (unsigned char *)ws, lay, status, d);
    launch_end(K_TC_BWD_GRAD, s);
    return cudaGetLastError();
}

}  // namespace gdn2
