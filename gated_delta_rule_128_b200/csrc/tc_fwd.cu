// Sequential part of the tensor-core forward of Gated Delta Rule-2 (bf16
// q/k/v/o, float32 gates and state, d_k = d_v = 128, chunk 64): the state
// pass and the outputs, from the chunk records of tc_prep.cu.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B): only the state crosses chunk borders.  Per chunk of 64 tokens
// entering with state S (the chunk's frame, with frame factor s, see REC_* in
// common.cuh; U = w.v):
//   Delta = T U - W (s S)
//   O = Qb (s S) + P Delta,   S_next = diag(gamma) S + r Kx^T Delta
// The state stays at its true scale in registers; only the operand s S
// changes frame from chunk to chunk.
//
// One CTA owns one (b, h) and one 64-column half of d_v and walks the
// sequence's chunks in order with its fp32 state slice in registers (each
// thread one key row, 32 columns).  The chunk records are double-buffered in
// shared memory and requested two chunks ahead, since they do not depend on
// the state.
//
// Both state-side products are M = 128 tcgen05.mma groups into one
// [Delta; O] accumulator (rows 0..63 Delta, 64..127 O; two such accumulators
// alternate between chunks):
//   (1) [T; 0] U + [-W; Qb] (s S)          -> Delta and Qb (s S)
//   (2) [0; P] Delta,  and  X = Kx^T Delta (a fresh accumulator)
// then S_next = gamma S + r X in registers.  Warp roles: warps 0, 1, 4, 5 (TMEM
// lanes 0..63) read Delta; warps 2, 3, 6, 7 (lanes 64..127) read the previous
// chunk's O and form the next chunk's U = w.v off the state's path; all warps
// update the state.
//
// Precision and range: fp16 operands carry 11 significant bits (bf16 carries
// 8, which left the output error at the 5e-3 tolerance); Delta is formed in
// the f32 accumulator.  Any operand beyond 6e4 in magnitude is reported as
// GDN2_ERR_RANGE.
//
// For the backward the call can also leave in the workspace (TcWs): every
// chunk's entry state in its frame, s S_c (fp16, a copy of the operand), and
// Delta per chunk.

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

namespace tfwd {
constexpr int kThreads = 256;
// one record stage: the record with an 8 KB zero tile between T and P, so
// that [T; 0] and [0; P] are M = 128 operands
constexpr uint32_t S_WQ = 0, S_KH = 32768, S_T = 49152, S_Z = 57344, S_P = 65536, S_FAC = 73728;
constexpr uint32_t STAGE = 74752;
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t STG = 0;                  // two record stages
constexpr uint32_t RAW_V = 2 * STAGE;        // v half, bf16 [64 pos][64]
constexpr uint32_t RAW_W = RAW_V + 8192;     // w half, f32 or bf16 [64 pos][64]
constexpr uint32_t OP_U = RAW_W + 16384;     // two U = w.v tiles [64 pos][64 v] MN-major, 8 KB each
constexpr uint32_t OP_S = OP_U + 16384;      // S (fp16)     [128 key][64 v] MN-major
constexpr uint32_t OP_D = OP_S + 16384;      // Delta        [64 pos][64 v]  MN-major
constexpr uint32_t MISC = OP_D + 8192;       // mbarriers, TMEM slot
constexpr uint32_t SMEM_BYTES = MISC + 128 + 1024;
// tensor memory columns (256 allocated): Kb^T Delta, then two [Delta; O] accumulators
constexpr uint32_t TM_S = 0, TM_X = 64;
constexpr uint32_t ID_KM128x64 = idesc_f16(128, 64, false, true);
constexpr uint32_t ID_MM128x64 = idesc_f16(128, 64, true, true);
constexpr long long kWait = 2000000000LL;  // ~1 s of SM clocks per wait
constexpr float kRange = 6.0e4f;           // largest operand magnitude kept in fp16
static_assert(STAGE % 1024 == 0 && MISC % 1024 == 0, "alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace tfwd

template <bool GB, bool ACT>  // w as bf16 (else float32); ACT: gate logits (GateAct)
__global__ void __launch_bounds__(tfwd::kThreads, 1)
tc_fwd_kernel(const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mw,
              const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ ST,
              unsigned char *__restrict__ ws, int keep, TcWs lay, SegPass sp, unsigned int *status, Dims d) {
    using namespace tfwd;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    // 0, 1 records of stages 0, 1; 2 v and w; 3, 4 the two product groups
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 64);
    float big = 0.f;  // largest operand magnitude seen (range check)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, n = blockIdx.z;
    // this CTA's task (SegPass in common.cuh): a real run of segment sg, or in
    // the first pass of a split sequence a run from zero (N_s) or from the
    // identity with no input (M_s); vh is the 64-column half
    int vh, sg = 0, mode = 0;  // mode 0 real, 1 from zero, 2 from the identity
    {
        const int x = blockIdx.x, mid = 2 * (sp.P - 2);
        if (sp.phase == 2) { sg = 1 + (x >> 1); vh = x & 1; }
        else if (x < 2) { vh = x; }
        else if (x < 2 + mid) { mode = 1; sg = 1 + ((x - 2) >> 1); vh = (x - 2) & 1; }
        else { mode = 2; sg = 1 + ((x - 2 - mid) >> 1); vh = (x - 2 - mid) & 1; }
    }
    const int v0 = vh * 64;
    // sequence n: tokens bos .. bos + T - 1 of batch row bb, chunks NC; a
    // segment narrows these to its own chunks
    const Seq sq = seq_of(d, n);
    int NC = sq.nc, T = sq.len, bos = sq.bos;
    const int bb = sq.brow;
    size_t tile0 = (size_t)tile_of(d, sq, h, 0);  // workspace tile of the run's first chunk
    const size_t bhx = (size_t)n * d.H + h;
    if (sp.P > 1) {
        const int L = seg_len(NC, sp.P), cb = sg * L;
        NC = min(L, NC - cb);
        T = min(T - 64 * cb, 64 * NC);
        bos += 64 * cb;
        tile0 += cb;
    }
    // the entry state (null: zero) and where the final state goes (null: nowhere)
    const bool first_seg = sp.P == 1 || (mode == 0 && sg == 0);
    const float *ent = mode != 0 ? nullptr : first_seg ? (S0 ? S0 + st_off(d, n, h) : nullptr)
                                                      : seg_buf(sp, bhx, sg, SEG_ENTRY);
    float *fin = mode == 1 ? seg_buf(sp, bhx, sg, SEG_ZERO)
               : mode == 2 ? seg_buf(sp, bhx, sg, SEG_MAP)
               : (sp.P == 1 || sg == sp.P - 1) ? (ST ? ST + st_off(d, n, h) : nullptr)
               : (sp.phase == 1 ? seg_buf(sp, bhx, 1, SEG_ENTRY) : nullptr);
    if (mode != 0) {  // no outputs of its own
        o = nullptr;
        keep = 0;
    }
    const bool use_u = mode != 2;  // the identity run has no input
    const GateAct ga = ACT ? gate_act(d.act) : GateAct{false, 1.f};  // logits in: w activated on load
    const int quarter = warp & 3, half = warp >> 2;
    const int key = quarter * 32 + lane;          // state row (TMEM lane) of this thread
    const bool dwarp = quarter < 2;               // reads Delta (lanes 0..63), else O (64..127)
    const int ot = (half * 2 + (quarter - 2)) * 32 + lane;  // 0..127 among the O warps
    const unsigned char *recs = ws + lay.rec + tile0 * (size_t)REC_BYTES;
    if (NC <= 0) {  // an empty sequence: S_T = S0
        if (fin) {
            const size_t so = (size_t)(tid >> 1) * 128 + v0 + 32 * (tid & 1);
            for (int j = 0; j < 32; ++j) fin[so + j] = ent ? ent[so + j] : 0.f;
        }
        return;
    }

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    // zero tiles of both stages
    for (int i = tid; i < 2 * 8192 / 16; i += kThreads)
        *reinterpret_cast<uint4 *>(sm + STG + (i >> 9) * STAGE + S_Z + (i & 511) * 16) = make_uint4(0, 0, 0, 0);
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    int issued[3] = {0, 0, 0};  // loads requested per barrier
    int groups[2] = {0, 0};     // product groups 1 and 2 issued (thread 0)
    auto load_rec = [&](int cc) {  // thread 0
        const int s = cc & 1;
        unsigned char *dst = sm + STG + s * STAGE;
        const unsigned char *src = recs + (size_t)cc * REC_BYTES;
        mbar_expect_tx(&bars[s], REC_BYTES);
        bulk_load(dst, src, REC_P, &bars[s]);                        // [-W; Qb], Kh, T
        bulk_load(dst + S_P, src + REC_P, 8192, &bars[s]);           // P
        bulk_load(dst + S_FAC, src + REC_FAC, REC_BYTES - REC_FAC, &bars[s]);
        ++issued[s];
    };
    auto load_vw = [&](int cc) {  // thread 64
        mbar_expect_tx(&bars[2], 8192 + (GB ? 8192 : 16384));
        tma_load_4d(sm + RAW_V, &mv, v0, h, bos + cc * 64, bb, &bars[2]);
        tma_load_4d(sm + RAW_W, &mw, v0, h, bos + cc * 64, bb, &bars[2]);
        ++issued[2];
    };
    // U = w.v of chunk cc into OP_U[cc & 1] (O warps: 4 rows x 8 columns each)
    auto make_u = [&](int cc) {
        const int jv = ot & 7;
        unsigned char *dst = sm + OP_U + (cc & 1) * 8192;
        if (!use_u) {  // no input: U = 0
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<uint4 *>(dst + sw128_chunk((ot >> 3) + 16 * i, jv, 64)) = make_uint4(0u, 0u, 0u, 0u);
            return;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = (ot >> 3) + 16 * i;
            const uint4 vr = *reinterpret_cast<const uint4 *>(sm + RAW_V + r * 128 + jv * 16);
            float4 w0, w1;
            if constexpr (GB) {
                w0 = gld4<true>(sm + RAW_W + r * 128 + jv * 16);
                w1 = gld4<true>(sm + RAW_W + r * 128 + jv * 16 + 8);
            } else {
                w0 = *reinterpret_cast<const float4 *>(sm + RAW_W + r * 256 + jv * 32);
                w1 = *reinterpret_cast<const float4 *>(sm + RAW_W + r * 256 + jv * 32 + 16);
            }
            w0 = act_w4(ga, w0);
            w1 = act_w4(ga, w1);
            const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vr);
            float u[8] = {w0.x * __low2float(v2[0]), w0.y * __high2float(v2[0]),
                          w0.z * __low2float(v2[1]), w0.w * __high2float(v2[1]),
                          w1.x * __low2float(v2[2]), w1.y * __high2float(v2[2]),
                          w1.z * __low2float(v2[3]), w1.w * __high2float(v2[3])};
            if (r >= T - 64 * cc) {  // past the sequence's end (a packed layout's next sequence)
#pragma unroll
                for (int e = 0; e < 8; ++e) u[e] = 0.f;
            }
            st_h8(dst + sw128_chunk(r, jv, 64), u);
            big = absmax8(u, big);
        }
    };
    // product group 1 of chunk cc (thread 0)
    auto group1 = [&](int cc) {
        const uint32_t st = smem_addr(sm + STG + (cc & 1) * STAGE);
        const uint32_t x = tm + TM_X + 64 * (cc & 1);
        const uint64_t dT = desc_kmajor(st + S_T, 128, 0),
                       dU = desc_mnmajor(smem_addr(sm + OP_U + (cc & 1) * 8192), 64, 0),
                       dW = desc_kmajor(st + S_WQ, 128, 0),
                       dS = desc_mnmajor(smem_addr(sm + OP_S), 128, 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(x, kstep_kmajor(dT, 128, ks), kstep_mnmajor(dU, ks), ID_KM128x64, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(x, kstep_kmajor(dW, 128, ks), kstep_mnmajor(dS, ks), ID_KM128x64, 1);
        mma_commit(&bars[3]);
        ++groups[0];
    };
    auto ckpt = [&](int c) { return ws + lay.ckS + ((tile0 + c) * 2 + vh) * 16384; };
    // O rows of chunk cc (O warps): accumulator rows 64..127, this warp's 32 columns
    auto store_o = [&](int cc) {
        float ov[32];
        const uint32_t x = tm + TM_X + 64 * (cc & 1);
        tmem_ld16(taddr(x, quarter * 32, 32 * half), ov);
        tmem_ld16(taddr(x, quarter * 32, 32 * half + 16), ov + 16);
        tmem_wait_ld();
        const int t = cc * 64 + key - 64;
        if (o && t < T) {
            unsigned char *dst = reinterpret_cast<unsigned char *>(o + tok(d, bb, bos + t, h, 128) + v0 + 32 * half);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) st_bf16x8(dst + 16 * jj, ov + 8 * jj);
        }
    };

    if (tid == 0) {
        load_rec(0);
        if (NC > 1) load_rec(1);
    }
    if (tid == 64 && use_u) load_vw(0);

    // ---------------- prologue: S of chunk 0 (registers, OP_S); U of chunk 0
    bool ok = mbar_wait(&bars[0], 0, kWait);
    float sreg[32];  // this thread's state row `key`, columns v0 + 32 half + j
    {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 t = ent ? *reinterpret_cast<const float4 *>(ent + (size_t)key * 128 + v0 + 32 * half + j)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            sreg[j] = t.x; sreg[j + 1] = t.y; sreg[j + 2] = t.z; sreg[j + 3] = t.w;
        }
        if (mode == 2) {  // the identity: column v0 + 32 half + j of I
#pragma unroll
            for (int j = 0; j < 32; ++j) sreg[j] = key == v0 + 32 * half + j ? 1.f : 0.f;
        }
        // the operand state s S in chunk 0's frame
        const float s0 = reinterpret_cast<const float *>(sm + STG + S_FAC)[128 + key];
        const float se = s0 < 0.f ? 1.f : s0;
        float x[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = se * sreg[j];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            st_h8(sm + OP_S + sw128_chunk(key, 4 * half + jj, 128), x + 8 * jj);
            big = absmax8(x + 8 * jj, big);
        }
    }
    if (!dwarp) {
        if (use_u) ok = mbar_wait(&bars[2], 0, kWait) && ok;
        make_u(0);
        named_sync(2, 128);  // raw v, w consumed
        if (tid == 64 && NC > 1 && use_u) load_vw(1);
    }
    fence_proxy_async();
    fence_before_sync();
    bool abort = __syncthreads_or(!ok);
    if (tid == 0 && !abort) {
        fence_after_sync();
        if (keep) {
            bulk_store(ckpt(0), sm + OP_S, 16384);
            bulk_commit();
        }
        group1(0);
    }

    for (int c = 0; c < NC && !abort; ++c) {
        const int s = c & 1;
        const uint32_t par = c & 1;
        unsigned char *stg = sm + STG + s * STAGE;
        const uint32_t x = tm + TM_X + 64 * s;
        if (dwarp) {
            // ---------------- Delta rows to fp16
            ok = mbar_wait(&bars[3], par, kWait);
            fence_after_sync();
            float dl[32];
            tmem_ld16(taddr(x, quarter * 32, 32 * half), dl);
            tmem_ld16(taddr(x, quarter * 32, 32 * half + 16), dl + 16);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                st_h8(sm + OP_D + sw128_chunk(key, 4 * half + jj, 64), dl + 8 * jj);
                big = absmax8(dl + 8 * jj, big);
            }
            fence_proxy_async();
            fence_before_sync();
            named_sync(1, 128);
            if (tid == 0) {
                fence_after_sync();
                bulk_wait_read();  // the checkpoint copy has left OP_S
                const uint32_t st = smem_addr(stg);
                const uint64_t dZP = desc_kmajor(st + S_Z, 128, 0), dK = desc_mnmajor(st + S_KH, 64, 0),
                               dD = desc_mnmajor(smem_addr(sm + OP_D), 64, 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(x, kstep_kmajor(dZP, 128, ks), kstep_mnmajor(dD, ks), ID_KM128x64, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tm + TM_S, kstep_mnmajor(dK, ks), kstep_mnmajor(dD, ks), ID_MM128x64, ks > 0);
                mma_commit(&bars[4]);
                ++groups[1];
                if (keep) {  // Delta of this chunk and half, for the backward
                    bulk_store(ws + lay.ckD + ((tile0 + c) * 2 + vh) * 8192, sm + OP_D, 8192);
                    bulk_commit();
                }
            }
        } else {
            // ---------------- previous chunk's O; next chunk's U
            if (c > 0) store_o(c - 1);
            if (c + 1 < NC) {
                if (use_u) ok = mbar_wait(&bars[2], (c + 1) & 1, kWait) && ok;
                make_u(c + 1);
                fence_proxy_async();
                named_sync(2, 128);  // raw v, w consumed
                if (tid == 64 && c + 2 < NC && use_u) {
                    load_vw(c + 2);
                    if (c + 3 < NC) {  // the v, w after those into L2
                        tma_prefetch_4d(&mv, v0, h, bos + (c + 3) * 64, bb);
                        tma_prefetch_4d(&mw, v0, h, bos + (c + 3) * 64, bb);
                    }
                }
            }
        }
        // ---------------- S_next = gamma S + Kb^T Delta
        ok = mbar_wait(&bars[4], par, kWait) && ok;
        const float gam = reinterpret_cast<const float *>(stg + S_FAC)[key];  // e^G_63
        const float sc = reinterpret_cast<const float *>(stg + S_FAC)[128 + key];
        const float rr = sc < 0.f ? 1.f : gam / sc;  // Kx^T Delta's scale in S_next
        // the next chunk's record has landed before its first products are issued
        float sn = 1.f;  // the next chunk's frame factor
        if (c + 1 < NC) {
            ok = mbar_wait(&bars[s ^ 1], ((c + 1) >> 1) & 1, kWait) && ok;
            const float sv = reinterpret_cast<const float *>(sm + STG + (s ^ 1) * STAGE + S_FAC)[128 + key];
            sn = sv < 0.f ? 1.f : sv;
        }
        fence_after_sync();
        {
            float xv[32];
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half), xv);
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), xv + 16);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) sreg[j] = fmaf(gam, sreg[j], rr * xv[j]);
            if (c + 1 < NC) {
#pragma unroll
                for (int j = 0; j < 32; ++j) xv[j] = sn * sreg[j];  // the operand state s S
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    st_h8(sm + OP_S + sw128_chunk(key, 4 * half + jj, 128), xv + 8 * jj);
                    big = absmax8(xv + 8 * jj, big);
                }
            } else if (fin) {
                float *dst = fin + (size_t)key * 128 + v0 + 32 * half;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
            }
        }
        if (tid == 0) bulk_wait_read();  // the Delta copy has left OP_D
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0) {
            fence_after_sync();
            if (c + 2 < NC) load_rec(c + 2);  // this stage's record is consumed
            if (c + 1 < NC) {
                if (keep) {
                    bulk_store(ckpt(c + 1), sm + OP_S, 16384);
                    bulk_commit();
                }
                group1(c + 1);
            }
            // the record after the next into L2, so that its copy takes the L2 latency
            if (c + 3 < NC) bulk_prefetch_l2(recs + (size_t)(c + 3) * REC_BYTES, REC_BYTES);
        }
    }
    if (!abort && !dwarp) store_o(NC - 1);
    if (!(big <= kRange)) record_status(status, GDN2_ERR_RANGE);
    if (tid == 0) bulk_wait_all();
    if (abort && (tid == 0 || tid == 64)) {
        if (tid == 0) record_status(status, GDN2_ERR_TIMEOUT);
        // let every requested copy land before the CTA's shared memory goes away
        for (int i = 0; i < 3; ++i)
            if (issued[i] > 0) mbar_wait(&bars[i], (issued[i] - 1) & 1, kWait);
        // and every issued product finish before the tensor memory is freed
        for (int i = 0; i < 2; ++i)
            if (groups[i] > 0) mbar_wait(&bars[3 + i], (groups[i] - 1) & 1, kWait);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

// ---------------------------------------------------------------- launcher
cudaError_t tc_prep_launch(const void *q, const void *k, const void *g, const void *b, void *ws,
                           unsigned int *status, const Dims &d, cudaStream_t s);

// the link step between the passes (seg_link.cu)
cudaError_t seg_link_launch(const SegPass &sp, int nbh, bool backward, cudaStream_t s);

template <bool GB, bool ACT>
static cudaError_t tc_fwd_run(const void *v, const void *w, const float *S0, void *o, float *ST,
                              void *ws, int keep, unsigned int *status, const Dims &d, cudaStream_t s) {
    CUtensorMap mv, mw;
    if (!make_btHd_map(&mv, v, true, d.B, d.T, d.H, 128, 64, 64) ||
        !make_btHd_map(&mw, w, GB, d.B, d.T, d.H, 128, 64, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tc_fwd_kernel<GB, ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tfwd::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const TcWs lay = tc_ws_layout(d);
    SegPass sp{1, 0, nullptr};
    // a split sequence needs the workspace that keeps the forward (its segment buffers)
    if (lay.P > 1 && keep) sp = SegPass{lay.P, 1, reinterpret_cast<float *>(static_cast<char *>(ws) + lay.seg)};
    launch_begin(K_TC_FWD, s);
    tc_fwd_kernel<GB, ACT><<<dim3(sp.P > 1 ? 2 + 4 * (sp.P - 2) : 2, d.H, num_seqs(d)), tfwd::kThreads,
                        tfwd::SMEM_BYTES, s>>>(mv, mw, S0, (__nv_bfloat16 *)o, ST, (unsigned char *)ws, keep,
                                               lay, sp, status, d);
    launch_end(K_TC_FWD, s);
    if (sp.P > 1) {
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = seg_link_launch(sp, d.B * d.H, false, s)) != cudaSuccess) return e;
        sp.phase = 2;
        launch_begin(K_TC_FWD, s);
        tc_fwd_kernel<GB, ACT><<<dim3(2 * (sp.P - 1), d.H, d.B), tfwd::kThreads, tfwd::SMEM_BYTES, s>>>(
            mv, mw, S0, (__nv_bfloat16 *)o, ST, (unsigned char *)ws, keep, lay, sp, status, d);
        launch_end(K_TC_FWD, s);
    }
    return cudaGetLastError();
}

// keep != 0: also leave the chunk states and Delta for the backward
cudaError_t tc_fwd_launch(const void *q, const void *k, const void *v, const void *g,
                          const void *b, const void *w, const float *S0, void *o, float *ST,
                          void *ws, int keep, unsigned int *status, const Dims &d, cudaStream_t s) {
    cudaError_t e = tc_prep_launch(q, k, g, b, ws, status, d, s);
    if (e != cudaSuccess) return e;
    if (d.act) return d.gb ? tc_fwd_run<true, true>(v, w, S0, o, ST, ws, keep, status, d, s)
                           : tc_fwd_run<false, true>(v, w, S0, o, ST, ws, keep, status, d, s);
    return d.gb ? tc_fwd_run<true, false>(v, w, S0, o, ST, ws, keep, status, d, s)
                : tc_fwd_run<false, false>(v, w, S0, o, ST, ws, keep, status, d, s);
}

}  // namespace gdn2
