// Chunk-parallel part of the tensor-core forward of Gated Delta Rule-2 (bf16
// q/k, float32 g/b, d_k = 128, chunk 64): everything about a chunk that does
// not depend on the state entering it.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B): once the state is normalised by the in-chunk cumulative decay,
// the decay folds into the two factors of every rank-one erase, and a single
// unit-lower-triangular inverse serves the erase and the write side.  With the
// factors taken relative to the chunk's middle row m (tc_common.cuh):
//   G = cumsum(g),  Qb = q.e^(G-G_m),  Kc = b.k.e^(G-G_m),  Kh = k.e^-(G-G_m)
//   A = strictly-lower(Kc Kh^T),  T = (I + A)^-1,  W = T Kc
//   P = lower-incl(Qb Kh^T)
// The kernel writes Qb, Kh, -W, T, P and the per-channel factors
// e^(G_L - G_m), e^G_m to the chunk's record in the workspace (layout REC_*
// in common.cuh); the sequential state kernel (tc_fwd.cu) and the backward
// read them from there.  Kc and Qb share one [128][128] tile (Kc on top), so
// that A and P come out of one M = 128 product: [Kc; Qb] Kh^T.
//
// Persistent: one CTA per SM walks the (b, h, chunk) tiles with a stride of
// the grid size.  TMA brings the raw q, k, g, b tiles; as soon as the
// operands are formed the next tile's raw tiles are requested, so that their
// transfer overlaps the products and the inversion of this tile.  A, P and W
// are tcgen05.mma products (fp16 operands, f32 accumulators in TMEM); T is
// inverted in float32 on the CUDA cores.

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

namespace tprep {
constexpr int kThreads = 256;
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_G = 32768, RAW_B = 65536;
constexpr uint32_t REC = 98304;  // the tile's record, laid out as in the workspace
constexpr uint32_t OP_WQ = REC + REC_WQ;  // [Kc; Qb], later [-W; Qb]
constexpr uint32_t OP_KH = REC + REC_KH;
constexpr uint32_t OP_T = REC + REC_T, OP_P = REC + REC_P, FAC = REC + REC_FAC;
constexpr uint32_t SCR = REC + REC_BYTES;  // float32 scratch of the inversion
constexpr uint32_t SCR_A = SCR, SCR_T = SCR + 64 * 65 * 4, SCR_M = SCR_T + 64 * 65 * 4;
constexpr uint32_t SCR_SCAN = SCR;  // per-warp cumsum totals [8][128] f32, before the inversion
constexpr uint32_t MISC = SCR_M + 8 * 16 * 9 * 4;  // mbarriers, TMEM slot
constexpr uint32_t SMEM_BYTES = MISC + 128 + 1024;
constexpr uint32_t TM_AP = 0, TM_W = 128;  // [A; P] (M = 128), W; 256 columns
constexpr uint32_t ID_KK128x64 = idesc_f16(128, 64, false, false);
constexpr uint32_t ID_KM128 = idesc_f16(64, 128, false, true);
constexpr long long kWait = 2000000000LL;  // ~1 s of SM clocks per wait
constexpr float kRange = 6.0e4f;
static_assert(MISC % 8 == 0, "mbarrier alignment");
}  // namespace tprep

// Warp-level tensor-core tile product D = A B + C (m16n8k8, tf32 operands,
// f32 accumulate) for the small 16x16 block products of the T inversion.
// Fragment layout (g = lane / 4, t = lane % 4): a0 (g, t), a1 (g + 8, t),
// a2 (g, t + 4), a3 (g + 8, t + 4); b0 (t, g), b1 (t + 4, g);
// c0 (g, 2t), c1 (g, 2t + 1), c2 (g + 8, 2t), c3 (g + 8, 2t + 1).
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float *c, const uint32_t *a, const uint32_t *b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// c += X[r0.., k0..k0+8) * Y[k0..k0+8, n0..n0+8) for row-major [.][65] f32 tiles
__device__ __forceinline__ void tile_mma(float *c, const float *X, int r0, int k0, const float *Y,
                                         int n0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    uint32_t a[4] = {to_tf32(X[(r0 + g) * 65 + k0 + t]), to_tf32(X[(r0 + g + 8) * 65 + k0 + t]),
                     to_tf32(X[(r0 + g) * 65 + k0 + t + 4]), to_tf32(X[(r0 + g + 8) * 65 + k0 + t + 4])};
    uint32_t b[2] = {to_tf32(Y[(k0 + t) * 65 + n0 + g]), to_tf32(Y[(k0 + t + 4) * 65 + n0 + g])};
    mma_tf32_16x8x8(c, a, b);
}

// T = (I + A)^-1 for the strictly-lower 64x64 A in sA ([64][65] f32), into
// sT ([64][65] f32), by blocks of 16: the diagonal blocks by forward
// substitution (one column per thread), then level by level
// T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ (I - J = 1, 2, 3) as warp-level
// tf32 tile products, each warp owning 8 columns of one block.  sM holds one
// 16x8 intermediate per warp ([8][16][9] f32).  All 256 threads; ends with a
// barrier.
__device__ __forceinline__ void invert_unit_lower(const float *sA, float *sT, float *sM, int tid) {
    if (tid < 64) {
        const int o16 = (tid >> 4) * 16, cl = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = r == cl ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < r; ++j) acc -= sA[(o16 + r) * 65 + o16 + j] * x[j];
            x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(o16 + r) * 65 + o16 + cl] = x[r];
    }
    for (int e = tid; e < 64 * 64; e += 256) {
        const int r = e >> 6, j = e & 63;
        if ((j >> 4) > (r >> 4)) sT[r * 65 + j] = 0.f;
    }
    __syncthreads();
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    float *mw = sM + warp * 16 * 9;
    for (int lvl = 1; lvl < 4; ++lvl) {
        const int nb = 4 - lvl;  // blocks on this level, two warps each
        if (warp < 2 * nb) {
            const int J = warp >> 1, I = J + lvl, n0 = 16 * J + 8 * (warp & 1);
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            for (int K = J; K < I; ++K) {
                tile_mma(c, sA, 16 * I, 16 * K, sT, n0, lane);
                tile_mma(c, sA, 16 * I, 16 * K + 8, sT, n0, lane);
            }
            mw[g * 9 + 2 * t] = c[0];
            mw[g * 9 + 2 * t + 1] = c[1];
            mw[(g + 8) * 9 + 2 * t] = c[2];
            mw[(g + 8) * 9 + 2 * t + 1] = c[3];
            __syncwarp();
            float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {
                uint32_t a[4] = {to_tf32(sT[(16 * I + g) * 65 + 16 * I + k0 + t]),
                                 to_tf32(sT[(16 * I + g + 8) * 65 + 16 * I + k0 + t]),
                                 to_tf32(sT[(16 * I + g) * 65 + 16 * I + k0 + t + 4]),
                                 to_tf32(sT[(16 * I + g + 8) * 65 + 16 * I + k0 + t + 4])};
                uint32_t b[2] = {to_tf32(mw[(k0 + t) * 9 + g]), to_tf32(mw[(k0 + t + 4) * 9 + g])};
                mma_tf32_16x8x8(e, a, b);
            }
            sT[(16 * I + g) * 65 + n0 + 2 * t] = -e[0];
            sT[(16 * I + g) * 65 + n0 + 2 * t + 1] = -e[1];
            sT[(16 * I + g + 8) * 65 + n0 + 2 * t] = -e[2];
            sT[(16 * I + g + 8) * 65 + n0 + 2 * t + 1] = -e[3];
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(tprep::kThreads, 1)
tc_prep_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
               const __grid_constant__ CUtensorMap mg, const __grid_constant__ CUtensorMap mb,
               unsigned char *__restrict__ ws, TcWs lay, unsigned int *status, Dims d) {
    using namespace tprep;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC);  // 0 raw tiles, 1 mma
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 64);
    float *sGam = reinterpret_cast<float *>(sm + FAC);
    float *sRef = sGam + 128;
    float big = 0.f, gbig = 0.f;  // range checks: operand magnitude, |G - G_m|

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int NC = d.NC, H = d.H;
    const int ntiles = d.B * H * NC;

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    int issued = 0;  // raw-tile loads requested (thread 0)
    auto load_raw = [&](int it) {
        const int c = it % NC, bh = it / NC, h = bh % H, bb = bh / H;
        mbar_expect_tx(&bars[0], 16384 * 2 + 32768 * 2);
        tma_load_4d(sm + RAW_Q, &mq, 0, h, c * 64, bb, &bars[0]);
        tma_load_4d(sm + RAW_K, &mk, 0, h, c * 64, bb, &bars[0]);
        tma_load_4d(sm + RAW_G, &mg, 0, h, c * 64, bb, &bars[0]);
        tma_load_4d(sm + RAW_B, &mb, 0, h, c * 64, bb, &bars[0]);
        ++issued;
    };
    if (tid == 0 && (int)blockIdx.x < ntiles) load_raw(blockIdx.x);

    bool abort = false;
    int n = 0;  // tiles done by this CTA
    for (int it = blockIdx.x; it < ntiles; it += gridDim.x, ++n) {
        unsigned char *rec = ws + lay.rec + (size_t)it * REC_BYTES;
        // ---------------- cumulative decay and operands
        bool ok = mbar_wait(&bars[0], n & 1, kWait);
        float G[8][4];
        cumsum_local(reinterpret_cast<const float *>(sm + RAW_G), reinterpret_cast<float *>(sm + SCR_SCAN),
                     warp, lane, G);
        if (tid == 0) bulk_wait_read();  // the previous tile's record has left shared memory
        if (__syncthreads_or(!ok)) { abort = true; break; }
        cumsum_finish(reinterpret_cast<const float *>(sm + SCR_SCAN), warp, lane, G, sGam, sRef);
        gbig = fmaxf(gbig, write_factors_rec(sm + RAW_Q, sm + RAW_K, reinterpret_cast<const float *>(sm + RAW_B),
                                           G, sm + OP_WQ, sm + OP_KH, warp, lane));
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            if (it + (int)gridDim.x < ntiles) load_raw(it + gridDim.x);  // raw tiles consumed
            const uint64_t kq = desc_kmajor(smem_addr(sm + OP_WQ), 128, 0),
                           kh = desc_kmajor(smem_addr(sm + OP_KH), 64, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_AP, kstep_kmajor(kq, 128, ks), kstep_kmajor(kh, 64, ks), ID_KK128x64, ks > 0);
            mma_commit(&bars[1]);
        }
        // ---------------- strictly-lower A to float32, masked P to fp16; T = (I + A)^-1
        ok = mbar_wait(&bars[1], 0, kWait);
        fence_after_sync();
        float *sA = reinterpret_cast<float *>(sm + SCR_A);
        float *sT = reinterpret_cast<float *>(sm + SCR_T);
        {
            // accumulator row quarter * 32 + lane: rows 0..63 are A, 64..127 are P;
            // this warp's 32 columns start at 32 * half
            float row[32];
            tmem_ld16(taddr(tm + TM_AP, quarter * 32, 32 * half), row);
            tmem_ld16(taddr(tm + TM_AP, quarter * 32, 32 * half + 16), row + 16);
            tmem_wait_ld();
            if (quarter < 2) {
                const int r = quarter * 32 + lane;
#pragma unroll
                for (int j = 0; j < 32; ++j) sA[r * 65 + 32 * half + j] = 32 * half + j < r ? row[j] : 0.f;
            } else {
                const int r = quarter * 32 + lane - 64;
#pragma unroll
                for (int j = 0; j < 32; ++j) row[j] = 32 * half + j <= r ? row[j] : 0.f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    st_h8(sm + OP_P + sw128_chunk(r, 4 * half + jj, 64), row + 8 * jj);
                    big = absmax8(row + 8 * jj, big);
                }
            }
        }
        if (__syncthreads_or(!ok)) { abort = true; break; }
        invert_unit_lower(sA, sT, reinterpret_cast<float *>(sm + SCR_M), tid);
        for (int e = tid; e < 64 * 8; e += kThreads) {
            const int r = e >> 3, jj = e & 7;
            st_h8(sm + OP_T + sw128_chunk(r, jj, 64), sT + r * 65 + 8 * jj);
            big = absmax8(sT + r * 65 + 8 * jj, big);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            // Kc (rows 0..63 of the [Kc; Qb] tile) as the MN-major B: its two
            // 64-key blocks lie 16 KB apart
            const uint64_t t = desc_kmajor(smem_addr(sm + OP_T), 64, 0),
                           kc = desc_mnmajor_lbo(smem_addr(sm + OP_WQ), 16384, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_W, kstep_kmajor(t, 64, ks), kstep_mnmajor(kc, ks), ID_KM128, ks > 0);
            mma_commit(&bars[1]);
        }
        // ---------------- -W to fp16 (over Kc, consumed by the product); the record
        ok = mbar_wait(&bars[1], 1, kWait);
        fence_after_sync();
        {
            float wv[64];
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(taddr(tm + TM_W, quarter * 32, 64 * half + 16 * j), wv + 16 * j);
            tmem_wait_ld();
            // lanes 0..15 hold the rows; lane l + 16 takes columns 32..63 of row l
            const int r = quarter * 16 + (lane & 15), hi = lane >> 4;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float t = __shfl_sync(0xffffffffu, wv[32 + j], lane & 15);
                wv[j] = -(hi ? t : wv[j]);
            }
#pragma unroll
            for (int j2 = 0; j2 < 4; ++j2) {
                st_h8(sm + OP_WQ + sw128_chunk(r, 8 * half + 4 * hi + j2, 128), wv + 8 * j2);
                big = absmax8(wv + 8 * j2, big);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0) {
            fence_after_sync();
            bulk_store(rec, sm + REC, REC_BYTES);
            bulk_commit();
        }
    }
    if (!(big <= kRange) || !(gbig <= 9.f)) record_status(status, GDN2_ERR_RANGE);
    if (tid == 0) {
        bulk_wait_all();
        if (abort) {
            record_status(status, GDN2_ERR_TIMEOUT);
            // let every requested tile land before the CTA's shared memory goes away
            if (issued > n) mbar_wait(&bars[0], (issued - 1) & 1, kWait);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

cudaError_t tc_prep_launch(const void *q, const void *k, const float *g, const float *b, void *ws,
                           unsigned int *status, const Dims &d, cudaStream_t s) {
    CUtensorMap mq, mk, mg, mb;
    if (!make_btHd_map(&mq, q, true, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mk, k, true, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mg, g, false, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mb, b, false, d.B, d.T, d.H, 128, 64, 128))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tprep::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const long long ntiles = (long long)d.B * d.H * d.NC;
    const int grid = (int)(ntiles < sm_count() ? ntiles : sm_count());
    launch_begin(K_TC_PREP, s);
    tc_prep_kernel<<<grid, tprep::kThreads, tprep::SMEM_BYTES, s>>>(
        mq, mk, mg, mb, (unsigned char *)ws, tc_ws_layout(d), status, d);
    launch_end(K_TC_PREP, s);
    return cudaGetLastError();
}

}  // namespace gdn2
