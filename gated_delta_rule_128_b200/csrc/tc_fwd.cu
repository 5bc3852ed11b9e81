// Fused chunkwise forward of Gated Delta Rule-2 on the sm_100a tensor cores,
// for bf16 q/k/v/o, float32 gates and state, d_k = d_v = 128, chunk 64.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B): the state is normalised by the in-chunk cumulative decay, so the
// channel-wise decay folds into the two factors of every rank-one erase, one
// WY/UT inverse serves the erase and the write side, and only the state
// crosses chunk borders.  Per chunk of 64 tokens entering with state S:
//   G = cumsum(g);  Qb = q.e^G,  Kc = b.k.e^G,  Kh = k.e^-G,  U = w.v
//   A = strictly-lower(Kc Kh^T),  P = lower-incl(Qb Kh^T),  T = (I + A)^-1
//   W = T Kc,  U' = T U,  Delta = U' - W S
//   O = Qb S + P Delta,   S_next = diag(e^G_L) (S + Kh^T Delta)
//
// One CTA owns one (b, h) and one 64-column half of d_v, and walks the
// sequence's chunks in order with its fp32 state slice resident in tensor
// memory.  Per chunk: TMA brings the raw q, k, v, w, g, b tiles into shared
// memory (the next chunk's tiles are requested as soon as this chunk's are
// consumed); the CUDA cores form the decay-scaled fp16 operands; seven
// tcgen05.mma groups (kind::f16 with fp16 operands, f32 accumulators in TMEM)
// form A, P, QbS, W|U', WS, P Delta and Kh^T Delta; the unit-lower-triangular
// T is inverted in float32 on the CUDA cores by blocked forward substitution
// (16x16 diagonal blocks, then three block levels).
//
// Precision and range: fp16 operands carry 11 significant bits (bf16 carries
// 8, which left the output error at the 5e-3 tolerance).  To keep them in
// fp16 range the decay factors are taken relative to the chunk's middle row
// m = 31 (see tc_common.cuh); the state products then use S_m = diag(e^G_m) S
// and the update becomes S_next = diag(e^(G_L-G_m)) (S_m + Kh^T Delta).  Any
// operand beyond 6e4 in magnitude is reported as GDN2_ERR_RANGE.
//
// For the backward the call can also leave in the workspace (TcWs): every
// chunk-entry state and S_T (fp16), T and P per chunk, and Delta per chunk.

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

namespace tfwd {
constexpr int kThreads = 256;
// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_V = 32768, RAW_W = 40960, RAW_G = 57344,
                   RAW_B = 90112;
constexpr uint32_t OP_KC = 122880;  // Kc, later W        [64 pos][128 key]  K-major
constexpr uint32_t OP_QB = 139264;  // Qb                 [64 pos][128 key]
constexpr uint32_t OP_KH = 155648;  // Kh                 [64 pos][128 key]
constexpr uint32_t OP_S = 172032;   // S_m (fp16)         [128 key][64 v]    MN-major B
constexpr uint32_t OP_U = 188416;   // U, later Delta     [64 pos][64 v]     MN-major B
constexpr uint32_t OP_T = 196608;   // T                  [64 r][64 j]       K-major
constexpr uint32_t OP_P = 204800;   // P                  [64 r][64 j]       K-major
constexpr uint32_t MISC = 212992;   // e^(G_L-G_m), e^G_m [128] f32 each, mbarriers, TMEM slot
constexpr uint32_t SMEM_BYTES = MISC + 1024 + 128 + 1024;
// float32 scratch while inverting T (inside the raw g/b tiles, reloaded after)
constexpr uint32_t SCR_A = RAW_G, SCR_T = RAW_G + 64 * 65 * 4, SCR_M = SCR_T + 64 * 65 * 4;
constexpr uint32_t SCR_SCAN = OP_T;  // per-warp cumsum totals [8][128] f32 during phase 1
// tensor memory columns (512 allocated)
constexpr uint32_t TM_S = 0, TM_A = 64, TM_P = 128, TM_WU = 192, TM_WS = 384, TM_O = 448;
constexpr uint32_t ID_KK64 = idesc_f16(64, 64, false, false);
constexpr uint32_t ID_KM64 = idesc_f16(64, 64, false, true);
constexpr uint32_t ID_KM128 = idesc_f16(64, 128, false, true);
constexpr uint32_t ID_MM128x64 = idesc_f16(128, 64, true, true);
constexpr long long kWait = 2000000000LL;  // ~1 s of SM clocks per wait
constexpr float kRange = 6.0e4f;           // largest operand magnitude kept in fp16
}  // namespace tfwd

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

__global__ void __launch_bounds__(tfwd::kThreads, 1)
tc_fwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
              const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mg,
              const __grid_constant__ CUtensorMap mb, const __grid_constant__ CUtensorMap mw,
              const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ ST,
              unsigned char *__restrict__ ws, TcWs lay, unsigned int *status, Dims d) {
    using namespace tfwd;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *sGam = reinterpret_cast<float *>(sm + MISC);        // e^(G_L - G_m)
    float *sRef = reinterpret_cast<float *>(sm + MISC + 512);  // e^G_m
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC + 1024);  // 0 qkvw, 1 gb, 2..5 mma
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 1024 + 64);
    float big = 0.f;   // largest operand magnitude seen (range check)
    float gbig = 0.f;  // largest |G - G_m| seen (range check of the decay factors)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int vh = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, v0 = vh * 64;
    const int NC = d.NC, T = d.T, H = d.H;
    const int quarter = warp & 3, half = warp >> 2;
    const size_t bh = (size_t)bb * H + h;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    int issued_qkvw = 0, issued_gb = 0;  // loads requested so far (thread 0)
    auto load_qkvw = [&](int cc) {
        mbar_expect_tx(&bars[0], 16384 * 2 + 8192 + 16384);
        tma_load_4d(sm + RAW_Q, &mq, 0, h, cc * 64, bb, &bars[0]);
        tma_load_4d(sm + RAW_K, &mk, 0, h, cc * 64, bb, &bars[0]);
        tma_load_4d(sm + RAW_V, &mv, v0, h, cc * 64, bb, &bars[0]);
        tma_load_4d(sm + RAW_W, &mw, v0, h, cc * 64, bb, &bars[0]);
        ++issued_qkvw;
    };
    auto load_gb = [&](int cc) {
        mbar_expect_tx(&bars[1], 32768 * 2);
        tma_load_4d(sm + RAW_G, &mg, 0, h, cc * 64, bb, &bars[1]);
        tma_load_4d(sm + RAW_B, &mb, 0, h, cc * 64, bb, &bars[1]);
        ++issued_gb;
    };
    if (tid == 0) {
        load_qkvw(0);
        load_gb(0);
    }

    const size_t so = st_off(d, bb, h);
    // initial state slice: fp32 into TMEM, fp16 (true scale) into OP_S for the checkpoint
    {
        const int key = quarter * 32 + lane, c0 = half * 32;
        float x[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 t = S0 ? *reinterpret_cast<const float4 *>(S0 + so + (size_t)key * 128 + v0 + c0 + j)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
            x[j] = t.x; x[j + 1] = t.y; x[j + 2] = t.z; x[j + 3] = t.w;
        }
        tmem_st16(taddr(tm + TM_S, quarter * 32, c0), x);
        tmem_st16(taddr(tm + TM_S, quarter * 32, c0 + 16), x + 16);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            st_h8(sm + OP_S + sw128_chunk(key, half * 4 + jj, 128), x + 8 * jj);
            big = absmax8(x + 8 * jj, big);
        }
        tmem_wait_st();
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    if (tid == 0 && ws) {
        bulk_store(ws + lay.ckS + ((bh * (NC + 1) + 0) * 2 + vh) * 16384, sm + OP_S, 16384);
        bulk_commit();
    }

    bool abort = false;
    for (int c = 0; c < NC; ++c) {
        const uint32_t par = c & 1;
        const int c0 = c * 64;
        // ---------------- phase 1: cumulative decay and operands
        bool ok = mbar_wait(&bars[0], par, kWait);
        ok = ok && mbar_wait(&bars[1], par, kWait);
        float G[8][4];
        cumsum_local(reinterpret_cast<const float *>(sm + RAW_G), reinterpret_cast<float *>(sm + SCR_SCAN),
                     warp, lane, G);
        if (__syncthreads_or(!ok)) { abort = true; break; }
        cumsum_finish(reinterpret_cast<const float *>(sm + SCR_SCAN), warp, lane, G, sGam, sRef);
        gbig = fmaxf(gbig, write_factors(sm + RAW_Q, sm + RAW_K, reinterpret_cast<const float *>(sm + RAW_B),
                                       G, sm + OP_QB, sm + OP_KC, sm + OP_KH, warp, lane));
        if (lane < 16) {
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int r = 8 * warp + m;
                uint2 vr = *reinterpret_cast<const uint2 *>(sm + RAW_V + r * 128 + lane * 8);
                float4 wv = *reinterpret_cast<const float4 *>(sm + RAW_W + r * 256 + lane * 16);
                const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vr);
                float u[4] = {wv.x * __low2float(v2[0]), wv.y * __high2float(v2[0]),
                              wv.z * __low2float(v2[1]), wv.w * __high2float(v2[1])};
                st_h4(sm + OP_U + sw128_off(r, 4 * lane, 64), u[0], u[1], u[2], u[3]);
#pragma unroll
                for (int i = 0; i < 4; ++i) big = fmaxf(big, fabsf(u[i]));
            }
        }
        if (tid == 0 && ws) bulk_wait_read();  // OP_S is rewritten just below
        __syncthreads();
        // state in the chunk's reference frame: S_m = diag(e^G_m) S (TMEM and fp16 copy)
        {
            const int key = quarter * 32 + lane;
            float sv[32];
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half), sv);
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), sv + 16);
            tmem_wait_ld();
            const float e = sRef[key];
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] *= e;
            tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half), sv);
            tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), sv + 16);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                st_h8(sm + OP_S + sw128_chunk(key, 4 * half + jj, 128), sv + 8 * jj);
                big = absmax8(sv + 8 * jj, big);
            }
            tmem_wait_st();
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            if (c + 1 < NC) load_qkvw(c + 1);
            const uint32_t kc = smem_addr(sm + OP_KC), qb = smem_addr(sm + OP_QB),
                           kh = smem_addr(sm + OP_KH), s = smem_addr(sm + OP_S);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_A, desc_kmajor(kc, 64, ks), desc_kmajor(kh, 64, ks), ID_KK64, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_P, desc_kmajor(qb, 64, ks), desc_kmajor(kh, 64, ks), ID_KK64, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_O, desc_kmajor(qb, 64, ks), desc_mnmajor(s, 128, ks), ID_KM64, ks > 0);
            mma_commit(&bars[2]);
        }
        // ---------------- phase 3: T = (I + A)^-1 and the masked P
        ok = mbar_wait(&bars[2], par, kWait);
        fence_after_sync();
        float *sA = reinterpret_cast<float *>(sm + SCR_A);
        float *sT = reinterpret_cast<float *>(sm + SCR_T);
        {
            float row[64];
            const uint32_t base = warp < 4 ? tm + TM_A : tm + TM_P;
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(taddr(base, quarter * 32, 16 * j), row + 16 * j);
            tmem_wait_ld();
            if (lane < 16) {
                const int r = quarter * 16 + lane;
                if (warp < 4) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) sA[r * 65 + j] = j < r ? row[j] : 0.f;
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) row[j] = j <= r ? row[j] : 0.f;
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        st_h8(sm + OP_P + sw128_chunk(r, jj, 64), row + 8 * jj);
                        big = absmax8(row + 8 * jj, big);
                    }
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
            if (c + 1 < NC) load_gb(c + 1);
            if (ws && vh == 0) {  // T and P of this chunk, for the backward
                unsigned char *dst = ws + lay.ckTP + (bh * NC + c) * 16384;
                bulk_store(dst, sm + OP_T, 8192);
                bulk_store(dst + 8192, sm + OP_P, 8192);
                bulk_commit();
            }
            const uint32_t t = smem_addr(sm + OP_T), kc = smem_addr(sm + OP_KC),
                           u = smem_addr(sm + OP_U);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_WU, desc_kmajor(t, 64, ks), desc_mnmajor(kc, 64, ks), ID_KM128, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_WU + 128, desc_kmajor(t, 64, ks), desc_mnmajor(u, 64, ks), ID_KM64, ks > 0);
            mma_commit(&bars[3]);
        }
        // ---------------- phase 5: W to shared memory (keep U' in registers)
        ok = mbar_wait(&bars[3], par, kWait);
        fence_after_sync();
        float up[32];
        {
            float wv[64];
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(taddr(tm + TM_WU, quarter * 32, 64 * half + 16 * j), wv + 16 * j);
            tmem_ld16(taddr(tm + TM_WU, quarter * 32, 128 + 32 * half), up);
            tmem_ld16(taddr(tm + TM_WU, quarter * 32, 128 + 32 * half + 16), up + 16);
            tmem_wait_ld();
            if (lane < 16) {
                const int r = quarter * 16 + lane;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    st_h8(sm + OP_KC + sw128_chunk(r, 8 * half + jj, 64), wv + 8 * jj);
                    big = absmax8(wv + 8 * jj, big);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0) {
            fence_after_sync();
            const uint32_t w = smem_addr(sm + OP_KC), s = smem_addr(sm + OP_S);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_WS, desc_kmajor(w, 64, ks), desc_mnmajor(s, 128, ks), ID_KM64, ks > 0);
            mma_commit(&bars[4]);
        }
        // ---------------- phase 7: Delta = U' - W S
        ok = mbar_wait(&bars[4], par, kWait);
        fence_after_sync();
        {
            float ws_[32];
            tmem_ld16(taddr(tm + TM_WS, quarter * 32, 32 * half), ws_);
            tmem_ld16(taddr(tm + TM_WS, quarter * 32, 32 * half + 16), ws_ + 16);
            tmem_wait_ld();
            if (lane < 16) {
                const int r = quarter * 16 + lane;
#pragma unroll
                for (int j = 0; j < 32; ++j) ws_[j] = up[j] - ws_[j];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    st_h8(sm + OP_U + sw128_chunk(r, 4 * half + jj, 64), ws_ + 8 * jj);
                    big = absmax8(ws_ + 8 * jj, big);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0) {
            fence_after_sync();
            if (ws) {  // Delta of this chunk and half, for the backward
                bulk_store(ws + lay.ckD + ((bh * NC + c) * 2 + vh) * 8192, sm + OP_U, 8192);
                bulk_commit();
            }
            const uint32_t p = smem_addr(sm + OP_P), dl = smem_addr(sm + OP_U),
                           kh = smem_addr(sm + OP_KH);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_O, desc_kmajor(p, 64, ks), desc_mnmajor(dl, 64, ks), ID_KM64, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_S, desc_mnmajor(kh, 64, ks), desc_mnmajor(dl, 64, ks), ID_MM128x64, 1);
            mma_commit(&bars[5]);
        }
        // ---------------- phase 9: output rows, state update and checkpoint
        ok = mbar_wait(&bars[5], par, kWait);
        fence_after_sync();
        {
            float ov[32];
            tmem_ld16(taddr(tm + TM_O, quarter * 32, 32 * half), ov);
            tmem_ld16(taddr(tm + TM_O, quarter * 32, 32 * half + 16), ov + 16);
            tmem_wait_ld();
            if (lane < 16) {
                const int r = quarter * 16 + lane;
                if (o && c0 + r < T) {
                    unsigned char *dst = reinterpret_cast<unsigned char *>(
                        o + tok(d, bb, c0 + r, h, 128) + v0 + 32 * half);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) st_bf16x8(dst + 16 * jj, ov + 8 * jj);
                }
            }
            const int key = quarter * 32 + lane;
            float sv[32];
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half), sv);
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), sv + 16);
            tmem_wait_ld();
            const float gk = sGam[key];
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] *= gk;
            tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half), sv);
            tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), sv + 16);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                st_h8(sm + OP_S + sw128_chunk(key, 4 * half + jj, 128), sv + 8 * jj);
                big = absmax8(sv + 8 * jj, big);
            }
            if (c == NC - 1 && ST) {
                float *dst = ST + so + (size_t)key * 128 + v0 + 32 * half;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
            }
            tmem_wait_st();
        }
        // the T/P and Delta copies read OP_T, OP_P and OP_U, all rewritten next chunk
        if (tid == 0 && ws) bulk_wait_read();
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0 && ws) {  // S_{c+1} (S_T after the last chunk), true scale
            bulk_store(ws + lay.ckS + ((bh * (NC + 1) + c + 1) * 2 + vh) * 16384, sm + OP_S, 16384);
            bulk_commit();
        }
    }
    if (!(big <= kRange) || !(gbig <= 9.f)) record_status(status, GDN2_ERR_RANGE);
    if (tid == 0) {
        if (ws) bulk_wait_all();
        if (abort) {
            record_status(status, GDN2_ERR_TIMEOUT);
            // let every requested tile land before the CTA's shared memory goes away
            if (issued_qkvw > 0) mbar_wait(&bars[0], (issued_qkvw - 1) & 1, kWait);
            if (issued_gb > 0) mbar_wait(&bars[1], (issued_gb - 1) & 1, kWait);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------- launcher
cudaError_t tc_fwd_launch(const void *q, const void *k, const void *v, const float *g,
                          const float *b, const float *w, const float *S0, void *o, float *ST,
                          void *ws, unsigned int *status, const Dims &d, cudaStream_t s) {
    CUtensorMap mq, mk, mv, mg, mb, mw;
    if (!make_btHd_map(&mq, q, true, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mk, k, true, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mv, v, true, d.B, d.T, d.H, 128, 64, 64) ||
        !make_btHd_map(&mg, g, false, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mb, b, false, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mw, w, false, d.B, d.T, d.H, 128, 64, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tc_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tfwd::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    launch_begin(K_TC_FWD, s);
    tc_fwd_kernel<<<dim3(2, d.H, d.B), tfwd::kThreads, tfwd::SMEM_BYTES, s>>>(
        mq, mk, mv, mg, mb, mw, S0, (__nv_bfloat16 *)o, ST, (unsigned char *)ws, tc_ws_layout(d),
        status, d);
    launch_end(K_TC_FWD, s);
    return cudaGetLastError();
}

}  // namespace gdn2
