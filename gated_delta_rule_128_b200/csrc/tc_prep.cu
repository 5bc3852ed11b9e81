// Chunk-parallel part of the tensor-core forward of Gated Delta Rule-2 (bf16
// q/k, float32 g/b, d_k = 128, chunk 64): everything about a chunk that does
// not depend on the state entering it.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B): once the state is normalised by the in-chunk cumulative decay,
// the decay folds into the two factors of every rank-one erase, and a single
// unit-lower-triangular inverse serves the erase and the write side.  With
// G the in-chunk cumulative log-decay (tc_common.cuh for the frames):
//   A[r][j] = sum_c b k_r,c k_j,c e^(G_r,c - G_j,c)   (j < r)
//   P[r][j] = sum_c q_r,c k_j,c e^(G_r,c - G_j,c)     (j <= r)
//   T = (I + A)^-1,  W = T Kc,  Kc = b.k.e^G,  Qb = q.e^G,  Kb = k.e^(G_63 - G)
// The chunk's record (layout REC_* in common.cuh) receives [-W; Qb], Kb, T,
// P and gamma = e^G_63; the sequential state kernels read it.
//
// A and P come in two parts, so that no factor overflows for any g <= 0:
//  * blocks of rows I > J (16 rows each): one fp16 tcgen05.mma per row block
//    I', M = 128 rows [b.k.a; q.a] (a = e^(G - s_I), <= 1) against
//    R_I'[j] = k_j e^(s_I' - G_j) for j < 16 I' (<= 1), K = 128 channels;
//  * the four 16 x 16 diagonal blocks: warp-level tf32 products of
//    [b.k.l; q.l] against k / l (l = e^(G' - G'_m), clamped, see
//    tc_common.cuh), each warp one diagonal block and one 8-column half of it.
// T is inverted in float32 on the CUDA cores; W = T Kc is a tcgen05.mma.
//
// Persistent: one CTA per SM walks the (b, h, chunk) tiles with a stride of
// the grid size.  TMA brings the raw q, k, g, b tiles; the next tile's are
// requested as soon as the diagonal products have read this tile's.

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

namespace tprep {
constexpr int kThreads = 256;
// raw tiles (128-B swizzled boxes, tc_common.cuh raw16 / raw32); the g tile
// later holds d = G' - G'_m per element
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_G = 32768, RAW_B = 65536;
constexpr uint32_t CO = 98304;        // [b.k.a; q.a] fp16 [128][128] K-major
constexpr uint32_t RR = CO + 32768;   // R_1 (16 rows), R_2 (32), R_3 (48): fp16 K-major
__host__ __device__ constexpr uint32_t rr_off(int I) { return I <= 1 ? 0u : (I == 2 ? 4096u : 12288u); }
constexpr uint32_t REC = RR + 24576;  // the tile's record, laid out as in the workspace
constexpr uint32_t OP_WQ = REC + REC_WQ;  // [Kc; Qb], later [-W; Qb]
constexpr uint32_t OP_KB = REC + REC_KH;
constexpr uint32_t OP_T = REC + REC_T, OP_P = REC + REC_P, FAC = REC + REC_FAC;
constexpr uint32_t TOT = OP_T;        // block totals of G [4][128] f32, before T is written
// float32 scratch of the inversion, over CO / RR once the products have read them
constexpr uint32_t SCR_A = CO, SCR_T = CO + 64 * 65 * 4, SCR_M = SCR_T + 64 * 65 * 4;
constexpr uint32_t MISC = REC + REC_BYTES;  // mbarriers, TMEM slot
constexpr uint32_t SMEM_BYTES = MISC + 128 + 1024;
constexpr uint32_t TM_C = 0, TM_W = 128;  // the three block products (96 columns); W
__host__ __device__ constexpr uint32_t tm_coff(int I) { return I <= 1 ? 0u : (I == 2 ? 16u : 48u); }
constexpr uint32_t ID_KM128 = idesc_f16(64, 128, false, true);
constexpr long long kWait = 2000000000LL;  // ~1 s of SM clocks per wait
constexpr float kRange = 6.0e4f;
static_assert(MISC % 8 == 0 && REC % 1024 == 0 && RR % 1024 == 0, "alignment");
static_assert(SCR_M + 8 * 16 * 9 * 4 <= REC, "inversion scratch fits over CO / RR");
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace tprep

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

__device__ __forceinline__ float2 ld_bf2(const unsigned char *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ float ld_bf(const unsigned char *p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
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
    float *tot = reinterpret_cast<float *>(sm + TOT);
    float big = 0.f;  // range check: largest fp16 operand magnitude

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;
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
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(sm + RAW_Q + x * 8192, &mq, 64 * x, h, c * 64, bb, &bars[0]);
            tma_load_4d(sm + RAW_K + x * 8192, &mk, 64 * x, h, c * 64, bb, &bars[0]);
        }
        for (int x = 0; x < 4; ++x) {
            tma_load_4d(sm + RAW_G + x * 8192, &mg, 32 * x, h, c * 64, bb, &bars[0]);
            tma_load_4d(sm + RAW_B + x * 8192, &mb, 32 * x, h, c * 64, bb, &bars[0]);
        }
        ++issued;
    };
    if (tid == 0 && (int)blockIdx.x < ntiles) load_raw(blockIdx.x);

    // factor phase ownership: 16 rows of block fb, channels fc, fc + 1
    const int fb = tid >> 6, fc = 2 * (tid & 63);

    bool abort = false;
    int n = 0;  // tiles done by this CTA
    for (int it = blockIdx.x; it < ntiles; it += gridDim.x, ++n) {
        unsigned char *rec = ws + lay.rec + (size_t)it * REC_BYTES;
        bool ok = mbar_wait(&bars[0], n & 1, kWait);
        if (tid == 0) bulk_wait_read();  // the previous tile's record has left shared memory
        if (__syncthreads_or(!ok)) { abort = true; break; }

        // ---------------- cumulative decay of this block's 16 rows, exact and clamped
        float gl[16][2], gc[16][2];
        {
            float run[2] = {0.f, 0.f}, runc[2] = {0.f, 0.f};
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float2 g2 = *reinterpret_cast<const float2 *>(sm + RAW_G + raw32(16 * fb + r, fc));
                run[0] += g2.x;
                run[1] += g2.y;
                runc[0] += fmaxf(g2.x, -kClampG);
                runc[1] += fmaxf(g2.y, -kClampG);
                gl[r][0] = run[0];
                gl[r][1] = run[1];
                gc[r][0] = runc[0];
                gc[r][1] = runc[1];
            }
            *reinterpret_cast<float2 *>(tot + fb * 128 + fc) = make_float2(run[0], run[1]);
        }
        __syncthreads();
        // ---------------- factors: record operands, block-product operands, d
        {
            float T4[4][2];
#pragma unroll
            for (int I = 0; I < 4; ++I) {
                const float2 t2 = *reinterpret_cast<const float2 *>(tot + I * 128 + fc);
                T4[I][0] = t2.x;
                T4[I][1] = t2.y;
            }
            float eS[2], eF[2], chi[4][2];  // e^s_I, e^(G_63 - e_I), chi_{I', fb}
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float s = 0.f, all = 0.f;
#pragma unroll
                for (int I = 0; I < 4; ++I) {
                    if (I < fb) s += T4[I][i];
                    all += T4[I][i];
                }
                eS[i] = __expf(s);
                eF[i] = __expf(all - s - T4[fb][i]);
                float between = 0.f;  // sum of the block totals strictly between fb and I'
#pragma unroll
                for (int I = 0; I < 4; ++I) {
                    chi[I][i] = I == fb + 1 ? 1.f : __expf(between);
                    if (I > fb) between += T4[I][i];
                }
                if (fb == 0) reinterpret_cast<float *>(sm + FAC)[fc + i] = __expf(all);  // gamma
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int t = 16 * fb + r;
                const float2 q2 = ld_bf2(sm + RAW_Q + raw16(t, fc)), k2 = ld_bf2(sm + RAW_K + raw16(t, fc));
                const float2 b2 = *reinterpret_cast<const float2 *>(sm + RAW_B + raw32(t, fc));
                const float qv[2] = {q2.x, q2.y}, kv[2] = {k2.x, k2.y}, bv[2] = {b2.x, b2.y};
                float bka[2], qa[2], kc[2], qb[2], kb[2], ka[2], dd[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float a = __expf(gl[r][i]), ab = __expf(T4[fb][i] - gl[r][i]);
                    bka[i] = bv[i] * kv[i] * a;
                    qa[i] = qv[i] * a;
                    kc[i] = bka[i] * eS[i];
                    qb[i] = qa[i] * eS[i];
                    kb[i] = kv[i] * ab * eF[i];
                    ka[i] = kv[i] * ab;
                    dd[i] = gc[r][i] - gc[7][i];
                    big = fmaxf(big, fmaxf(fabsf(bka[i]), fmaxf(fabsf(qa[i]), fabsf(ka[i]))));
                }
                *reinterpret_cast<uint32_t *>(sm + CO + sw128_off(t, fc, 128)) = pack_f16(bka[0], bka[1]);
                *reinterpret_cast<uint32_t *>(sm + CO + sw128_off(64 + t, fc, 128)) = pack_f16(qa[0], qa[1]);
                *reinterpret_cast<uint32_t *>(sm + OP_WQ + sw128_off(t, fc, 128)) = pack_f16(kc[0], kc[1]);
                *reinterpret_cast<uint32_t *>(sm + OP_WQ + sw128_off(64 + t, fc, 128)) = pack_f16(qb[0], qb[1]);
                *reinterpret_cast<uint32_t *>(sm + OP_KB + sw128_off(t, fc, 64)) = pack_f16(kb[0], kb[1]);
#pragma unroll
                for (int I = 1; I < 4; ++I)
                    if (I > fb)
                        *reinterpret_cast<uint32_t *>(sm + RR + rr_off(I) + sw128_off(t, fc, 16 * I)) =
                            pack_f16(ka[0] * chi[I][0], ka[1] * chi[I][1]);
                *reinterpret_cast<float2 *>(sm + RAW_G + raw32(t, fc)) = make_float2(dd[0], dd[1]);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            const uint64_t co = desc_kmajor(smem_addr(sm + CO), 128, 0);
#pragma unroll
            for (int I = 1; I < 4; ++I) {
                const uint64_t rr = desc_kmajor(smem_addr(sm + RR + rr_off(I)), 16 * I, 0);
                const uint32_t id = idesc_f16(128, 16 * I, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tm + TM_C + tm_coff(I), kstep_kmajor(co, 128, ks), kstep_kmajor(rr, 16 * I, ks), id,
                             ks > 0);
            }
            mma_commit(&bars[1]);
        }
        // ---------------- diagonal blocks: warp (block db, 8 columns dn) in tf32
        const int db = warp >> 1, dn = warp & 1, gq = lane >> 2, tq = lane & 3;
        float cA[4] = {0.f, 0.f, 0.f, 0.f}, cP[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int r0 = 16 * db + gq, r1 = r0 + 8, jj = 16 * db + 8 * dn + gq;
#pragma unroll 4
            for (int k0 = 0; k0 < 128; k0 += 8) {
                uint32_t aA[4], aP[4], bb[2];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = (e & 1) ? r1 : r0, c = k0 + tq + ((e & 2) ? 4 : 0);
                    const float l = __expf(*reinterpret_cast<const float *>(sm + RAW_G + raw32(r, c)));
                    const float kv = ld_bf(sm + RAW_K + raw16(r, c)), qv = ld_bf(sm + RAW_Q + raw16(r, c));
                    const float bv = *reinterpret_cast<const float *>(sm + RAW_B + raw32(r, c));
                    aA[e] = to_tf32(bv * kv * l);
                    aP[e] = to_tf32(qv * l);
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int c = k0 + tq + 4 * e;
                    const float il = __expf(-*reinterpret_cast<const float *>(sm + RAW_G + raw32(jj, c)));
                    bb[e] = to_tf32(ld_bf(sm + RAW_K + raw16(jj, c)) * il);
                }
                mma_tf32_16x8x8(cA, aA, bb);
                mma_tf32_16x8x8(cP, aP, bb);
            }
        }
        // ---------------- assemble A (float32, for the inversion) and P (record)
        ok = mbar_wait(&bars[1], 0, kWait);
        fence_after_sync();
        __syncthreads();  // the block products have read CO / RR; the raw tiles are consumed
        if (tid == 0 && it + (int)gridDim.x < ntiles) load_raw(it + gridDim.x);
        float *sA = reinterpret_cast<float *>(sm + SCR_A);
        float *sT = reinterpret_cast<float *>(sm + SCR_T);
        {
            // diagonal blocks from the warps' fragments: rows 16 db + gq (+ 8),
            // columns 16 db + 8 dn + 2 tq (+ 1)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int rl = gq + ((e & 2) ? 8 : 0), jl = 8 * dn + 2 * tq + (e & 1);
                const int r = 16 * db + rl, j = 16 * db + jl;
                sA[r * 65 + j] = jl < rl ? cA[e] : 0.f;
                cP[e] = jl <= rl ? cP[e] : 0.f;
            }
            const int rA = 16 * db + gq, jA = 16 * db + 8 * dn + 2 * tq;
            *reinterpret_cast<uint32_t *>(sm + OP_P + sw128_off(rA, jA, 64)) = pack_f16(cP[0], cP[1]);
            *reinterpret_cast<uint32_t *>(sm + OP_P + sw128_off(rA + 8, jA, 64)) = pack_f16(cP[2], cP[3]);
            big = fmaxf(big, fmaxf(fmaxf(fabsf(cP[0]), fabsf(cP[1])), fmaxf(fabsf(cP[2]), fabsf(cP[3]))));
            // blocks above the diagonal of P are zero
            for (int e = tid; e < 64 * 8; e += kThreads) {
                const int r = e >> 3, jc = e & 7;
                if ((jc >> 1) > (r >> 4))
                    *reinterpret_cast<uint4 *>(sm + OP_P + sw128_chunk(r, jc, 64)) = make_uint4(0, 0, 0, 0);
            }
            // blocks below the diagonal from tensor memory: row r of block I
            // (lane r: A, lane 64 + r: P) needs columns j < 16 I of product I
            const int row = 32 * (quarter & 1) + lane, I = row >> 4, part = warp >> 2;
            const bool isP = quarter >= 2;
            // quarter 0/2: rows 0..31 need product 1 (16 columns, warps 0..3);
            // quarter 1/3: rows 32..47 product 2 (32 columns, warps 0..3),
            // rows 48..63 product 3 (48 columns, warps 4..7)
            const int prod = (quarter & 1) == 0 ? 1 : (part == 0 ? 2 : 3);
            if ((quarter & 1) == 1 || part == 0) {
                for (int c0 = 0; c0 < 16 * prod; c0 += 16) {
                    float v[16];
                    tmem_ld16(taddr(tm + TM_C + tm_coff(prod) + c0, quarter * 32, 0), v);
                    tmem_wait_ld();
                    if (I == prod) {
                        if (!isP) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) sA[row * 65 + c0 + j] = v[j];
                        } else {
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                st_h8(sm + OP_P + sw128_chunk(row, (c0 >> 3) + jj, 64), v + 8 * jj);
                                big = absmax8(v + 8 * jj, big);
                            }
                        }
                    }
                }
            }
        }
        fence_proxy_async();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        // ---------------- T = (I + A)^-1
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
            const int half = warp >> 2;
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
    if (!(big <= kRange)) record_status(status, GDN2_ERR_RANGE);
    if (tid == 0) {
        bulk_wait_all();
        if (abort) {
            record_status(status, GDN2_ERR_TIMEOUT);
            // let every requested tile land, and every issued product finish,
            // before the CTA's shared and tensor memory go away
            if (issued > n) mbar_wait(&bars[0], (issued - 1) & 1, kWait);
            mbar_wait(&bars[1], 0, kWait);
            mbar_wait(&bars[1], 1, kWait);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

cudaError_t tc_prep_launch(const void *q, const void *k, const float *g, const float *b, void *ws,
                           unsigned int *status, const Dims &d, cudaStream_t s) {
    CUtensorMap mq, mk, mg, mb;
    if (!make_btHd_map(&mq, q, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mk, k, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mg, g, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mb, b, false, d.B, d.T, d.H, 128, 64, 32, true))
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
