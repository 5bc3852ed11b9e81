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
// P, gamma = e^G_63 and a frame factor s; the sequential state kernels read it.
//
// A mild tile (tc_common.cuh: every channel's G within e^4 of its row 31)
// takes one frame for the whole chunk: Kc, Qb, Kb above are taken times
// e^-G_31 (Kb times e^G_31 / e^G_63, i.e. Kh = k e^(G_31 - G)), s = e^G_31,
// and A and P come from one fp16 product [Kc; Qb] Kh^T.  Any other tile keeps
// the chunk-start frame (s = 1, stored as -1 to mark it) and takes A and P in
// two parts, so that no factor overflows for any g <= 0:
//  * blocks of rows I > J (16 rows each): one fp16 tcgen05.mma per row block
//    I', M = 128 rows [b.k.a; q.a] (a = e^(G - s_I), <= 1) against
//    R_I'[j] = k_j e^(s_I' - G_j) for j < 16 I' (<= 1), K = 128 channels;
//  * the four 16 x 16 diagonal blocks: warp-level tf32 products of
//    [b.k.l; q.l] against k / l (l = e^(G' - G'_m), clamped, see
//    tc_common.cuh), each warp one diagonal block and one 8-column half of it.
// T is inverted on the CUDA cores (float32 diagonal blocks, tf32 block
// columns); W = T Kc is a tcgen05.mma.
//
// Persistent: one CTA per SM walks the (b, h, chunk) tiles with a stride of
// the grid size.  TMA brings the raw q, k, g, b tiles; the next tile's are
// requested during the inversion, by a warp that is idle then (issuing a TMA
// load holds its thread a long time).  The record leaves by bulk copies in
// four pieces, each as soon as it is final.

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

namespace tprep {
constexpr int kThreads = 256;
// raw tiles (128-B swizzled boxes, tc_common.cuh raw16 / raw32; g and b as
// float32 or bf16, graw); the g tile later holds d = G' - G'_m per element
// (float32, raw32), once the cumulative decay has read g
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_G = 32768, RAW_B = 65536;
constexpr uint32_t CO = 98304;        // [b.k.a; q.a] fp16 [128][128] K-major
constexpr uint32_t RR = CO + 32768;   // R_1 (16 rows), R_2 (32), R_3 (48): fp16 K-major
__host__ __device__ constexpr uint32_t rr_off(int I) { return I <= 1 ? 0u : (I == 2 ? 4096u : 12288u); }
constexpr uint32_t REC = RR + 24576;  // the tile's record, laid out as in the workspace
constexpr uint32_t OP_WQ = REC + REC_WQ;  // [Kc; Qb], later [-W; Qb]
constexpr uint32_t OP_KB = REC + REC_KH;
constexpr uint32_t OP_T = REC + REC_T, OP_P = REC + REC_P, FAC = REC + REC_FAC;
// float32 scratch of the inversion, over CO / RR once the products have read them:
// A with rows kSA floats apart and T with rows kST apart (row strides chosen so
// that the warp-level tile loads of either operand role avoid bank conflicts)
constexpr int kSA = 68, kST = 72;
constexpr uint32_t SCR_A = CO, SCR_T = CO + 64 * kSA * 4, SCR_M = SCR_T + 64 * kST * 4;
constexpr uint32_t MISC = REC + REC_BYTES;  // mbarriers, TMEM slot
// 8-row totals of G [2][8][128] f32, outside the record so that they can be
// formed while the previous tile's record is still leaving
constexpr uint32_t TOT = MISC + 128;
constexpr uint32_t SMEM_BYTES = TOT + 8192 + 1024;
constexpr uint32_t TM_C = 0, TM_W = 128;  // the three block products (96 columns); W
__host__ __device__ constexpr uint32_t tm_coff(int I) { return I <= 1 ? 0u : (I == 2 ? 16u : 48u); }
constexpr uint32_t ID_WP128 = idesc_f16(128, 128, false, true);
constexpr uint32_t ID_KK128x64 = idesc_f16(128, 64, false, false);
constexpr long long kWait = 2000000000LL;  // ~1 s of SM clocks per wait
constexpr float kRange = 6.0e4f;
static_assert(MISC % 8 == 0 && REC % 1024 == 0 && RR % 1024 == 0, "alignment");
static_assert(SCR_M + 8 * 16 * 9 * 4 <= REC, "inversion scratch fits over CO / RR");
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace tprep

// c += X[r0.., k0..k0+8) * Y[k0..k0+8, n0..n0+8) for row-major f32 tiles with
// rows SX and SY floats apart
template <int SX, int SY>
__device__ __forceinline__ void tile_mma(float *c, const float *X, int r0, int k0, const float *Y,
                                         int n0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    uint32_t a[4] = {to_tf32(X[(r0 + g) * SX + k0 + t]), to_tf32(X[(r0 + g + 8) * SX + k0 + t]),
                     to_tf32(X[(r0 + g) * SX + k0 + t + 4]), to_tf32(X[(r0 + g + 8) * SX + k0 + t + 4])};
    uint32_t b[2] = {to_tf32(Y[(k0 + t) * SY + n0 + g]), to_tf32(Y[(k0 + t + 4) * SY + n0 + g])};
    mma_tf32_16x8x8(c, a, b);
}

// T = (I + A)^-1 for the strictly-lower 64x64 A in sA (f32, rows kSA apart),
// written as fp16 into the record's T tile rT ([64][64] K-major, 128-byte
// swizzle); returns the running largest magnitude of T.  Blocks of 16: the
// four diagonal blocks by forward substitution (one column per thread, 64
// threads) into sT (f32, rows kST apart), while the other warps clear the
// blocks above the diagonal of rT.  Then warp w owns the 8 columns n0 = 8 w of
// block column J = w / 2 and walks down it, T_IJ = -T_II sum_{K=J}^{I-1}
// A_IK T_KJ for I = J+1 .. 3, as warp-level tf32 tile products.  A warp reads
// back only the diagonal blocks and what it wrote itself, so the block levels
// need no barrier across warps.  sM holds one 16x8 intermediate per warp
// ([8][16][9] f32).  Warp 7 has no block below its diagonal block: its lane 0
// runs `idle` during the block columns.  All 256 threads; the caller fences
// and synchronises.
template <typename Idle>
__device__ __forceinline__ float invert_unit_lower(const float *sA, float *sT, float *sM,
                                                   unsigned char *rT, int tid, float big, Idle &&idle) {
    using tprep::kSA;
    using tprep::kST;
    if (tid < 64) {
        // column cl of the block's inverse, right-looking: once x[j] is final,
        // every later row takes its term at once, so the dependent chain is
        // 16 multiply-adds long instead of 120
        const int o16 = (tid >> 4) * 16, cl = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = r == cl ? 1.f : 0.f;
#pragma unroll
        for (int j = 0; j < 15; ++j) {
            const float xj = x[j];
#pragma unroll
            for (int r = j + 1; r < 16; ++r) x[r] = fmaf(-sA[(o16 + r) * kSA + o16 + j], xj, x[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(o16 + r) * kST + o16 + cl] = x[r];
    } else {
        // 16-byte chunks of rT above the diagonal blocks
        for (int e = tid - 64; e < 64 * 8; e += 192) {
            const int r = e >> 3, jc = e & 7;
            if ((jc >> 1) > (r >> 4)) *reinterpret_cast<uint4 *>(rT + sw128_chunk(r, jc, 64)) = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int J = warp >> 1, n0 = 8 * warp;
    if (lane < 16) {  // this warp's columns of the diagonal block, one row a lane
        const float *src = sT + (16 * J + lane) * kST + n0;
        st_h8(rT + sw128_chunk(16 * J + lane, warp, 64), src);
        big = absmax8(src, big);
    }
    if (tid == 224) idle();
    // right-looking over the block rows: acc[I] collects sum_K A_IK T_KJ, and
    // once T_IJ is final every lower block row takes its term at once, so the
    // dependent chain is two tile products per block row
    float *mw = sM + warp * 16 * 9;
    float acc[4][4] = {};
#pragma unroll
    for (int I = 1; I < 4; ++I)
        if (I > J) {
            tile_mma<kSA, kST>(acc[I], sA, 16 * I, 16 * J, sT, n0, lane);
            tile_mma<kSA, kST>(acc[I], sA, 16 * I, 16 * J + 8, sT, n0, lane);
        }
#pragma unroll
    for (int I = 1; I < 4; ++I) {
        if (I <= J) continue;
        mw[g * 9 + 2 * t] = acc[I][0];
        mw[g * 9 + 2 * t + 1] = acc[I][1];
        mw[(g + 8) * 9 + 2 * t] = acc[I][2];
        mw[(g + 8) * 9 + 2 * t + 1] = acc[I][3];
        __syncwarp();
        float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 16; k0 += 8) {
            uint32_t a[4] = {to_tf32(sT[(16 * I + g) * kST + 16 * I + k0 + t]),
                             to_tf32(sT[(16 * I + g + 8) * kST + 16 * I + k0 + t]),
                             to_tf32(sT[(16 * I + g) * kST + 16 * I + k0 + t + 4]),
                             to_tf32(sT[(16 * I + g + 8) * kST + 16 * I + k0 + t + 4])};
            uint32_t b[2] = {to_tf32(mw[(k0 + t) * 9 + g]), to_tf32(mw[(k0 + t + 4) * 9 + g])};
            mma_tf32_16x8x8(e, a, b);
        }
        // T_IJ = -e: rows 16 I + g (+ 8), columns n0 + 2 t (+ 1)
        const int r = 16 * I + g, cc = n0 + 2 * t;
        sT[r * kST + cc] = -e[0];
        sT[r * kST + cc + 1] = -e[1];
        sT[(r + 8) * kST + cc] = -e[2];
        sT[(r + 8) * kST + cc + 1] = -e[3];
        *reinterpret_cast<uint32_t *>(rT + sw128_off(r, cc, 64)) = pack_f16(-e[0], -e[1]);
        *reinterpret_cast<uint32_t *>(rT + sw128_off(r + 8, cc, 64)) = pack_f16(-e[2], -e[3]);
        big = fmaxf(big, fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3]))));
        __syncwarp();  // T_IJ before the lower block rows read it; mw free again
#pragma unroll
        for (int I2 = I + 1; I2 < 4; ++I2) {
            tile_mma<kSA, kST>(acc[I2], sA, 16 * I2, 16 * I, sT, n0, lane);
            tile_mma<kSA, kST>(acc[I2], sA, 16 * I2, 16 * I + 8, sT, n0, lane);
        }
    }
    return big;
}

__device__ __forceinline__ float2 ld_bf2(const unsigned char *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ float ld_bf(const unsigned char *p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}

template <bool GB, bool ACT>  // g, b as bf16 (else float32); ACT: gate logits (GateAct)
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
    float *tot = reinterpret_cast<float *>(sm + TOT);         // [8 row groups][128]
    float *totc = reinterpret_cast<float *>(sm + TOT + 4096);  // the same, clamped
    float big = 0.f;  // range check: largest fp16 operand magnitude

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;
    const int ntiles = total_tiles(d);
    const GateAct ga = ACT ? gate_act(d.act) : GateAct{false, 1.f};  // logits in: g, b activated on load

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

    // raw-tile loads requested: counted by every thread (the conditions are
    // uniform); thread 0 requests the first tile, thread 224 the later ones
    int issued = 0;
    auto load_raw = [&](int it) {
        int n, h, c;
        tile_decode(d, it, n, h, c);
        const Seq sq = seq_of(d, n);
        const int row0 = sq.bos + 64 * c, bb = sq.brow;
        mbar_expect_tx(&bars[0], 16384 * 2 + gate_tile_bytes<GB>() * 2);
        tma_load_5d(sm + RAW_Q, &mq, 0, h, row0, 0, bb, &bars[0]);
        tma_load_5d(sm + RAW_K, &mk, 0, h, row0, 0, bb, &bars[0]);
        tma_load_5d(sm + RAW_G, &mg, 0, h, row0, 0, bb, &bars[0]);
        tma_load_5d(sm + RAW_B, &mb, 0, h, row0, 0, bb, &bars[0]);
    };
    if ((int)blockIdx.x < ntiles) {
        if (tid == 0) load_raw(blockIdx.x);
        issued = 1;
    }

    // the record leaves in pieces, each as soon as it is final (thread 64's
    // bulk group): [Kx] and the Qb rows of [-W; Qb]; P and the factors; T; -W
    auto store_piece = [&](unsigned char *rec, uint32_t off, uint32_t bytes) {
        bulk_store(rec + off, sm + REC + off, bytes);
    };
    auto store_early = [&](unsigned char *rec) {
        if (tid == 64) {
            fence_after_sync();
            store_piece(rec, REC_KH, 16384);
            store_piece(rec, REC_WQ + 8192, 8192);
            store_piece(rec, REC_WQ + 24576, 8192);
            bulk_commit();
        }
    };

    // factor phase ownership: warp = 8 rows (block fb, half fh), lane = 4 channels from fc4
    const int fb = warp >> 1, fh = warp & 1, fc4 = 4 * lane;

    bool abort = false;
    int n = 0;  // tiles done by this CTA
    // rows of tile `it` inside its sequence (64 unless a packed sequence ends in it)
    auto rows_of = [&](int it) {
        int tn, th, tc;
        tile_decode(d, it, tn, th, tc);
        return seq_of(d, tn).len - 64 * tc;
    };
    int L_next = (int)blockIdx.x < ntiles ? rows_of(blockIdx.x) : 0;
    for (int it = blockIdx.x; it < ntiles; it += gridDim.x, ++n) {
        unsigned char *rec = ws + lay.rec + (size_t)it * REC_BYTES;
        bool ok = mbar_wait(&bars[0], n & 1, kWait);
        if (__syncthreads_or(!ok)) { abort = true; break; }
        // rows L.. of the tile lie past its sequence's end
        const int L = L_next;  // found during the previous tile
        if (d.cu && L < 64) {  // packed sequences: those rows belong to the next one
            zero_rows(sm + RAW_Q, 12, L, tid, kThreads);  // q, k, g, b: 96 KB of 8 KB boxes
            __syncthreads();
        }

        // ---------------- cumulative decay (log2 units) of this warp's 8 rows,
        // exact and clamped; lane fq owns channels 4 fq .. 4 fq + 3
        float gl[8][4], gc[8][4];
        {
            float run[4] = {0.f, 0.f, 0.f, 0.f}, runc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // past the end, no decay (a zero logit would activate to log 1/2)
                const float4 g4 = 8 * warp + i < L ? act_g4(ga, gld4<GB>(sm + RAW_G + graw<GB>(8 * warp + i, fc4)))
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                const float gv[4] = {g4.x * kLog2e, g4.y * kLog2e, g4.z * kLog2e, g4.w * kLog2e};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    run[e] += gv[e];
                    runc[e] += fmaxf(gv[e], -kClampG2);
                    gl[i][e] = run[e];
                    gc[i][e] = runc[e];
                }
            }
            *reinterpret_cast<float4 *>(tot + warp * 128 + fc4) = make_float4(run[0], run[1], run[2], run[3]);
            *reinterpret_cast<float4 *>(totc + warp * 128 + fc4) = make_float4(runc[0], runc[1], runc[2], runc[3]);
        }
        if (tid == 64) bulk_wait_read();  // the previous tile's record has left shared memory
        __syncthreads();
        // ---------------- mild tile?  Then the whole chunk fits one frame
        // relative to its row 31: every factor e^(+-(G - G_31)) stays within
        // e^kMildG, and one fp16 product gives A and P (tc_common.cuh).
        bool mild;
        {
            float pre[4] = {0.f, 0.f, 0.f, 0.f}, g31[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int r8 = 0; r8 < 8; ++r8) {
                const float4 t4 = *reinterpret_cast<const float4 *>(tot + r8 * 128 + fc4);
                const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (r8 < warp) pre[e] += tv[e];
                    if (r8 < 4) g31[e] += tv[e];
                }
            }
            // the mild test, and the mild tile's operands written speculatively (a
            // steep tile overwrites them): Kc = b k E, Qb = q E, Kh = k / E with
            // E = e^(G - G_31)
            float dmax = 0.f, xmax = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = 8 * warp + i;
                float qv[4], kv[4];
                ld_bf4(sm + RAW_Q + raw16(t, fc4), qv);
                ld_bf4(sm + RAW_K + raw16(t, fc4), kv);
                const float4 b4 = act_b4(ga, gld4<GB>(sm + RAW_B + graw<GB>(t, fc4)));
                const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
                float kcm[4], qbm[4], khm[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float dl = pre[e] + gl[i][e] - g31[e];
                    dmax = fmaxf(dmax, fabsf(dl));
                    const float bk = bv[e] * kv[e];
                    xmax = fmaxf(xmax, fmaxf(fabsf(qv[e]), fmaxf(fabsf(kv[e]), fabsf(bk))));
                    const float E = ex2(dl), Ei = ex2(-dl);
                    kcm[e] = bk * E;
                    qbm[e] = qv[e] * E;
                    khm[e] = kv[e] * Ei;
                }
                st_h4v(sm + OP_WQ + sw128_off(t, fc4, 128), kcm);
                st_h4v(sm + OP_WQ + sw128_off(64 + t, fc4, 128), qbm);
                st_h4v(sm + OP_KB + sw128_off(t, fc4, 64), khm);
            }
            fence_proxy_async();
            fence_before_sync();
            mild = !__syncthreads_or(!(dmax <= kMildG2 && xmax <= kMildX));
            if (mild) {
                // ---------------- mild: the record takes the single frame of row 31:
                // the frame factor s = e^G_31; A and P are [Kc; Qb] Kh^T
                float all[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r8 = 0; r8 < 8; ++r8) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(tot + r8 * 128 + fc4);
                    all[0] += t4.x; all[1] += t4.y; all[2] += t4.z; all[3] += t4.w;
                }
                if (warp == 0) {
                    *reinterpret_cast<float4 *>(sm + FAC + 4 * fc4) =
                        make_float4(ex2(all[0]), ex2(all[1]), ex2(all[2]), ex2(all[3]));  // gamma
                    *reinterpret_cast<float4 *>(sm + FAC + 512 + 4 * fc4) =
                        make_float4(ex2(g31[0]), ex2(g31[1]), ex2(g31[2]), ex2(g31[3]));  // s
                }
                if (tid == 0) {
                    fence_after_sync();
                    const uint64_t co = desc_kmajor(smem_addr(sm + OP_WQ), 128, 0),
                                   kh = desc_kmajor(smem_addr(sm + OP_KB), 64, 0);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(tm + TM_C, kstep_kmajor(co, 128, ks), kstep_kmajor(kh, 64, ks), ID_KK128x64, ks > 0);
                    mma_commit(&bars[1]);
                }
                store_early(rec);
            }
        }
        float cA[4] = {0.f, 0.f, 0.f, 0.f}, cP[4] = {0.f, 0.f, 0.f, 0.f};
        const int db = warp >> 1, dn = warp & 1, gq = lane >> 2, tq = lane & 3;
        if (!mild) {
        // ---------------- factors: record operands, block-product operands, d
        {
            // per channel: the four block totals; s (before this block), the
            // block's first-half and whole totals, G_63; chi_{I', fb}
            float btot[4][4], h0[4], h0c[4], sg[4], bt[4], all[4];
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                const float4 a4 = *reinterpret_cast<const float4 *>(tot + (2 * J) * 128 + fc4);
                const float4 b4 = *reinterpret_cast<const float4 *>(tot + (2 * J + 1) * 128 + fc4);
                btot[J][0] = a4.x + b4.x; btot[J][1] = a4.y + b4.y; btot[J][2] = a4.z + b4.z; btot[J][3] = a4.w + b4.w;
                if (J == fb) { h0[0] = a4.x; h0[1] = a4.y; h0[2] = a4.z; h0[3] = a4.w; }
            }
            {
                const float4 c4 = *reinterpret_cast<const float4 *>(totc + 2 * fb * 128 + fc4);
                h0c[0] = c4.x; h0c[1] = c4.y; h0c[2] = c4.z; h0c[3] = c4.w;
            }
            float eS[4], eF[4], chi[4][4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sg[e] = 0.f;
                all[e] = 0.f;
#pragma unroll
                for (int J = 0; J < 4; ++J) {
                    if (J < fb) sg[e] += btot[J][e];
                    if (J == fb) bt[e] = btot[J][e];
                    all[e] += btot[J][e];
                }
                eS[e] = ex2(sg[e]);
                eF[e] = ex2(all[e] - sg[e] - bt[e]);
                float between = 0.f;  // block totals strictly between fb and I
#pragma unroll
                for (int I = 0; I < 4; ++I) {
                    chi[I][e] = ex2(between);
                    if (I > fb) between += btot[I][e];
                }
            }
            if (warp == 0) {
                *reinterpret_cast<float4 *>(sm + FAC + 4 * fc4) =
                    make_float4(ex2(all[0]), ex2(all[1]), ex2(all[2]), ex2(all[3]));  // gamma
                // the chunk-start frame: frame factor 1, marked by a negative s
                *reinterpret_cast<float4 *>(sm + FAC + 512 + 4 * fc4) = make_float4(-1.f, -1.f, -1.f, -1.f);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = 8 * warp + i;
                float qv[4], kv[4];
                ld_bf4(sm + RAW_Q + raw16(t, fc4), qv);
                ld_bf4(sm + RAW_K + raw16(t, fc4), kv);
                const float4 b4 = act_b4(ga, gld4<GB>(sm + RAW_B + graw<GB>(t, fc4)));
                const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
                float bka[4], qa[4], kc[4], qb[4], kb[4], ka[4], dd[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float loc = fh ? h0[e] + gl[i][e] : gl[i][e];  // G_t - s_I
                    const float a = ex2(loc), ab = ex2(bt[e] - loc);
                    bka[e] = bv[e] * kv[e] * a;
                    qa[e] = qv[e] * a;
                    kc[e] = bka[e] * eS[e];
                    qb[e] = qa[e] * eS[e];
                    ka[e] = kv[e] * ab;
                    kb[e] = ka[e] * eF[e];
                    dd[e] = fh ? gc[i][e] : gc[i][e] - h0c[e];  // G'_t - G'_m, m = the block's row 7
                    big = fmaxf(big, fmaxf(fabsf(bka[e]), fmaxf(fabsf(qa[e]), fabsf(ka[e]))));
                }
                st_h4v(sm + CO + sw128_off(t, fc4, 128), bka);
                st_h4v(sm + CO + sw128_off(64 + t, fc4, 128), qa);
                st_h4v(sm + OP_WQ + sw128_off(t, fc4, 128), kc);
                st_h4v(sm + OP_WQ + sw128_off(64 + t, fc4, 128), qb);
                st_h4v(sm + OP_KB + sw128_off(t, fc4, 64), kb);
#pragma unroll
                for (int I = 1; I < 4; ++I)
                    if (I > fb) {
                        const float kx[4] = {ka[0] * chi[I][0], ka[1] * chi[I][1], ka[2] * chi[I][2], ka[3] * chi[I][3]};
                        st_h4v(sm + RR + rr_off(I) + sw128_off(t, fc4, 16 * I), kx);
                    }
                *reinterpret_cast<float4 *>(sm + RAW_G + raw32(t, fc4)) = make_float4(dd[0], dd[1], dd[2], dd[3]);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        store_early(rec);
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
        // ---------------- diagonal blocks: warp (block db, 8 columns dn) in tf32.
        // The contraction runs over channels in the order that lets a lane
        // load 4 consecutive channels at once: k-step 2p takes channels
        // 16p + 4t, 16p + 4t + 1 as k = t, t + 4; k-step 2p + 1 takes
        // 16p + 4t + 2, + 3.
        {
            const int r0 = 16 * db + gq, r1 = r0 + 8, jj = 16 * db + 8 * dn + gq;
#pragma unroll 2
            for (int p = 0; p < 8; ++p) {
                const int c = 16 * p + 4 * tq;
                uint32_t aA[2][4], aP[2][4], bb[4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // rows r0, r1
                    const int r = h ? r1 : r0;
                    const float4 d4 = *reinterpret_cast<const float4 *>(sm + RAW_G + raw32(r, c));
                    const float4 b4 = act_b4(ga, gld4<GB>(sm + RAW_B + graw<GB>(r, c)));
                    float qv[4], kv[4];
                    ld_bf4(sm + RAW_Q + raw16(r, c), qv);
                    ld_bf4(sm + RAW_K + raw16(r, c), kv);
                    const float lv[4] = {ex2(d4.x), ex2(d4.y), ex2(d4.z), ex2(d4.w)};
                    const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // channel c + e: k-step 2p + (e >> 1), k index t (+4 when e odd)
                        aA[e >> 1][h + 2 * (e & 1)] = to_tf32(bv[e] * kv[e] * lv[e]);
                        aP[e >> 1][h + 2 * (e & 1)] = to_tf32(qv[e] * lv[e]);
                    }
                }
                {
                    const float4 d4 = *reinterpret_cast<const float4 *>(sm + RAW_G + raw32(jj, c));
                    float kv[4];
                    ld_bf4(sm + RAW_K + raw16(jj, c), kv);
                    bb[0] = to_tf32(kv[0] * ex2(-d4.x));
                    bb[1] = to_tf32(kv[1] * ex2(-d4.y));
                    bb[2] = to_tf32(kv[2] * ex2(-d4.z));
                    bb[3] = to_tf32(kv[3] * ex2(-d4.w));
                }
                mma_tf32_16x8x8(cA, aA[0], bb);
                mma_tf32_16x8x8(cP, aP[0], bb);
                mma_tf32_16x8x8(cA, aA[1], bb + 2);
                mma_tf32_16x8x8(cP, aP[1], bb + 2);
            }
        }
        }  // !mild
        // ---------------- assemble A (float32, for the inversion) and P (record)
        ok = mbar_wait(&bars[1], 0, kWait);
        fence_after_sync();
        __syncthreads();  // the block products have read CO / RR; the raw tiles are consumed
        float *sA = reinterpret_cast<float *>(sm + SCR_A);
        float *sT = reinterpret_cast<float *>(sm + SCR_T);
        if (mild) {
            // accumulator row quarter * 32 + lane: rows 0..63 are A, 64..127 are P;
            // this warp's 32 columns start at 32 * (warp >> 2)
            const int half = warp >> 2;
            float row[32];
            tmem_ld16(taddr(tm + TM_C, quarter * 32, 32 * half), row);
            tmem_ld16(taddr(tm + TM_C, quarter * 32, 32 * half + 16), row + 16);
            tmem_wait_ld();
            if (quarter < 2) {
                const int r = quarter * 32 + lane;
#pragma unroll
                for (int j = 0; j < 32; ++j) row[j] = 32 * half + j < r ? row[j] : 0.f;
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4)
                    *reinterpret_cast<float4 *>(sA + r * kSA + 32 * half + 4 * j4) =
                        make_float4(row[4 * j4], row[4 * j4 + 1], row[4 * j4 + 2], row[4 * j4 + 3]);
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
        } else {
            // diagonal blocks from the warps' fragments: rows 16 db + gq (+ 8),
            // columns 16 db + 8 dn + 2 tq (+ 1)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int rl = gq + ((e & 2) ? 8 : 0), jl = 8 * dn + 2 * tq + (e & 1);
                const int r = 16 * db + rl, j = 16 * db + jl;
                sA[r * kSA + j] = jl < rl ? cA[e] : 0.f;
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
                            for (int j4 = 0; j4 < 4; ++j4)
                                *reinterpret_cast<float4 *>(sA + row * kSA + c0 + 4 * j4) =
                                    make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
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
        if (tid == 64) {  // P and the factors are final
            fence_after_sync();
            store_piece(rec, REC_P, 8192);
            store_piece(rec, REC_FAC, REC_BYTES - REC_FAC);
            bulk_commit();
        }
        // ---------------- T = (I + A)^-1, into the record as fp16
        // the raw tiles are consumed: the next tile's are requested by a warp
        // that is idle during the inversion's block columns
        const bool has_next = it + (int)gridDim.x < ntiles;
        big = invert_unit_lower(sA, sT, reinterpret_cast<float *>(sm + SCR_M), sm + OP_T, tid, big, [&] {
            if (has_next) load_raw(it + gridDim.x);
        });
        issued += has_next;
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 64) {
            fence_after_sync();
            store_piece(rec, REC_T, 8192);
            bulk_commit();
        }
        if (tid == 0) {
            fence_after_sync();
            // Kc (rows 0..63 of the [Kc; Qb] tile) as the MN-major B: its two
            // 64-key blocks lie 16 KB apart
            // [T; P] (the record's T and P tiles follow each other) as one M = 128
            // A operand, so that W lands one row per tensor-memory lane; P Kc in
            // lanes 64..127 is not read
            const uint64_t t = desc_kmajor(smem_addr(sm + OP_T), 128, 0),
                           kc = desc_mnmajor_lbo(smem_addr(sm + OP_WQ), 16384, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_W, kstep_kmajor(t, 128, ks), kstep_mnmajor(kc, ks), ID_WP128, ks > 0);
            mma_commit(&bars[1]);
        }
        // ---------------- -W to fp16 (over Kc, consumed by the product); the record
        if (it + (int)gridDim.x < ntiles) L_next = rows_of(it + gridDim.x);  // while W runs
        ok = mbar_wait(&bars[1], 1, kWait);
        fence_after_sync();
        if (quarter < 2) {  // lanes 0..63: row 32 quarter + lane, 64 columns from 64 half
            float wv[64];
            const int half = warp >> 2, r = quarter * 32 + lane;
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(taddr(tm + TM_W, quarter * 32, 64 * half + 16 * j), wv + 16 * j);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 64; ++j) wv[j] = -wv[j];
#pragma unroll
            for (int j2 = 0; j2 < 8; ++j2) {
                st_h8(sm + OP_WQ + sw128_chunk(r, 8 * half + j2, 128), wv + 8 * j2);
                big = absmax8(wv + 8 * j2, big);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 64) {  // -W: rows 0..63 of both 64-key blocks
            fence_after_sync();
            store_piece(rec, REC_WQ, 8192);
            store_piece(rec, REC_WQ + 16384, 8192);
            bulk_commit();
        }
    }
    if (!(big <= kRange)) record_status(status, GDN2_ERR_RANGE);
    if (tid == 64) bulk_wait_all();
    if (tid == 0) {
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

template <bool GB, bool ACT>
static cudaError_t tc_prep_run(const void *q, const void *k, const void *g, const void *b, void *ws,
                               unsigned int *status, const Dims &d, cudaStream_t s) {
    CUtensorMap mq, mk, mg, mb;
    if (!make_wide_map(&mq, q, true, d.B, d.T, d.H, 128, 64) || !make_wide_map(&mk, k, true, d.B, d.T, d.H, 128, 64) ||
        !make_wide_map(&mg, g, GB, d.B, d.T, d.H, 128, 64) || !make_wide_map(&mb, b, GB, d.B, d.T, d.H, 128, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tc_prep_kernel<GB, ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tprep::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // (packed sequences: NC bounds the total chunks; the kernel reads the count)
    const long long ntiles = (long long)d.B * d.H * d.NC;
    const int grid = (int)(ntiles < sm_count() ? ntiles : sm_count());
    launch_begin(K_TC_PREP, s);
    tc_prep_kernel<GB, ACT><<<grid, tprep::kThreads, tprep::SMEM_BYTES, s>>>(
        mq, mk, mg, mb, (unsigned char *)ws, tc_ws_layout(d), status, d);
    launch_end(K_TC_PREP, s);
    return cudaGetLastError();
}

cudaError_t tc_prep_launch(const void *q, const void *k, const void *g, const void *b, void *ws,
                           unsigned int *status, const Dims &d, cudaStream_t s) {
    if (d.act) return d.gb ? tc_prep_run<true, true>(q, k, g, b, ws, status, d, s)
                           : tc_prep_run<false, true>(q, k, g, b, ws, status, d, s);
    return d.gb ? tc_prep_run<true, false>(q, k, g, b, ws, status, d, s)
                : tc_prep_run<false, false>(q, k, g, b, ws, status, d, s);
}

}  // namespace gdn2
