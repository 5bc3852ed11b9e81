// Chunk-parallel part of the gate-aware backward of Gated Delta Rule-2 on
// the sm_100a tensor cores (bf16 I/O, d_k = d_v = 128, chunk 64): dq, dk, db
// and dg of every chunk from its record, its entry state S_c, Delta, -dU and
// the state gradient dS' leaving it (all left in the workspace by the forward
// and by the state kernel of tc_bwd.cu).
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B, D.6; digg thread 11/): the per-channel gates cannot be pulled
// out of the products that accumulate the gradient of the strictly-lower A,
// so they stay inside them: b enters dA and dKc through Kc in every channel
// sum below.
//
// Chunk equations (chunk-start frame, tc_common.cuh; E = e^G,
// F = e^(G_63 - G)):
//   dP = lower-incl(dO Delta^T),        dA = -strictly-lower(dU Delta^T)
//   Y1 = dO S_c^T,  Y2 = -dU S_c^T,  Y3 = Delta dS'^T        (state parts)
//   Z1_r = sum_j dP_rj k_j e^(G_r - G_j),   Z2_r = sum_j dA_rj k_j e^(G_r - G_j)
//   Z3_j = sum_r (dP_rj q_r + dA_rj b_r k_r) e^(G_r - G_j)   (pair parts)
//   dq = Y1 E + Z1,   dKc = Y2 E + Z2,   dk = Y3 F + Z3 + dKc b,   db = dKc k
//   dG = q dq + 2 b k dKc - k dk, plus on the last row the chunk-end term
//        rowsum(dS' . S_{c+1}) = gamma rowsum(dS' . S_c) + sum_t Kb_t Y3_t
//   dg = reverse in-chunk cumsum of dG
// (the chunk-end term is the derivative through the chunk's total decay,
// since S_{c+1} = diag(e^G_63) S_c + Kb^T Delta).

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

namespace tbg {
constexpr int kCompute = 512;             // warps 0..15 form operands and outputs
constexpr int kThreads = kCompute;        // thread 0 also issues the copies and products
constexpr int kWarps = kCompute / 32;
// raw tiles (128-B swizzled TMA boxes, tc_common.cuh raw16 / raw32); the
// outputs are formed in place
constexpr uint32_t RQ = 0;        // q (bf16), then dq
constexpr uint32_t RK = 16384;    // k (bf16), then dk
constexpr uint32_t RB = 32768;    // b (f32), then db
constexpr uint32_t RG = 65536;    // g (f32), then d = G' - G'_m, then dG, then dg
// operands of the tensor-core products
constexpr uint32_t DN = 98304;    // [dO; -dU] [128][128] K-major (K-blocks of 16 KB)
constexpr uint32_t DL = 131072;   // Delta [64 pos][128 v] K-major
constexpr uint32_t SMT = 147456;  // S_c [128 key][128 v] K-major
constexpr uint32_t DXT = 180224;  // dS' [128 key][128 v] K-major
// once the products have read them, the same 112 KB hold the pair-term data
// ([64 rows][128 channels] fp16 tiles, swizzled as raw16)
constexpr uint32_t KA = 98304;    // k e^(e_I - G)
constexpr uint32_t QA = 114688;   // q e^(G - s_I)
constexpr uint32_t BA = 131072;   // b k e^(G - s_I)
constexpr uint32_t AL = 147456;   // e^(G - s_I)
constexpr uint32_t AB = 163840;   // e^(e_I - G)
// mild tiles (E = e^(G - G_31)): E and 1 / E in place of g once the cumulative
// decay has read it; q E, b k E and k / E, the second products' operands, over
// Delta and S_c, so that [dO; -dU] is free once the first products have read
// it and Delta, S_c, dS' once the second products have
constexpr uint32_t MEM = RG, MEI = RG + 16384, MQB = DL, MKC = SMT, MKH = SMT + 16384;
constexpr uint32_t PD = 180224;   // masked dP [64][64] fp16 (sw128, R = 64)
constexpr uint32_t AD = 188416;   // masked dA
constexpr uint32_t DG32 = 196608; // diagonal blocks of dP, dA as tf32 bits [2][4][16][17]
constexpr uint32_t ESF = 205824;  // e^s_I and e^(G_63 - e_I) per block and channel [2][4][128] f32
constexpr uint32_t MISC = 212992; // per-channel values (below), mbarriers, TMEM slot
// 8-row totals of G and of the clamped G [2][8][128]; chi [6][128]; the
// chunk-end parts [4][128] twice; gamma [128]
constexpr uint32_t M_TOT = 0, M_CHI = 8192, M_END1 = 11264, M_ENDK = 13312, M_GAM = 15360,
                   M_FLAG = 15872, M_BAR = 15936;
constexpr uint32_t SMEM_BYTES = MISC + M_BAR + 128 + 1024;
constexpr uint32_t LOAD_A = 32768 + 81920;  // dO, -dU; Delta, S_c, dS'
constexpr uint32_t TM_Y1 = 0, TM_Y2 = 128, TM_Y3 = 256, TM_PA = 384;  // 512 columns
constexpr uint32_t ID_PA = idesc_f16(128, 64, false, false);
constexpr uint32_t ID_KK128 = idesc_f16(64, 128, false, false);
constexpr uint32_t ID_KM128 = idesc_f16(64, 128, false, true);
constexpr uint32_t ID_MM128 = idesc_f16(64, 128, true, true);
constexpr long long kWait = 2000000000LL;
constexpr float kRange = 6.0e4f;
static_assert(DG32 + 2 * 4 * 16 * 17 * 4 <= ESF && ESF + 4096 <= MISC, "pair-term data fits over the operands");
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace tbg

// descriptor of K step kstep of a K-major operand whose 64-wide K-blocks lie
// blk bytes apart (d0 = its K step 0)
__device__ __forceinline__ uint64_t kstep_kmajor_blk(uint64_t d0, uint32_t blk, int kstep) {
    return d0 + (uint64_t)((((uint32_t)(kstep >> 2) * blk) + (kstep & 3) * 32) >> 4);
}

// 16 TMEM lanes x 8 columns in the m16n8 accumulator-fragment layout: rows
// base + t/4 (v0, v1) and base + t/4 + 8 (v2, v3), columns c + 2 (t % 4), + 1
__device__ __forceinline__ void tmem_ld16x256x1(uint32_t taddr, float *v) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

// index of the block pair (I, J), I > J, among the six
__host__ __device__ constexpr int pair_ix(int I, int J) { return I * (I - 1) / 2 + J; }

// Persistent: one CTA per SM walks the (b, h, chunk) tiles, full d_v.  Thread
// 0 also loads the tile (raw q, k, b, g, dO as 128-B swizzled TMA boxes; S_c,
// dS', Delta, -dU from the workspace) and issues the tensor-core products (16
// warps leave 128 registers per thread); warp w owns row block I = w % 4 (16
// rows, TMEM lane quarter I) and channel quarter Q = w / 4 (32 channels):
//   (1) [dP; dA] = [dO; -dU] Delta^T (M = 128), Y1 = dO S_c^T, Y2 = -dU S_c^T,
//       Y3 = Delta dS'^T on the tensor cores, while the warps form the
//       cumulative decay and the block factors;
//   (2) the chunk-end sum rowsum(dS' . S_c) and the masked dP, dA;
//   (3) the pair terms Z1, Z2, Z3 as warp-level products: blocks below the
//       diagonal in fp16 (m16n8k16) with the block-boundary frames, the
//       diagonal blocks in tf32 (m16n8k8) with the clamped mid-block frame;
//   (4) dq, dk, db, dG per (row, channel) in the accumulator-fragment layout,
//       which the 16x256b tensor-memory loads share, written in place of q,
//       k, b, g, and dq, dk, db leave by TMA stores; then dg, the reverse
//       in-chunk cumsum of dG plus the chunk-end term, straight from the scan
//       to global memory.
template <bool GB, bool ACT>  // g, b, dg, db as bf16 (else float32); ACT: gate logits (GateAct)
__global__ void __launch_bounds__(tbg::kThreads, 1)
tc_bwd_grad_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mb, const __grid_constant__ CUtensorMap mg,
                   const __grid_constant__ CUtensorMap mdo, const __grid_constant__ CUtensorMap mdq,
                   const __grid_constant__ CUtensorMap mdk, const __grid_constant__ CUtensorMap mdb,
                   const void *__restrict__ g_in, void *__restrict__ dq_out,
                   void *__restrict__ dk_out, void *__restrict__ db_out, void *__restrict__ dg_out,
                   unsigned char *__restrict__ ws, TcWs lay, unsigned int *status, Dims d) {
    using namespace tbg;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *mtot = reinterpret_cast<float *>(sm + MISC + M_TOT);    // [8][128] 8-row totals (log2 units)
    float *mtotc = mtot + 8 * 128;                                 // [8][128] the same, clamped
    float *mchi = reinterpret_cast<float *>(sm + MISC + M_CHI);    // [6][128] chi_IJ
    float *mend1 = reinterpret_cast<float *>(sm + MISC + M_END1);  // [4][128] rowsum(dS' . S_c) parts
    float *mendk = reinterpret_cast<float *>(sm + MISC + M_ENDK);  // [4][128] sum_t Kb Y3 parts
    float *mgam = reinterpret_cast<float *>(sm + MISC + M_GAM);    // [128] gamma
    float *mes = reinterpret_cast<float *>(sm + ESF);              // [4][128] e^s_I (after the first products)
    float *mef = mes + 4 * 128;                                    // [4][128] e^(G_63 - e_I)
    // 0 first-product operands (two parts), 1 products, 2 second products
    // (mild), 3 raw g, 4 raw q, k, b
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC + M_BAR);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + M_BAR + 64);
    float big = 0.f;  // range check: largest fp16 operand magnitude

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = total_tiles(d);
    const GateAct ga = ACT ? gate_act(d.act) : GateAct{false, 1.f};  // logits in: g, b activated on load, db and dg by the chain rule
    const int I = warp & 3, Q = (warp >> 2) & 3;  // row block (TMEM lane quarter); channel quarter
    const int gq = lane >> 2, tq = lane & 3;
    const bool compute = true, issuer = tid == 0;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (issuer) {
        mbar_init(&bars[0], 2);
        for (int i = 1; i < 4; ++i) mbar_init(&bars[i], 1);
        mbar_init(&bars[4], 1);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    // tile `it` in (sequence, head, chunk) order (tile_decode); copies requested by the issuer
    int issued[3] = {0, 0, 0};  // operand parts 1, 2 and raw tiles
    // the tile's head, first row and batch row
    auto tile_rows = [&](int it, int &h, int &row0, int &bb) {
        int n, c;
        tile_decode(d, it, n, h, c);
        const Seq sq = seq_of(d, n);
        row0 = sq.bos + 64 * c;
        bb = sq.brow;
    };
    auto load_a1 = [&](int it) {  // dO (TMA) and -dU: [dO; -dU]
        int h, row0, bb;
        tile_rows(it, h, row0, bb);
        mbar_expect_tx(&bars[0], 32768);
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(sm + DN + x * 16384, &mdo, 64 * x, h, row0, bb, &bars[0]);
            bulk_load(sm + DN + x * 16384 + 8192, ws + lay.ckndU + ((size_t)it * 2 + x) * 8192, 8192, &bars[0]);
        }
        ++issued[0];
    };
    auto load_a2 = [&](int it) {  // Delta, S_c, dS'; the chunk's frame factor (4 channels)
        mbar_expect_tx(&bars[0], LOAD_A - 32768 + 16);
        bulk_load(sm + MISC + M_FLAG, ws + lay.rec + (size_t)it * REC_BYTES + REC_FAC + 512, 16, &bars[0]);
        bulk_load(sm + DL, ws + lay.ckD + ((size_t)it * 2) * 8192, 16384, &bars[0]);
        bulk_load(sm + SMT, ws + lay.ckS + ((size_t)it * 2) * 16384, 32768, &bars[0]);
        bulk_load(sm + DXT, ws + lay.ckdS + ((size_t)it * 2) * 16384, 32768, &bars[0]);
        ++issued[1];
    };
    // raw q, k, b, g in two parts on two barriers: g (bars[3]) as soon as the
    // scan has read dG out of its tile, then q, k, b (bars[4]) once dq, dk, db
    // have left theirs
    int pend_b = -1;  // tile whose g has been requested but not its q, k, b
    auto load_b_g = [&](int it) {
        int h, row0, bb;
        tile_rows(it, h, row0, bb);
        mbar_expect_tx(&bars[3], gate_tile_bytes<GB>());
        tma_load_5d(sm + RG, &mg, 0, h, row0, 0, bb, &bars[3]);
        ++issued[2];
        pend_b = it;
    };
    auto load_b_rest = [&](int it) {
        int h, row0, bb;
        tile_rows(it, h, row0, bb);
        mbar_expect_tx(&bars[4], 32768 + gate_tile_bytes<GB>());
        tma_load_5d(sm + RQ, &mq, 0, h, row0, 0, bb, &bars[4]);
        tma_load_5d(sm + RK, &mk, 0, h, row0, 0, bb, &bars[4]);
        tma_load_5d(sm + RB, &mb, 0, h, row0, 0, bb, &bars[4]);
        pend_b = -1;
    };
    if (issuer && (int)blockIdx.x < ntiles) {
        load_a1(blockIdx.x);
        load_a2(blockIdx.x);
        load_b_g(blockIdx.x);
        load_b_rest(blockIdx.x);
    }

    bool ok = true, aborted = false;  // aborted: some thread's wait gave up (block-wide)
    int nmild = 0;  // mild tiles done (second product groups committed to bars[2])
    for (int it = blockIdx.x, n = 0; it < ntiles; it += gridDim.x, ++n) {
        int tn, h, c;
        tile_decode(d, it, tn, h, c);
        const Seq sq = seq_of(d, tn);
        const int c0 = sq.bos + 64 * c, bb = sq.brow;
        // a packed sequence's tail chunk: rows L..63 hold the next sequence's tokens
        const int L = sq.len - 64 * c;
        const bool tail = d.cu != nullptr && L < 64;
        const uint32_t par = n & 1;
        const int nxt = it + (int)gridDim.x;
        const bool more = nxt < ntiles;
        ok = mbar_wait(&bars[0], par, kWait) && ok;

        // ---------------- dO to fp16, in place in the dO rows of [dO; -dU]
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int i = tid + kCompute * m;
            unsigned char *p = sm + DN + (i >> 9) * 16384 + (i & 511) * 16;
            uint4 raw = *reinterpret_cast<const uint4 *>(p);
            if (((i & 511) >> 3) >= L) raw = make_uint4(0u, 0u, 0u, 0u);  // rows past the sequence's end
            const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
            float x[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[2 * e] = __low2float(b2[e]);
                x[2 * e + 1] = __high2float(b2[e]);
            }
            st_h8(p, x);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();  // dO converted
        if (issuer) {
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
        ok = mbar_wait(&bars[3], par, kWait) && ok;  // raw g
        if (tail) {
            ok = mbar_wait(&bars[4], par, kWait) && ok;  // raw q, k, b
            zero_rows(sm + RQ, 12, L, tid, kThreads);  // q, k, b, g: 96 KB of 8 KB boxes
            __syncthreads();
        }
        // ---------------- cumulative decay (log2 units): warp w = rows 8 (w & 7)
        // .. + 7 (block fb, half fh), channels fc, fc + 1 with fc = 64 (w >> 3) + 2 lane
        const int frg = warp & 7, fb = frg >> 1, fh = frg & 1, fc = 64 * ((warp >> 3) & 1) + 2 * lane;
        float gl[8][2], gc[8][2];
        {
            float run[2] = {0.f, 0.f}, runc[2] = {0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // past the end, no decay (a zero logit would activate to log 1/2)
                const float2 g2 = 8 * frg + i < L ? act_g2(ga, gld2<GB>(sm + RG + graw<GB>(8 * frg + i, fc)))
                                                  : make_float2(0.f, 0.f);
                const float gv[2] = {g2.x * kLog2e, g2.y * kLog2e};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    run[e] += gv[e];
                    runc[e] += fmaxf(gv[e], -kClampG2);
                    gl[i][e] = run[e];
                    gc[i][e] = runc[e];
                }
            }
            *reinterpret_cast<float2 *>(mtot + frg * 128 + fc) = make_float2(run[0], run[1]);
            *reinterpret_cast<float2 *>(mtotc + frg * 128 + fc) = make_float2(runc[0], runc[1]);
        }
        named_sync(1, kCompute);
        float btot[4][2], h0[2], h0c[2], sg[2], bt[2], all[2], pre[2] = {0.f, 0.f}, g31[2];
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            const float2 a2 = *reinterpret_cast<const float2 *>(mtot + (2 * J) * 128 + fc);
            const float2 b2 = *reinterpret_cast<const float2 *>(mtot + (2 * J + 1) * 128 + fc);
            btot[J][0] = a2.x + b2.x;
            btot[J][1] = a2.y + b2.y;
            if (J == fb) { h0[0] = a2.x; h0[1] = a2.y; }
            if (2 * J < frg) { pre[0] += a2.x; pre[1] += a2.y; }
            if (2 * J + 1 < frg) { pre[0] += b2.x; pre[1] += b2.y; }
        }
        {
            const float2 c2 = *reinterpret_cast<const float2 *>(mtotc + 2 * fb * 128 + fc);
            h0c[0] = c2.x;
            h0c[1] = c2.y;
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            sg[e] = 0.f;
            all[e] = 0.f;
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                if (J < fb) sg[e] += btot[J][e];
                if (J == fb) bt[e] = btot[J][e];
                all[e] += btot[J][e];
            }
            g31[e] = btot[0][e] + btot[1][e];
        }
        // ---------------- the frame of the chunk's record: mild (row 31, with S_c and
        // dS' in the workspace as e^G_31 S_c and e^(G_63 - G_31) dS') or the
        // chunk-start frame (a negative frame factor)
        const bool mild = reinterpret_cast<const float *>(sm + MISC + M_FLAG)[0] > 0.f;
        // ---------------- factors, held until the products have read S_c and dS':
        // mild: q E, b k E, k / E, E, 1 / E (E = e^(G - G_31));
        // else: k a_bar, q a, b k a, a, a_bar, and d = G' - G'_m in place of g
        uint32_t pk[8][5];
        if (!mild) {
            float chi[4][2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float between = 0.f;  // block totals strictly between fb and I
#pragma unroll
                for (int I2 = 0; I2 < 4; ++I2) {
                    chi[I2][e] = ex2(between);
                    if (I2 > fb) between += btot[I2][e];
                }
            }
            if (fh == 0) {
#pragma unroll
                for (int I2 = 1; I2 < 4; ++I2)
                    if (I2 > fb + 1)
                        *reinterpret_cast<float2 *>(mchi + pair_ix(I2, fb) * 128 + fc) = make_float2(chi[I2][0], chi[I2][1]);
            }
        }
        if (fh == 0 && fb == 0) *reinterpret_cast<float2 *>(mgam + fc) = make_float2(ex2(all[0]), ex2(all[1]));
        if (!tail) ok = mbar_wait(&bars[4], par, kWait) && ok;  // raw q, k, b
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * frg + i;
            const float2 q2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + RQ + raw16(t, fc)));
            const float2 k2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + RK + raw16(t, fc)));
            const float2 b2 = act_b2(ga, gld2<GB>(sm + RB + graw<GB>(t, fc)));
            const float qv[2] = {q2.x, q2.y}, kv[2] = {k2.x, k2.y}, bv[2] = {b2.x, b2.y};
            float v[5][2], dd[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                if (mild) {
                    const float dl = pre[e] + gl[i][e] - g31[e];
                    const float E = ex2(dl), Ei = ex2(-dl);
                    v[0][e] = qv[e] * E;
                    v[1][e] = bv[e] * kv[e] * E;
                    v[2][e] = kv[e] * Ei;
                    v[3][e] = E;
                    v[4][e] = Ei;
                } else {
                    const float loc = fh ? h0[e] + gl[i][e] : gl[i][e];  // G_t - s_I
                    const float a = ex2(loc), ab = ex2(bt[e] - loc);
                    v[0][e] = kv[e] * ab;
                    v[1][e] = qv[e] * a;
                    v[2][e] = bv[e] * kv[e] * a;
                    v[3][e] = a;
                    v[4][e] = ab;
                    dd[e] = fh ? gc[i][e] : gc[i][e] - h0c[e];  // G'_t - G'_m, m = the block's row 7
                }
                // a mild tile's factors are within 256 e^4 by its test (tc_common.cuh)
                if (!mild) big = fmaxf(big, fmaxf(fabsf(v[0][e]), fmaxf(fabsf(v[1][e]), fabsf(v[2][e]))));
            }
#pragma unroll
            for (int x = 0; x < 5; ++x) pk[i][x] = pack_f16(v[x][0], v[x][1]);
            if (mild) {  // E, 1 / E over g, which the cumulative decay has read
                *reinterpret_cast<uint32_t *>(sm + MEM + raw16(t, fc)) = pk[i][3];
                *reinterpret_cast<uint32_t *>(sm + MEI + raw16(t, fc)) = pk[i][4];
            } else {
                *reinterpret_cast<float2 *>(sm + RG + raw32(t, fc)) = make_float2(dd[0], dd[1]);
            }
        }
        // ---------------- chunk-end sum, once the products have read S_c and dS'
        ok = mbar_wait(&bars[1], par, kWait) && ok;
        fence_after_sync();
        {
            // channel 32 (warp >> 2) + lane, d_v quarter warp & 3: 32 values of S_c
            // and dS' (mild: of S_m and dX, whose product carries gamma already)
            const int ec = 32 * ((warp >> 2) & 3) + lane, ev = warp & 3;
            float acc = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const uint32_t off = (uint32_t)((ev >> 1) * 16384) + sw128_chunk(ec, 4 * (ev & 1) + jj, 128);
                float s8[8], d8[8];
                ld_h8(sm + SMT + off, s8);
                ld_h8(sm + DXT + off, d8);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc = fmaf(s8[e], d8[e], acc);
            }
            mend1[ev * 128 + ec] = acc;
        }
        named_sync(1, kCompute);  // S_c, dS', Delta, [dO; -dU] are consumed
        if (issuer && mild && more) load_a1(nxt);  // the mild tiles leave [dO; -dU] free
        if (!mild && fh == 0) {
            *reinterpret_cast<float2 *>(mes + fb * 128 + fc) = make_float2(ex2(sg[0]), ex2(sg[1]));
            *reinterpret_cast<float2 *>(mef + fb * 128 + fc) =
                make_float2(ex2(all[0] - sg[0] - bt[0]), ex2(all[1] - sg[1] - bt[1]));
        }
        // ---------------- masked dP, dA (TMEM lanes 0..63 dP, 64..127 dA)
        {
            float row[16];
            tmem_ld16(taddr(tm + TM_PA, I * 32, 16 * Q), row);
            tmem_wait_ld();
            const int pr = I * 32 + lane, r = pr & 63;
            const bool isA = pr >= 64;
#pragma unroll
            for (int j = 0; j < 16; ++j) row[j] = (isA ? 16 * Q + j < r : 16 * Q + j <= r) ? row[j] : 0.f;
            unsigned char *dst = sm + (isA ? AD : PD);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                st_h8(dst + sw128_chunk(r, 2 * Q + jj, 64), row + 8 * jj);
                big = absmax8(row + 8 * jj, big);
            }
            if (!mild && (r >> 4) == Q) {
                uint32_t *dg32 = reinterpret_cast<uint32_t *>(sm + DG32) + ((isA ? 4 : 0) + Q) * 16 * 17 + (r & 15) * 17;
#pragma unroll
                for (int j = 0; j < 16; ++j) dg32[j] = to_tf32(row[j]);
            }
        }
        // ---------------- the factors as fp16 tiles
        if (mild) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t off = raw16(8 * frg + i, fc);
                *reinterpret_cast<uint32_t *>(sm + MQB + off) = pk[i][0];
                *reinterpret_cast<uint32_t *>(sm + MKC + off) = pk[i][1];
                *reinterpret_cast<uint32_t *>(sm + MKH + off) = pk[i][2];
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t off = raw16(8 * frg + i, fc);
#pragma unroll
                for (int x = 0; x < 5; ++x) *reinterpret_cast<uint32_t *>(sm + KA + x * 16384 + off) = pk[i][x];
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();  // dP, dA and the factor tiles are in place
        if (mild) {
            fence_after_sync();
            if (issuer) {  // Y1 += dP Kh, Y2 += dA Kh: Y3 stays as it is for the chunk-end term
                const uint64_t kP = desc_kmajor(smem_addr(sm + PD), 64, 0), kA = desc_kmajor(smem_addr(sm + AD), 64, 0),
                               kh_d = desc_mnmajor(smem_addr(sm + MKH), 64, 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t b_kh = kstep_mnmajor(kh_d, ks);
                    mma_bf16(tm + TM_Y1, kstep_kmajor(kP, 64, ks), b_kh, ID_KM128, 1);
                    mma_bf16(tm + TM_Y2, kstep_kmajor(kA, 64, ks), b_kh, ID_KM128, 1);
                }
            }
            // ---------------- Kb^T Delta's share of the chunk-end term: sum_t Kh_m Y3
            // with Y3 = Delta dX^T before the second products add to it
            const int r0 = 16 * I + gq;
            float y3a[16];  // the four 8-column groups of this warp's 32 channels
            tmem_ld16x256x4(taddr(tm + TM_Y3 + 32 * Q, I * 32, 0), y3a);
            tmem_wait_ld();
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int cc = 32 * Q + 8 * nt + 2 * tq;
                const float *y3 = y3a + 4 * nt;
                float part[2] = {0.f, 0.f};
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const float2 kh = __half22float2(*reinterpret_cast<const __half2 *>(sm + MKH + raw16(r0 + 8 * h2, cc)));
                    part[0] = fmaf(kh.x, y3[2 * h2], part[0]);
                    part[1] = fmaf(kh.y, y3[2 * h2 + 1], part[1]);
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = part[e];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (gq == 0) mendk[I * 128 + cc + e] = v;
                }
            }
            fence_before_sync();
            __syncthreads();  // Y3 has been read
            if (issuer) {
                fence_after_sync();
                const uint64_t mP = desc_mnmajor(smem_addr(sm + PD), 64, 0), mA = desc_mnmajor(smem_addr(sm + AD), 64, 0),
                               qb = desc_mnmajor(smem_addr(sm + MQB), 64, 0), kc = desc_mnmajor(smem_addr(sm + MKC), 64, 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    mma_bf16(tm + TM_Y3, kstep_mnmajor(mP, ks), kstep_mnmajor(qb, ks), ID_MM128, 1);
                    mma_bf16(tm + TM_Y3, kstep_mnmajor(mA, ks), kstep_mnmajor(kc, ks), ID_MM128, 1);
                }
                mma_commit(&bars[2]);
            }
            ok = mbar_wait(&bars[2], nmild & 1, kWait) && ok;
            ++nmild;
            fence_after_sync();
            // Delta, S_c, dS' and the second products' operands over them are consumed
            if (issuer && more) load_a2(nxt);
        }
        float mdG[4][4];  // mild tiles: dG of rows r0, r0 + 8 and channels 32 Q + 8 nt + 2 t, + 1
        if (!mild) {
            const uint32_t spd = smem_addr(sm + PD), sad = smem_addr(sm + AD);
            const uint32_t *dgP = reinterpret_cast<const uint32_t *>(sm + DG32) + I * 16 * 17;
            const uint32_t *dgA = dgP + 4 * 16 * 17;
            const int r0 = 16 * I + gq;  // this thread's fragment rows r0, r0 + 8
            // per 8-channel n-tile: the pair terms Z1, Z2 (rows of block I), Z3
            // (rows of block I as columns), then the outputs of those 8 channels
#pragma unroll 1
            for (int nt = 0; nt < 4; ++nt) {
                const int cb = 32 * Q + 8 * nt;  // the n-tile's first channel
                float c1[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f}, c3[4] = {0.f, 0.f, 0.f, 0.f};
                // blocks below the diagonal, fp16
                for (int J = 0; J < I; ++J) {
                    uint32_t aP[4], aA[4], bk[2];
                    const int ar = 16 * I + (lane & 7) + 8 * ((lane >> 3) & 1), ac = 16 * J + 8 * (lane >> 4);
                    ldsm_x4(aP, spd + sw128_off(ar, ac, 64));
                    ldsm_x4(aA, sad + sw128_off(ar, ac, 64));
                    ldsm_x2_t(bk, smem_addr(sm + KA + raw16(16 * J + (lane & 7) + 8 * ((lane >> 3) & 1), cb)));
                    if (J + 1 < I) {
                        const float chi = mchi[pair_ix(I, J) * 128 + cb + gq];
                        bk[0] = h2scale(bk[0], chi);
                        bk[1] = h2scale(bk[1], chi);
                    }
                    mma_f16_16x8x16(c1, aP, bk);
                    mma_f16_16x8x16(c2, aA, bk);
                }
                for (int I2 = I + 1; I2 < 4; ++I2) {
                    uint32_t aP[4], aA[4], bq[2], bb2[2];
                    const int sr = 16 * I2 + (lane & 7) + 8 * (lane >> 4), sc = 16 * I + 8 * ((lane >> 3) & 1);
                    ldsm_x4_t(aP, spd + sw128_off(sr, sc, 64));
                    ldsm_x4_t(aA, sad + sw128_off(sr, sc, 64));
                    const int br = 16 * I2 + (lane & 7) + 8 * ((lane >> 3) & 1);
                    ldsm_x2_t(bq, smem_addr(sm + QA + raw16(br, cb)));
                    ldsm_x2_t(bb2, smem_addr(sm + BA + raw16(br, cb)));
                    if (I2 > I + 1) {
                        const float chi = mchi[pair_ix(I2, I) * 128 + cb + gq];
                        bq[0] = h2scale(bq[0], chi);
                        bq[1] = h2scale(bq[1], chi);
                        bb2[0] = h2scale(bb2[0], chi);
                        bb2[1] = h2scale(bb2[1], chi);
                    }
                    mma_f16_16x8x16(c3, aP, bq);
                    mma_f16_16x8x16(c3, aA, bb2);
                }
                // diagonal block in tf32: B operands k / l (Z1, Z2), q l and b k l (Z3)
                // at rows 16 I + k0 + t (+4), channel cb + g
                float d1[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f}, d3[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k0 = 0; k0 < 16; k0 += 8) {
                    uint32_t bkl[2], bql[2], bbl[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = 16 * I + k0 + tq + 4 * e, cc = cb + gq;
                        const float dv = *reinterpret_cast<const float *>(sm + RG + raw32(j, cc));
                        const float l = ex2(dv), il = ex2(-dv);
                        const float kv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + RK + raw16(j, cc)));
                        const float qv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + RQ + raw16(j, cc)));
                        const float bv = ga.b(gld1<GB>(sm + RB + graw<GB>(j, cc)));
                        bkl[e] = to_tf32(kv * il);
                        bql[e] = to_tf32(qv * l);
                        bbl[e] = to_tf32(bv * kv * l);
                    }
                    // A = dP_II, dA_II: a0 (g, t), a1 (g + 8, t), a2 (g, t + 4), a3 (g + 8, t + 4)
                    const uint32_t aP[4] = {dgP[gq * 17 + k0 + tq], dgP[(gq + 8) * 17 + k0 + tq],
                                            dgP[gq * 17 + k0 + tq + 4], dgP[(gq + 8) * 17 + k0 + tq + 4]};
                    const uint32_t aA[4] = {dgA[gq * 17 + k0 + tq], dgA[(gq + 8) * 17 + k0 + tq],
                                            dgA[gq * 17 + k0 + tq + 4], dgA[(gq + 8) * 17 + k0 + tq + 4]};
                    // their transposes (rows j, contraction over r)
                    const uint32_t aPt[4] = {dgP[(k0 + tq) * 17 + gq], dgP[(k0 + tq) * 17 + gq + 8],
                                             dgP[(k0 + tq + 4) * 17 + gq], dgP[(k0 + tq + 4) * 17 + gq + 8]};
                    const uint32_t aAt[4] = {dgA[(k0 + tq) * 17 + gq], dgA[(k0 + tq) * 17 + gq + 8],
                                             dgA[(k0 + tq + 4) * 17 + gq], dgA[(k0 + tq + 4) * 17 + gq + 8]};
                    mma_tf32_16x8x8(d1, aP, bkl);
                    mma_tf32_16x8x8(d2, aA, bkl);
                    mma_tf32_16x8x8(d3, aPt, bql);
                    mma_tf32_16x8x8(d3, aAt, bbl);
                }
                // the outputs of rows r0, r0 + 8 and channels cb + 2 t, + 1
                float y1[4], y2[4], y3[4];
                tmem_ld16x256x1(taddr(tm + TM_Y1 + cb, I * 32, 0), y1);
                tmem_ld16x256x1(taddr(tm + TM_Y2 + cb, I * 32, 0), y2);
                tmem_ld16x256x1(taddr(tm + TM_Y3 + cb, I * 32, 0), y3);
                tmem_wait_ld();
                const int cc = cb + 2 * tq;
                const float2 es = *reinterpret_cast<const float2 *>(mes + I * 128 + cc);
                const float2 ef = *reinterpret_cast<const float2 *>(mef + I * 128 + cc);
                const float esv[2] = {es.x, es.y}, efv[2] = {ef.x, ef.y};
                float endk[2] = {0.f, 0.f};
                __syncwarp();  // every read of this warp's raw region for these channels is done
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int r = r0 + 8 * h2;
                    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(sm + AL + raw16(r, cc)));
                    const float2 ab = __half22float2(*reinterpret_cast<const __half2 *>(sm + AB + raw16(r, cc)));
                    const float2 dv = *reinterpret_cast<const float2 *>(sm + RG + raw32(r, cc));
                    const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + RQ + raw16(r, cc)));
                    const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + RK + raw16(r, cc)));
                    const float2 bx = gld2<GB>(sm + RB + graw<GB>(r, cc)), bf = act_b2(ga, bx);
                    const float av[2] = {a.x, a.y}, abv[2] = {ab.x, ab.y}, dvv[2] = {dv.x, dv.y},
                                qv[2] = {qf.x, qf.y}, kv[2] = {kf.x, kf.y}, bv[2] = {bf.x, bf.y},
                                bxv[2] = {bx.x, bx.y};
                    float dq[2], dk[2], db[2], dG[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int x = 2 * h2 + e;
                        const float l = ex2(dvv[e]), il = ex2(-dvv[e]);
                        const float z1 = av[e] * c1[x] + l * d1[x];
                        const float z2 = av[e] * c2[x] + l * d2[x];
                        const float z3 = abv[e] * c3[x] + il * d3[x];
                        const float E = av[e] * esv[e], F = abv[e] * efv[e];
                        dq[e] = fmaf(y1[x], E, z1);
                        const float dkc = fmaf(y2[x], E, z2);
                        const float y3f = y3[x] * F;
                        dk[e] = y3f + z3 + dkc * bv[e];
                        db[e] = dkc * kv[e] * ga.db(bxv[e]);  // of b, or of its logit
                        dG[e] = qv[e] * dq[e] + 2.f * bv[e] * kv[e] * dkc - kv[e] * dk[e];
                        endk[e] = fmaf(kv[e], y3f, endk[e]);
                    }
                    *reinterpret_cast<uint32_t *>(sm + RQ + raw16(r, cc)) = pack_bf16(dq[0], dq[1]);
                    *reinterpret_cast<uint32_t *>(sm + RK + raw16(r, cc)) = pack_bf16(dk[0], dk[1]);
                    gst2<GB>(sm + RB + graw<GB>(r, cc), db[0], db[1]);
                    *reinterpret_cast<float2 *>(sm + RG + raw32(r, cc)) = make_float2(dG[0], dG[1]);
                }
                // sum the Kb Y3 parts over this warp's 16 rows (lanes with equal t % 4)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = endk[e];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (gq == 0) mendk[I * 128 + cc + e] = v;
                }
                __syncwarp();
            }
        } else {
            // ---------------- mild: dq = Y1 E, dKc = Y2 E, dk = Y3 / E + dKc b; dG
            // waits in registers until every thread has read E and 1 / E
            const int r0 = 16 * I + gq;
            float y1a[16], y2a[16], y3a[16];  // all four 8-column groups at once
            tmem_ld16x256x4(taddr(tm + TM_Y1 + 32 * Q, I * 32, 0), y1a);
            tmem_ld16x256x4(taddr(tm + TM_Y2 + 32 * Q, I * 32, 0), y2a);
            tmem_ld16x256x4(taddr(tm + TM_Y3 + 32 * Q, I * 32, 0), y3a);
            tmem_wait_ld();
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int cb = 32 * Q + 8 * nt, cc = cb + 2 * tq;
                const float *y1 = y1a + 4 * nt, *y2 = y2a + 4 * nt, *y3 = y3a + 4 * nt;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int r = r0 + 8 * h2;
                    const float2 E2 = __half22float2(*reinterpret_cast<const __half2 *>(sm + MEM + raw16(r, cc)));
                    const float2 Ei2 = __half22float2(*reinterpret_cast<const __half2 *>(sm + MEI + raw16(r, cc)));
                    const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + RQ + raw16(r, cc)));
                    const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + RK + raw16(r, cc)));
                    const float2 bx = gld2<GB>(sm + RB + graw<GB>(r, cc)), bf = act_b2(ga, bx);
                    const float Ev[2] = {E2.x, E2.y}, Eiv[2] = {Ei2.x, Ei2.y}, qv[2] = {qf.x, qf.y},
                                kv[2] = {kf.x, kf.y}, bv[2] = {bf.x, bf.y}, bxv[2] = {bx.x, bx.y};
                    float dq[2], dk[2], db[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int x = 2 * h2 + e;
                        dq[e] = y1[x] * Ev[e];
                        const float dkc = y2[x] * Ev[e];
                        const float y3e = y3[x] * Eiv[e];
                        dk[e] = fmaf(dkc, bv[e], y3e);
                        db[e] = dkc * kv[e] * ga.db(bxv[e]);  // of b, or of its logit
                        // q dq + 2 b k dKc - k dk = q dq + k (b dKc - Y3 / E)
                        mdG[nt][x] = fmaf(qv[e], dq[e], kv[e] * fmaf(dkc, bv[e], -y3e));
                    }
                    *reinterpret_cast<uint32_t *>(sm + RQ + raw16(r, cc)) = pack_bf16(dq[0], dq[1]);
                    *reinterpret_cast<uint32_t *>(sm + RK + raw16(r, cc)) = pack_bf16(dk[0], dk[1]);
                    gst2<GB>(sm + RB + graw<GB>(r, cc), db[0], db[1]);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();  // dq, dk, db, dG formed; the pair-term data is consumed
        if (issuer) {
            fence_after_sync();
            if (more && !mild) {  // the next tile's operands into the space the pair terms used
                load_a1(nxt);
                load_a2(nxt);
            }
            if (!tail) {
                tma_store_5d(&mdq, sm + RQ, 0, h, c0, 0, bb);
                tma_store_5d(&mdk, sm + RK, 0, h, c0, 0, bb);
                tma_store_5d(&mdb, sm + RB, 0, h, c0, 0, bb);
                bulk_commit();
            }
        }
        if (tail) {  // rows 0 .. L - 1 only
            const size_t row = tok(d, bb, c0, h, 128);
            const size_t st16 = (size_t)d.H * 128 * 2, stg = (size_t)d.H * 128 * (GB ? 2 : 4);
            store_rows(reinterpret_cast<unsigned char *>(dq_out) + row * 2, st16, sm + RQ, 2, L, tid, kThreads);
            store_rows(reinterpret_cast<unsigned char *>(dk_out) + row * 2, st16, sm + RK, 2, L, tid, kThreads);
            store_rows(reinterpret_cast<unsigned char *>(db_out) + row * (GB ? 2 : 4), stg, sm + RB, GB ? 2 : 4, L,
                       tid, kThreads);
        }
        if (mild) {  // dG over E and 1 / E, which every thread has read
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2)
                    *reinterpret_cast<float2 *>(sm + RG + raw32(16 * I + gq + 8 * h2, 32 * Q + 8 * nt + 2 * tq)) =
                        make_float2(mdG[nt][2 * h2], mdG[nt][2 * h2 + 1]);
            named_sync(1, kCompute);
        }
        // ---------------- dg: reverse in-chunk cumsum of dG plus the chunk-end term
        if (compute) {
            const int fc2 = 32 * Q + lane;
            float x[16], run = 0.f;
#pragma unroll
            for (int r = 15; r >= 0; --r) {
                run += *reinterpret_cast<const float *>(sm + RG + raw32(16 * I + r, fc2));
                x[r] = run;
            }
            mtot[I * 128 + fc2] = run;
            // logits in: dg of the logit x_g is dg sigmoid(-x_g); x_g comes back from
            // global memory (L2), since g's tile now holds dG
            float sx[16];
            if (ga.on) {
#pragma unroll
                for (int r = 0; r < 16; ++r)
                    sx[r] = 16 * I + r < L ? gld1<GB>(static_cast<const unsigned char *>(g_in) +
                                                      (tok(d, bb, c0 + 16 * I + r, h, 128) + fc2) * (GB ? 2 : 4))
                                           : 0.f;
            }
            named_sync(1, kCompute);  // dG is read: g's tile is free
            if (issuer && more) load_b_g(nxt);
            // rowsum(dS' . S_c) carries gamma already in the mild frame (S_m dX)
            float after = (mild ? 1.f : mgam[fc2]) * (mend1[fc2] + mend1[128 + fc2] + mend1[256 + fc2] + mend1[384 + fc2]) +
                          mendk[fc2] + mendk[128 + fc2] + mendk[256 + fc2] + mendk[384 + fc2];
#pragma unroll
            for (int J = 0; J < 4; ++J)
                if (J > I) after += mtot[J * 128 + fc2];
            // dg leaves from the scan's registers: for each row a warp writes 32
            // consecutive channels, so g's tile is free once the scan has read dG
            constexpr int ges = GB ? 2 : 4;
            unsigned char *dgp = static_cast<unsigned char *>(dg_out) + (tok(d, bb, c0 + 16 * I, h, 128) + fc2) * ges;
            const size_t rstride = (size_t)d.H * 128 * ges;
#pragma unroll
            for (int r = 0; r < 16; ++r)
                if (16 * I + r < L) gst1<GB>(dgp + r * rstride, ga.on ? (x[r] + after) * ga.dg(sx[r]) : x[r] + after);
        }
        fence_before_sync();
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        if (issuer) {
            bulk_wait_read();  // dq, dk, db have left the raw tiles
            if (more) load_b_rest(nxt);
        }
    }
    if (issuer) bulk_wait_all();
    if (!(big <= kRange)) record_status(status, GDN2_ERR_RANGE);
    if (aborted && issuer) {
        record_status(status, GDN2_ERR_TIMEOUT);
        // every copy landed and every issued product done before the shared
        // and tensor memory go away
        if (issued[0] > 0) mbar_wait(&bars[0], (issued[0] - 1) & 1, kWait);
        if (pend_b >= 0) load_b_rest(pend_b);  // the requested tile's bytes complete its phase
        if (issued[2] > 0) {
            mbar_wait(&bars[3], (issued[2] - 1) & 1, kWait);
            mbar_wait(&bars[4], (issued[2] - 1) & 1, kWait);
        }
        mbar_wait(&bars[1], 0, kWait);
        mbar_wait(&bars[1], 1, kWait);
        if (nmild > 0) mbar_wait(&bars[2], (nmild - 1) & 1, kWait);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------- launcher
template <bool GB, bool ACT>
static cudaError_t tc_bwd_grad_run(const void *q, const void *k, const void *g, const void *b,
                                   const void *dO, void *dq, void *dk, void *dg, void *db, void *ws,
                                   unsigned int *status, const Dims &d, cudaStream_t s) {
    CUtensorMap mq, mk, mb, mg, mdo, mdq, mdk, mdb;
    if (!make_wide_map(&mq, q, true, d.B, d.T, d.H, 128, 64) || !make_wide_map(&mk, k, true, d.B, d.T, d.H, 128, 64) ||
        !make_wide_map(&mb, b, GB, d.B, d.T, d.H, 128, 64) || !make_wide_map(&mg, g, GB, d.B, d.T, d.H, 128, 64) ||
        !make_btHd_map(&mdo, dO, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_wide_map(&mdq, dq, true, d.B, d.T, d.H, 128, 64) || !make_wide_map(&mdk, dk, true, d.B, d.T, d.H, 128, 64) ||
        !make_wide_map(&mdb, db, GB, d.B, d.T, d.H, 128, 64))
        return cudaErrorInvalidValue;
    const TcWs lay = tc_ws_layout(d);
    cudaError_t e = cudaFuncSetAttribute(tc_bwd_grad_kernel<GB, ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tbg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    launch_begin(K_TC_BWD_GRAD, s);
    const long long ntiles = (long long)d.B * d.H * d.NC;
    const int grid = (int)(ntiles < sm_count() ? ntiles : sm_count());
    tc_bwd_grad_kernel<GB, ACT><<<grid, tbg::kThreads, tbg::SMEM_BYTES, s>>>(
        mq, mk, mb, mg, mdo, mdq, mdk, mdb, g, dq, dk, db, dg, (unsigned char *)ws, lay, status, d);
    launch_end(K_TC_BWD_GRAD, s);
    return cudaGetLastError();
}

cudaError_t tc_bwd_grad_launch(const void *q, const void *k, const void *g, const void *b,
                               const void *dO, void *dq, void *dk, void *dg, void *db, void *ws,
                               unsigned int *status, const Dims &d, cudaStream_t s) {
    if (d.act) return d.gb ? tc_bwd_grad_run<true, true>(q, k, g, b, dO, dq, dk, dg, db, ws, status, d, s)
                           : tc_bwd_grad_run<false, true>(q, k, g, b, dO, dq, dk, dg, db, ws, status, d, s);
    return d.gb ? tc_bwd_grad_run<true, false>(q, k, g, b, dO, dq, dk, dg, db, ws, status, d, s)
                : tc_bwd_grad_run<false, false>(q, k, g, b, dO, dq, dk, dg, db, ws, status, d, s);
}

}  // namespace gdn2
