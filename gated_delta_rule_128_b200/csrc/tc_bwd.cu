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
//  * tc_bwd_grad_kernel: one CTA per (b, h, chunk), all chunks in parallel,
//    full d_v; five products, then three accumulations, then dq, dk, db, dg.

#include "common.cuh"
#include "tc.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace gdn2 {
using namespace tc;
using namespace tcc;

// ============================================================ state kernel
namespace tbs {
constexpr int kThreads = 256;
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
// half-sums go to the workspace for the gradient kernel.
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
    const int quarter = warp & 3, half = warp >> 2;
    const int key = quarter * 32 + lane;
    const int r16 = quarter * 16 + lane;  // row of an M = 64 accumulator (lanes 0..15)
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

    int issued[5] = {0, 0, 0, 0, 0};  // loads requested per barrier (thread 0)
    int groups[3] = {0, 0, 0};        // commits to barriers 5, 6, 7 (thread 0)
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
    // dU of chunk cc (TMEM) -> dv, dw in place of v, w; -dU staged; then the
    // stores, and the next v, w tiles (chunk cc - 1).  All threads.
    auto flush_du = [&](int cc, uint32_t vw_par, uint32_t du_par) {
        bool fine = mbar_wait(&bars[7], du_par, kWait);
        fine = mbar_wait(&bars[4], vw_par, kWait) && fine;
        fence_after_sync();
        float du[32];
        tmem_ld16(taddr(tm + TM_DU, quarter * 32, 32 * half), du);
        tmem_ld16(taddr(tm + TM_DU, quarter * 32, 32 * half + 16), du + 16);
        tmem_wait_ld();
        if (lane < 16) {
            const int r = r16;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {  // v chunk 4 * half + jj: 8 columns
                unsigned char *pv = sm + VV + sw128_chunk(r, 4 * half + jj, 64);
                const uint4 vq = *reinterpret_cast<const uint4 *>(pv);
                const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vq);
                unsigned char *pw0 = sm + VW + half * 8192 + sw128_chunk(r, 2 * jj, 64);
                unsigned char *pw1 = sm + VW + half * 8192 + sw128_chunk(r, 2 * jj + 1, 64);
                const float4 w0 = *reinterpret_cast<const float4 *>(pw0);
                const float4 w1 = *reinterpret_cast<const float4 *>(pw1);
                const float *u = du + 8 * jj;
                float dv8[8] = {u[0] * w0.x, u[1] * w0.y, u[2] * w0.z, u[3] * w0.w,
                                u[4] * w1.x, u[5] * w1.y, u[6] * w1.z, u[7] * w1.w};
                *reinterpret_cast<float4 *>(pw0) = make_float4(
                    u[0] * __low2float(v2[0]), u[1] * __high2float(v2[0]), u[2] * __low2float(v2[1]),
                    u[3] * __high2float(v2[1]));
                *reinterpret_cast<float4 *>(pw1) = make_float4(
                    u[4] * __low2float(v2[2]), u[5] * __high2float(v2[2]), u[6] * __low2float(v2[3]),
                    u[7] * __high2float(v2[3]));
                st_bf16x8(pv, dv8);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) du[j] = -du[j];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                st_h8(sm + NDU + sw128_chunk(r, 4 * half + jj, 64), du + 8 * jj);
                big = absmax8(du + 8 * jj, big);
            }
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&mdv, sm + VV, v0, h, cc * 64, bb);
            tma_store_4d(&mdw, sm + VW, v0, h, cc * 64, bb);
            tma_store_4d(&mdw, sm + VW + 8192, v0 + 32, h, cc * 64, bb);
            bulk_store(ws + lay.ckndU + ((bh * NC + cc) * 2 + vh) * 8192, sm + NDU, 8192);
            bulk_commit();
            bulk_wait_read();  // VV, VW and NDU may be rewritten
            if (cc > 0) load_vw(cc - 1);
        }
        return fine;
    };

    if (tid == 0) {
        load_rec(NC - 1);
        if (NC > 1) load_rec(NC - 2);
        load_do(NC - 1);
        load_s(NC);
        load_vw(NC - 1);
    }
    // ---------------- prologue: dS_T (or zero), the last chunk's end term and dX; dO
    bool ok;
    {
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
        if (half == 0)
            reinterpret_cast<float *>(ws + lay.ckEnd + ((bh * NC + NC - 1) * 2 + vh) * 512)[key] =
                sEnd[key] + sEnd[128 + key];
        if (tid == 0) {
            fence_after_sync();
            bulk_store(ws + lay.ckdS + ((bh * NC + NC - 1) * 2 + vh) * 16384, sm + OP_DS, 16384);
            bulk_commit();
            if (NC > 1) {
                load_s(NC - 1);
                load_do(NC - 2);
            }
        }
    }

    for (int i = 0; i < NC && !abort; ++i) {
        const int c = NC - 1 - i;
        const uint32_t par = i & 1;
        unsigned char *stg = sm + STG + (c & 1) * REC_BYTES;
        // ---------------- (1) dDelta products, then Qb^T dO
        ok = mbar_wait(&bars[c & 1], (i >> 1) & 1, kWait) && ok;  // record c
        if (tid == 0) {
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
        if (c + 1 < NC) ok = flush_du(c + 1, (i - 1) & 1, (i - 1) & 1) && ok;
        // ---------------- dDelta to fp16, (2) products
        ok = mbar_wait(&bars[5], par, kWait) && ok;
        fence_after_sync();
        {
            float dd[32];
            tmem_ld16(taddr(tm + TM_DD, quarter * 32, 32 * half), dd);
            tmem_ld16(taddr(tm + TM_DD, quarter * 32, 32 * half + 16), dd + 16);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    st_h8(sm + OP_DD + sw128_chunk(r16, 4 * half + jj, 64), dd + 8 * jj);
                    big = absmax8(dd + 8 * jj, big);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
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
            bulk_wait_read();  // the dX copy has left OP_DS
        }
        // ---------------- dS_c; the previous chunk's end term, dX and dO
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
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (c > 0) {
            if (half == 0)
                reinterpret_cast<float *>(ws + lay.ckEnd + ((bh * NC + c - 1) * 2 + vh) * 512)[key] =
                    sEnd[key] + sEnd[128 + key];
            if (tid == 0) {
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
            }
        }
    }
    if (!abort) ok = flush_du(0, (NC - 1) & 1, (NC - 1) & 1);
    if (!(big <= kRange)) record_status(status, GDN2_ERR_RANGE);
    if (tid == 0) bulk_wait_all();
    if (tid == 0 && (abort || !ok)) {
        record_status(status, GDN2_ERR_TIMEOUT);
        for (int k2 = 0; k2 < 5; ++k2)
            if (issued[k2] > 0) mbar_wait(&bars[k2], (issued[k2] - 1) & 1, kWait);
        for (int k2 = 0; k2 < 3; ++k2)
            if (groups[k2] > 0) mbar_wait(&bars[5 + k2], (groups[k2] - 1) & 1, kWait);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

// ============================================================ chunk kernel
namespace tbg {
constexpr int kThreads = 256;
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_B = 32768, RAW_G = 65536;  // g, later G - G_m
constexpr uint32_t OP_DO = 98304;     // dO fp16 [64 pos][128 v] K-major (in place of raw dO)
constexpr uint32_t BL_S = 114688;     // S_m [128 key][128 v] K-major B (the checkpoint; later Qb, Kc, Kh; then dG)
constexpr uint32_t BL_DS = 147456;    // dS_m [128 key][128 v]
constexpr uint32_t BL_D = 180224;     // Delta [64 pos][128 v]              (later dP, dA)
constexpr uint32_t BL_NDU = 196608;   // -dU [64 pos][128 v]
constexpr uint32_t OP_QB = BL_S, OP_KC = BL_S + 16384, OP_KH = BL_S + 32768;
constexpr uint32_t OP_DP = BL_D, OP_DA = BL_D + 8192;
constexpr uint32_t MISC = 212992;     // sGam, sRef [128]; sEnd [128]; scan [8][128]; mbarriers; slot
constexpr uint32_t SMEM_BYTES = MISC + 1536 + 4096 + 128 + 1024;
constexpr uint32_t TM_DP = 0, TM_DA = 64, TM_Y1 = 128, TM_Y2 = 256, TM_Y3 = 384;
constexpr uint32_t ID_KK64 = idesc_f16(64, 64, false, false);
constexpr uint32_t ID_KK128 = idesc_f16(64, 128, false, false);
constexpr uint32_t ID_KM128 = idesc_f16(64, 128, false, true);
constexpr uint32_t ID_MM128 = idesc_f16(64, 128, true, true);
constexpr long long kWait = 2000000000LL;
constexpr float kRange = 6.0e4f;
}  // namespace tbg

__global__ void __launch_bounds__(tbg::kThreads, 1)
tc_bwd_grad_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mdo, const __grid_constant__ CUtensorMap mg,
                   const __grid_constant__ CUtensorMap mb, __nv_bfloat16 *__restrict__ dqout,
                   __nv_bfloat16 *__restrict__ dkout, float *__restrict__ dbout,
                   float *__restrict__ dgout, unsigned char *__restrict__ ws, TcWs lay,
                   unsigned int *status, Dims d) {
    using namespace tbg;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *sGam = reinterpret_cast<float *>(sm + MISC);
    float *sRef = reinterpret_cast<float *>(sm + MISC + 512);
    float *sEnd = reinterpret_cast<float *>(sm + MISC + 1024);
    float *scan = reinterpret_cast<float *>(sm + MISC + 1536);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC + 1536 + 4096);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 1536 + 4096 + 64);
    float big = 0.f, gbig = 0.f;  // range checks: operand magnitude, |G - G_m|

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, c0 = c * 64;
    const int NC = d.NC, T = d.T, H = d.H, L = min(64, T - c0);
    const int quarter = warp & 3, half = warp >> 2;
    const size_t bh = (size_t)bb * H + h;

    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    if (tid == 0) {
        mbar_expect_tx(&bars[0], 16384 * 2 + 32768 * 2 + 16384 + 32768 * 2 + 16384 * 2);
        tma_load_4d(sm + RAW_Q, &mq, 0, h, c0, bb, &bars[0]);
        tma_load_4d(sm + RAW_K, &mk, 0, h, c0, bb, &bars[0]);
        tma_load_4d(sm + RAW_B, &mb, 0, h, c0, bb, &bars[0]);
        tma_load_4d(sm + RAW_G, &mg, 0, h, c0, bb, &bars[0]);
        tma_load_4d(sm + OP_DO, &mdo, 0, h, c0, bb, &bars[0]);
        bulk_load(sm + BL_S, ws + lay.ckS + ((bh * (NC + 1) + c) * 2) * 16384, 32768, &bars[0]);
        bulk_load(sm + BL_DS, ws + lay.ckdS + ((bh * NC + c) * 2) * 16384, 32768, &bars[0]);
        bulk_load(sm + BL_D, ws + lay.ckD + ((bh * NC + c) * 2) * 8192, 16384, &bars[0]);
        bulk_load(sm + BL_NDU, ws + lay.ckndU + ((bh * NC + c) * 2) * 8192, 16384, &bars[0]);
    }
    if (tid < 128) {
        const float *e0 = reinterpret_cast<const float *>(ws + lay.ckEnd + ((bh * NC + c) * 2) * 512);
        sEnd[tid] = e0[tid] + e0[128 + tid];
    }
    bool ok = mbar_wait(&bars[0], 0, kWait);
    // ---------------- G1: decay, dO operand; five products (the checkpoint holds S_m)
    float G[8][4];
    cumsum_local(reinterpret_cast<const float *>(sm + RAW_G), scan, warp, lane, G);
    // dO: raw bf16 rows [64][128] -> fp16 K-major tile in place (values held in registers)
    uint2 dor[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) dor[m] = *reinterpret_cast<const uint2 *>(sm + OP_DO + (8 * warp + m) * 256 + lane * 8);
    bool abort = __syncthreads_or(!ok);
    if (!abort) {
        cumsum_finish(scan, warp, lane, G, sGam, sRef);
        float *sG = reinterpret_cast<float *>(sm + RAW_G);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = 8 * warp + m;
            *reinterpret_cast<float4 *>(sG + r * 128 + 4 * lane) = make_float4(G[m][0], G[m][1], G[m][2], G[m][3]);
            const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(&dor[m]);
            st_h4(sm + OP_DO + sw128_off(r, 4 * lane, 64), __low2float(d2[0]), __high2float(d2[0]),
                  __low2float(d2[1]), __high2float(d2[1]));
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            const uint64_t dO = desc_kmajor(smem_addr(sm + OP_DO), 64, 0),
                           S = desc_kmajor(smem_addr(sm + BL_S), 128, 0),
                           DS = desc_kmajor(smem_addr(sm + BL_DS), 128, 0),
                           D = desc_kmajor(smem_addr(sm + BL_D), 64, 0),
                           NDU = desc_kmajor(smem_addr(sm + BL_NDU), 64, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a_do = kstep_kmajor(dO, 64, ks), a_ndu = kstep_kmajor(NDU, 64, ks),
                               a_d = kstep_kmajor(D, 64, ks), b_s = kstep_kmajor(S, 128, ks);
                mma_bf16(tm + TM_DP, a_do, a_d, ID_KK64, ks > 0);
                mma_bf16(tm + TM_DA, a_ndu, a_d, ID_KK64, ks > 0);
                mma_bf16(tm + TM_Y1, a_do, b_s, ID_KK128, ks > 0);
                mma_bf16(tm + TM_Y2, a_ndu, b_s, ID_KK128, ks > 0);
                mma_bf16(tm + TM_Y3, a_d, kstep_kmajor(DS, 128, ks), ID_KK128, ks > 0);
            }
            mma_commit(&bars[1]);
        }
        // ---------------- G2: masked dP, dA; Qb, Kc, Kh; three accumulations
        ok = mbar_wait(&bars[1], 0, kWait);
        fence_after_sync();
        {
            float row[64];
            const uint32_t base = warp < 4 ? tm + TM_DP : tm + TM_DA;
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld16(taddr(base, quarter * 32, 16 * j), row + 16 * j);
            tmem_wait_ld();
            if (lane < 16) {
                const int r = quarter * 16 + lane;
                // dP keeps j <= r; dA = -strictly-lower(dU Delta^T) = strictly-lower of (-dU) Delta^T
#pragma unroll
                for (int j = 0; j < 64; ++j) row[j] = (warp < 4 ? j <= r : j < r) ? row[j] : 0.f;
                unsigned char *dst = sm + (warp < 4 ? OP_DP : OP_DA);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    st_h8(dst + sw128_chunk(r, jj, 64), row + 8 * jj);
                    big = absmax8(row + 8 * jj, big);
                }
            }
        }
        gbig = fmaxf(gbig, write_factors(sm + RAW_Q, sm + RAW_K, reinterpret_cast<const float *>(sm + RAW_B),
                                       G, sm + OP_QB, sm + OP_KC, sm + OP_KH, warp, lane));
        fence_proxy_async();
        fence_before_sync();
        abort = __syncthreads_or(!ok);
    }
    if (!abort) {
        if (tid == 0) {
            fence_after_sync();
            const uint32_t dP = smem_addr(sm + OP_DP), dA = smem_addr(sm + OP_DA);
            const uint64_t kP = desc_kmajor(dP, 64, 0), kA = desc_kmajor(dA, 64, 0),
                           mP = desc_mnmajor(dP, 64, 0), mA = desc_mnmajor(dA, 64, 0),
                           qb = desc_mnmajor(smem_addr(sm + OP_QB), 64, 0),
                           kc = desc_mnmajor(smem_addr(sm + OP_KC), 64, 0),
                           kh = desc_mnmajor(smem_addr(sm + OP_KH), 64, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t b_kh = kstep_mnmajor(kh, ks);
                mma_bf16(tm + TM_Y1, kstep_kmajor(kP, 64, ks), b_kh, ID_KM128, 1);
                mma_bf16(tm + TM_Y2, kstep_kmajor(kA, 64, ks), b_kh, ID_KM128, 1);
                mma_bf16(tm + TM_Y3, kstep_mnmajor(mP, ks), kstep_mnmajor(qb, ks), ID_MM128, 1);
                mma_bf16(tm + TM_Y3, kstep_mnmajor(mA, ks), kstep_mnmajor(kc, ks), ID_MM128, 1);
            }
            mma_commit(&bars[2]);
        }
        // ---------------- G3: dq, dk, db and dG per (row, channel)
        // The three accumulators go through shared memory (YS, [3][64][128]
        // f32 with 16-byte chunks XOR-swizzled by row) so that every warp then
        // walks whole rows with lanes across channels: conflict-free reads and
        // coalesced output rows.
        ok = mbar_wait(&bars[2], 0, kWait);
        fence_after_sync();
        float *YS = reinterpret_cast<float *>(sm + BL_S);  // operands of G2 are consumed
        {
            const int r = quarter * 16 + lane;
#pragma unroll 1
            for (int a = 0; a < 3; ++a) {
                const uint32_t col0 = (a == 0 ? TM_Y1 : a == 1 ? TM_Y2 : TM_Y3) + 64 * half;
                float y[64];
#pragma unroll
                for (int j = 0; j < 4; ++j) tmem_ld16(taddr(tm + col0, quarter * 32, 16 * j), y + 16 * j);
                tmem_wait_ld();
                if (lane < 16) {
                    float *row = YS + (a * 64 + r) * 128;
#pragma unroll
                    for (int ch = 0; ch < 16; ++ch) {  // logical 16-B chunk 16 * half + ch
                        const int lc = 16 * half + ch, pc = lc ^ (r & 31);
                        *reinterpret_cast<float4 *>(row + 4 * pc) =
                            make_float4(y[4 * ch], y[4 * ch + 1], y[4 * ch + 2], y[4 * ch + 3]);
                    }
                }
            }
        }
        __syncthreads();
        {
            const float *sG = reinterpret_cast<const float *>(sm + RAW_G);
            const float *rb = reinterpret_cast<const float *>(sm + RAW_B);
            float *sdG = YS;  // row r of dG overwrites row r of Y1 (read first, same warp)
#pragma unroll 1
            for (int i8 = 0; i8 < 8; ++i8) {
                const int r = warp + 8 * i8, pc = lane ^ (r & 31);
                const float4 y1 = *reinterpret_cast<const float4 *>(YS + (0 * 64 + r) * 128 + 4 * pc);
                const float4 y2 = *reinterpret_cast<const float4 *>(YS + (1 * 64 + r) * 128 + 4 * pc);
                const float4 y3 = *reinterpret_cast<const float4 *>(YS + (2 * 64 + r) * 128 + 4 * pc);
                const float4 G4 = *reinterpret_cast<const float4 *>(sG + r * 128 + 4 * lane);
                const float4 b4 = *reinterpret_cast<const float4 *>(rb + r * 128 + 4 * lane);
                const uint2 qr = *reinterpret_cast<const uint2 *>(sm + RAW_Q + r * 256 + 8 * lane);
                const uint2 kr = *reinterpret_cast<const uint2 *>(sm + RAW_K + r * 256 + 8 * lane);
                const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qr);
                const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kr);
                const float Y1[4] = {y1.x, y1.y, y1.z, y1.w}, Y2[4] = {y2.x, y2.y, y2.z, y2.w},
                            Y3[4] = {y3.x, y3.y, y3.z, y3.w}, Gv[4] = {G4.x, G4.y, G4.z, G4.w},
                            bf[4] = {b4.x, b4.y, b4.z, b4.w};
                const float qf[4] = {__low2float(q2[0]), __high2float(q2[0]), __low2float(q2[1]), __high2float(q2[1])};
                const float kf[4] = {__low2float(k2[0]), __high2float(k2[0]), __low2float(k2[1]), __high2float(k2[1])};
                float dq[4], dk[4], db[4], dG[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float E = __expf(Gv[e]), Ei = __expf(-Gv[e]);
                    const float dkc = Y2[e] * E, dkh = Y3[e] * Ei;
                    dq[e] = Y1[e] * E;
                    db[e] = dkc * kf[e];
                    dk[e] = dkc * bf[e] + dkh;
                    dG[e] = dq[e] * qf[e] + dkc * bf[e] * kf[e] - dkh * kf[e];
                }
                *reinterpret_cast<float4 *>(sdG + r * 128 + 4 * lane) = make_float4(dG[0], dG[1], dG[2], dG[3]);
                if (r < L) {
                    const size_t o4 = tok(d, bb, c0 + r, h, 128) + 4 * lane;
                    *reinterpret_cast<uint2 *>(dqout + o4) = make_uint2(pack_bf16(dq[0], dq[1]), pack_bf16(dq[2], dq[3]));
                    *reinterpret_cast<uint2 *>(dkout + o4) = make_uint2(pack_bf16(dk[0], dk[1]), pack_bf16(dk[2], dk[3]));
                    *reinterpret_cast<float4 *>(dbout + o4) = make_float4(db[0], db[1], db[2], db[3]);
                }
            }
        }
        abort = __syncthreads_or(!ok);
        if (!abort) {
            // dg = reverse in-chunk cumsum of dG with the chunk-end term on the last row;
            // thread (channel, part): part 1 scans rows 32..63, part 0 rows 0..31 after
            // adding the sum of rows 32..63 itself
            const float *sdG = YS;
            const int ch = tid & 127, part = tid >> 7;
            float acc = sEnd[ch];
            if (part == 0)
                for (int rr = 32; rr < 64; ++rr) acc += sdG[rr * 128 + ch];
            const int hi = part ? 63 : 31, lo = part ? 32 : 0;
            for (int rr = hi; rr >= lo; --rr) {
                acc += sdG[rr * 128 + ch];
                if (rr < L) dgout[tok(d, bb, c0 + rr, h, 128) + ch] = acc;
            }
        }
    }
    if (!(big <= kRange) || !(gbig <= 9.f)) record_status(status, GDN2_ERR_RANGE);
    if (abort && tid == 0) {
        record_status(status, GDN2_ERR_TIMEOUT);
        mbar_wait(&bars[0], 0, kWait);
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
    CUtensorMap mq, mk, mdo_half, mdo, mg, mb, mv, mw, mdv, mdw;
    if (!make_btHd_map(&mq, q, true, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mk, k, true, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mdo_half, dO, true, d.B, d.T, d.H, 128, 64, 64) ||
        !make_btHd_map(&mv, v, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mw, w, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mdv, dv, true, d.B, d.T, d.H, 128, 64, 64, true) ||
        !make_btHd_map(&mdw, dw, false, d.B, d.T, d.H, 128, 64, 32, true) ||
        !make_btHd_map(&mdo, dO, true, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mg, g, false, d.B, d.T, d.H, 128, 64, 128) ||
        !make_btHd_map(&mb, b, false, d.B, d.T, d.H, 128, 64, 128))
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
    tc_bwd_grad_kernel<<<dim3(d.NC, d.H, d.B), tbg::kThreads, tbg::SMEM_BYTES, s>>>(
        mq, mk, mdo, mg, mb, (__nv_bfloat16 *)dq, (__nv_bfloat16 *)dk, db, dg, (unsigned char *)ws,
        lay, status, d);
    launch_end(K_TC_BWD_GRAD, s);
    return cudaGetLastError();
}

}  // namespace gdn2
