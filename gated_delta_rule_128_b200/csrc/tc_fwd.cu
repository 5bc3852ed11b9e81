// Sequential part of the tensor-core forward of Gated Delta Rule-2 (bf16
// q/k/v/o, float32 gates and state, d_k = d_v = 128, chunk 64): the state
// pass and the outputs, from the chunk records of tc_prep.cu.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B): only the state crosses chunk borders.  Per chunk of 64 tokens
// entering with state S (factors relative to the chunk's middle row m,
// S_m = diag(e^G_m) S, U = w.v):
//   Delta = T U - W S_m
//   O = Qb S_m + P Delta,   S_next = diag(e^(G_L - G_m)) (S_m + Kh^T Delta)
//
// One CTA owns one (b, h) and one 64-column half of d_v and walks the
// sequence's chunks in order with its fp32 state slice resident in tensor
// memory.  The chunk records (Qb, Kh, -W, T, P, decay factors; 65 KB) are
// double-buffered in shared memory and requested two chunks ahead, since
// they do not depend on the state; v and w arrive by TMA one chunk ahead.
// Per chunk two tcgen05.mma round trips sit on the state's path:
//   (1) D = T U + (-W) S_m,  O = Qb S_m          (D in TMEM is Delta)
//   (2) O += P Delta,        S += Kh^T Delta
// then the state is rescaled into the next chunk's frame in TMEM and copied
// to fp16 for the next chunk's products.
//
// Precision and range: fp16 operands carry 11 significant bits (bf16 carries
// 8, which left the output error at the 5e-3 tolerance); Delta is formed in
// the f32 accumulator.  Any operand beyond 6e4 in magnitude is reported as
// GDN2_ERR_RANGE.
//
// For the backward the call can also leave in the workspace (TcWs): every
// chunk-entry state and S_T (fp16, true scale) and Delta per chunk.

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
constexpr uint32_t STG = 0;                  // two chunk records, REC_BYTES each
constexpr uint32_t RAW_V = 2 * REC_BYTES;    // v half, bf16 [64 pos][64]
constexpr uint32_t RAW_W = RAW_V + 8192;     // w half, f32  [64 pos][64]
constexpr uint32_t OP_U = RAW_W + 16384;     // U = w.v      [64 pos][64 v]  MN-major B
constexpr uint32_t OP_S = OP_U + 8192;       // S_m (fp16)   [128 key][64 v] MN-major B
constexpr uint32_t OP_D = OP_S + 16384;      // Delta        [64 pos][64 v]  MN-major B
constexpr uint32_t MISC = OP_D + 8192;       // mbarriers, TMEM slot
constexpr uint32_t SMEM_BYTES = MISC + 128 + 1024;
// tensor memory columns (256 allocated)
constexpr uint32_t TM_S = 0, TM_D = 64, TM_O = 128;
constexpr uint32_t ID_KM64 = idesc_f16(64, 64, false, true);
constexpr uint32_t ID_MM128x64 = idesc_f16(128, 64, true, true);
constexpr long long kWait = 2000000000LL;  // ~1 s of SM clocks per wait
constexpr float kRange = 6.0e4f;           // largest operand magnitude kept in fp16
}  // namespace tfwd

__global__ void __launch_bounds__(tfwd::kThreads, 1)
tc_fwd_kernel(const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mw,
              const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ ST,
              unsigned char *__restrict__ ws, int keep, TcWs lay, unsigned int *status, Dims d) {
    using namespace tfwd;
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~static_cast<uintptr_t>(1023));
    // 0, 1 records of stages 0, 1; 2 v and w; 3, 4 the two product groups
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + MISC + 64);
    float big = 0.f;  // largest operand magnitude seen (range check)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int vh = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, v0 = vh * 64;
    const int NC = d.NC, T = d.T, H = d.H;
    const int quarter = warp & 3, half = warp >> 2;
    const int key = quarter * 32 + lane;  // state row of this thread
    const size_t bh = (size_t)bb * H + h;
    const unsigned char *recs = ws + lay.rec + bh * NC * (size_t)REC_BYTES;

    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = *tslot;

    int issued[3] = {0, 0, 0};  // loads requested per barrier (thread 0)
    auto load_rec = [&](int cc) {
        const int s = cc & 1;
        mbar_expect_tx(&bars[s], REC_BYTES);
        bulk_load(sm + STG + s * REC_BYTES, recs + (size_t)cc * REC_BYTES, REC_BYTES, &bars[s]);
        ++issued[s];
    };
    auto load_vw = [&](int cc) {
        mbar_expect_tx(&bars[2], 8192 + 16384);
        tma_load_4d(sm + RAW_V, &mv, v0, h, cc * 64, bb, &bars[2]);
        tma_load_4d(sm + RAW_W, &mw, v0, h, cc * 64, bb, &bars[2]);
        ++issued[2];
    };
    if (tid == 0) {
        load_rec(0);
        if (NC > 1) load_rec(1);
        load_vw(0);
    }
    // state checkpoint c of this half: [128 key][64 v] fp16, true scale
    auto ckpt = [&](int c) { return ws + lay.ckS + ((bh * (NC + 1) + c) * 2 + vh) * 16384; };

    // initial state slice: S_m of chunk 0 into TMEM and OP_S; S0 itself to checkpoint 0
    bool ok = mbar_wait(&bars[0], 0, kWait);
    {
        const size_t so = st_off(d, bb, h);
        float x[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 t = S0 ? *reinterpret_cast<const float4 *>(S0 + so + (size_t)key * 128 + v0 + 32 * half + j)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
            x[j] = t.x; x[j + 1] = t.y; x[j + 2] = t.z; x[j + 3] = t.w;
        }
        if (keep)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) st_h8(ckpt(0) + sw128_chunk(key, 4 * half + jj, 128), x + 8 * jj);
        const float e = ok ? reinterpret_cast<const float *>(sm + STG + REC_FAC)[128 + key] : 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] *= e;
        tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half), x);
        tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), x + 16);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            st_h8(sm + OP_S + sw128_chunk(key, 4 * half + jj, 128), x + 8 * jj);
            big = absmax8(x + 8 * jj, big);
        }
        tmem_wait_st();
    }
    fence_proxy_async();
    fence_before_sync();
    bool abort = __syncthreads_or(!ok);

    for (int c = 0; c < NC && !abort; ++c) {
        const int s = c & 1, c0 = c * 64;
        const uint32_t par = c & 1;
        unsigned char *stg = sm + STG + s * REC_BYTES;
        // ---------------- U = w.v for this half, then product group 1
        ok = mbar_wait(&bars[s], (c >> 1) & 1, kWait);
        ok = ok && mbar_wait(&bars[2], par, kWait);
        const float gam = reinterpret_cast<const float *>(stg + REC_FAC)[key];  // e^(G_L - G_m)
        {
            const int r = tid >> 2, cg = tid & 3;  // row, 16-column group
            const uint4 vr0 = *reinterpret_cast<const uint4 *>(sm + RAW_V + r * 128 + cg * 32);
            const uint4 vr1 = *reinterpret_cast<const uint4 *>(sm + RAW_V + r * 128 + cg * 32 + 16);
            const float4 *wr = reinterpret_cast<const float4 *>(sm + RAW_W + r * 256 + cg * 64);
            const __nv_bfloat162 *va = reinterpret_cast<const __nv_bfloat162 *>(&vr0);
            const __nv_bfloat162 *vb = reinterpret_cast<const __nv_bfloat162 *>(&vr1);
            float u[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 w4 = wr[i];
                const __nv_bfloat162 p0 = i < 2 ? va[2 * i] : vb[2 * i - 4];
                const __nv_bfloat162 p1 = i < 2 ? va[2 * i + 1] : vb[2 * i - 3];
                u[4 * i] = w4.x * __low2float(p0);
                u[4 * i + 1] = w4.y * __high2float(p0);
                u[4 * i + 2] = w4.z * __low2float(p1);
                u[4 * i + 3] = w4.w * __high2float(p1);
            }
            st_h8(sm + OP_U + sw128_chunk(r, 2 * cg, 64), u);
            st_h8(sm + OP_U + sw128_chunk(r, 2 * cg + 1, 64), u + 8);
            big = absmax8(u, big);
            big = absmax8(u + 8, big);
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0) {
            fence_after_sync();
            if (c + 1 < NC) load_vw(c + 1);  // raw v and w consumed
            const uint32_t st = smem_addr(stg), u = smem_addr(sm + OP_U), sS = smem_addr(sm + OP_S);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_D, desc_kmajor(st + REC_T, 64, ks), desc_mnmajor(u, 64, ks), ID_KM64, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_D, desc_kmajor(st + REC_WN, 64, ks), desc_mnmajor(sS, 128, ks), ID_KM64, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tm + TM_O, desc_kmajor(st + REC_QB, 64, ks), desc_mnmajor(sS, 128, ks), ID_KM64, ks > 0);
            mma_commit(&bars[3]);
        }
        // ---------------- Delta to fp16, product group 2
        ok = mbar_wait(&bars[3], par, kWait);
        fence_after_sync();
        {
            float dl[32];
            tmem_ld16(taddr(tm + TM_D, quarter * 32, 32 * half), dl);
            tmem_ld16(taddr(tm + TM_D, quarter * 32, 32 * half + 16), dl + 16);
            tmem_wait_ld();
            if (lane < 16) {
                const int r = quarter * 16 + lane;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    st_h8(sm + OP_D + sw128_chunk(r, 4 * half + jj, 64), dl + 8 * jj);
                    big = absmax8(dl + 8 * jj, big);
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0) {
            fence_after_sync();
            if (keep) {  // Delta of this chunk and half, for the backward
                bulk_store(ws + lay.ckD + ((bh * NC + c) * 2 + vh) * 8192, sm + OP_D, 8192);
                bulk_commit();
            }
            const uint32_t st = smem_addr(stg), dl = smem_addr(sm + OP_D);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_O, desc_kmajor(st + REC_P, 64, ks), desc_mnmajor(dl, 64, ks), ID_KM64, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tm + TM_S, desc_mnmajor(st + REC_KH, 64, ks), desc_mnmajor(dl, 64, ks), ID_MM128x64, 1);
            mma_commit(&bars[4]);
        }
        // ---------------- output rows; state into the next chunk's frame
        ok = mbar_wait(&bars[4], par, kWait);
        float ref = 1.f;  // e^G_m of the next chunk
        if (c + 1 < NC) {
            ok = ok && mbar_wait(&bars[s ^ 1], ((c + 1) >> 1) & 1, kWait);
            ref = reinterpret_cast<const float *>(sm + STG + (s ^ 1) * REC_BYTES + REC_FAC)[128 + key];
        }
        fence_after_sync();
        {
            float ov[32], sv[32];
            tmem_ld16(taddr(tm + TM_O, quarter * 32, 32 * half), ov);
            tmem_ld16(taddr(tm + TM_O, quarter * 32, 32 * half + 16), ov + 16);
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half), sv);
            tmem_ld16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), sv + 16);
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
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] *= gam;  // S_{c+1}, true scale
            if (keep)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) st_h8(ckpt(c + 1) + sw128_chunk(key, 4 * half + jj, 128), sv + 8 * jj);
            if (c == NC - 1 && ST) {
                float *dst = ST + st_off(d, bb, h) + (size_t)key * 128 + v0 + 32 * half;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
            }
            if (c + 1 < NC) {
#pragma unroll
                for (int j = 0; j < 32; ++j) sv[j] *= ref;  // S_m of the next chunk
                tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half), sv);
                tmem_st16(taddr(tm + TM_S, quarter * 32, 32 * half + 16), sv + 16);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    st_h8(sm + OP_S + sw128_chunk(key, 4 * half + jj, 128), sv + 8 * jj);
                    big = absmax8(sv + 8 * jj, big);
                }
                tmem_wait_st();
            }
        }
        if (tid == 0 && keep) bulk_wait_read();  // the Delta copy reads OP_D, rewritten next chunk
        fence_proxy_async();
        fence_before_sync();
        if (__syncthreads_or(!ok)) { abort = true; break; }
        if (tid == 0 && c + 2 < NC) load_rec(c + 2);  // this stage's record is consumed
    }
    if (!(big <= kRange)) record_status(status, GDN2_ERR_RANGE);
    if (tid == 0) {
        bulk_wait_all();
        if (abort) {
            record_status(status, GDN2_ERR_TIMEOUT);
            // let every requested copy land before the CTA's shared memory goes away
            for (int i = 0; i < 3; ++i)
                if (issued[i] > 0) mbar_wait(&bars[i], (issued[i] - 1) & 1, kWait);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

// ---------------------------------------------------------------- launcher
cudaError_t tc_prep_launch(const void *q, const void *k, const float *g, const float *b, void *ws,
                           unsigned int *status, const Dims &d, cudaStream_t s);

// keep != 0: also leave the chunk states and Delta for the backward
cudaError_t tc_fwd_launch(const void *q, const void *k, const void *v, const float *g,
                          const float *b, const float *w, const float *S0, void *o, float *ST,
                          void *ws, int keep, unsigned int *status, const Dims &d, cudaStream_t s) {
    cudaError_t e = tc_prep_launch(q, k, g, b, ws, status, d, s);
    if (e != cudaSuccess) return e;
    CUtensorMap mv, mw;
    if (!make_btHd_map(&mv, v, true, d.B, d.T, d.H, 128, 64, 64) ||
        !make_btHd_map(&mw, w, false, d.B, d.T, d.H, 128, 64, 64))
        return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(tc_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tfwd::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    launch_begin(K_TC_FWD, s);
    tc_fwd_kernel<<<dim3(2, d.H, d.B), tfwd::kThreads, tfwd::SMEM_BYTES, s>>>(
        mv, mw, S0, (__nv_bfloat16 *)o, ST, (unsigned char *)ws, keep, tc_ws_layout(d), status, d);
    launch_end(K_TC_FWD, s);
    return cudaGetLastError();
}

}  // namespace gdn2
