// Pieces shared by the tensor-core forward and backward kernels: the in-chunk
// cumulative log-decay, the decay-scaled fp16 operand tiles, and small store
// helpers.  Thread layout of these helpers (256 threads, 64-row chunk, 128 key
// channels): warp w owns rows 8w..8w+7, lane l owns channels 4l..4l+3.
//
// Decay factors are taken relative to the chunk's middle row m = 31
// ("Gated DeltaNet-2", LIT-802 review, Key takeaways 2: the state is
// normalised by the cumulative decay; here the normalisation point is moved
// to the chunk's middle to keep every factor within fp16 range):
//   E = e^(G - G_m),  Qb = q.E,  Kc = b.k.E,  Kh = k / E,
//   gamma_m = e^(G_L - G_m) (sGam),  e^(G_m) (sRef).
#pragma once

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {
namespace tcc {
using namespace tc;

__device__ __forceinline__ void st_h4(unsigned char *p, float a, float b, float c, float d) {
    uint2 v = make_uint2(pack_f16(a, b), pack_f16(c, d));
    *reinterpret_cast<uint2 *>(p) = v;
}
__device__ __forceinline__ void st_h8(unsigned char *p, const float *x) {
    uint4 v = make_uint4(pack_f16(x[0], x[1]), pack_f16(x[2], x[3]), pack_f16(x[4], x[5]),
                         pack_f16(x[6], x[7]));
    *reinterpret_cast<uint4 *>(p) = v;
}
__device__ __forceinline__ void st_bf16x8(unsigned char *p, const float *x) {
    uint4 v = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                         pack_bf16(x[6], x[7]));
    *reinterpret_cast<uint4 *>(p) = v;
}
__device__ __forceinline__ float absmax8(const float *x, float m) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
    return m;
}
// 8 fp16 values of a 16-B chunk, widened
__device__ __forceinline__ void ld_h8(const unsigned char *p, float *x) {
    uint4 v = *reinterpret_cast<const uint4 *>(p);
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// Step 1 of the cumsum: local inclusive prefix over the warp's 8 rows (raw g
// tile row-major [64][128] f32); the warp's totals go to scan[warp][128].
__device__ __forceinline__ void cumsum_local(const float *rg, float *scan, int warp, int lane,
                                             float G[8][4]) {
    float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        float4 t = *reinterpret_cast<const float4 *>(rg + (8 * warp + m) * 128 + 4 * lane);
        run[0] += t.x; run[1] += t.y; run[2] += t.z; run[3] += t.w;
#pragma unroll
        for (int i = 0; i < 4; ++i) G[m][i] = run[i];
    }
    *reinterpret_cast<float4 *>(scan + warp * 128 + 4 * lane) = make_float4(run[0], run[1], run[2], run[3]);
}

// Step 2 (after a block barrier): add the earlier warps' totals and express G
// relative to row 31; warp 0 writes e^(G_L - G_m) and e^(G_m) per channel.
// Rows past the chunk's end hold g = 0 (zero-filled tiles), so row 63
// carries G_L of a short last chunk.
__device__ __forceinline__ void cumsum_finish(const float *scan, int warp, int lane, float G[8][4],
                                              float *sGam, float *sRef) {
    float pre[4] = {0.f, 0.f, 0.f, 0.f}, tot[4] = {0.f, 0.f, 0.f, 0.f}, ref[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) {
        float4 t = *reinterpret_cast<const float4 *>(scan + w2 * 128 + 4 * lane);
        float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (w2 < warp) pre[i] += tv[i];
            if (w2 < 4) ref[i] += tv[i];
            tot[i] += tv[i];
        }
    }
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i) G[m][i] += pre[i] - ref[i];
    if (warp == 0)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            sGam[4 * lane + i] = __expf(tot[i] - ref[i]);
            sRef[4 * lane + i] = __expf(ref[i]);
        }
}

// Operands of the chunk record from the raw q, k (bf16 [64][128]) and b (f32
// [64][128]) tiles: Kc = b.k.E into rows 0..63 and Qb = q.E into rows
// 64..127 of the [128][128] K-major tile at oWQ, Kh = k / E into the
// [64][128] K-major tile at oKh (E = e^(G - G_m)).  Every input row is loaded
// before the first store, so that the loads overlap.  Returns the largest
// |G - G_m| seen: with |q|, |k|, |b| <= 8 every factor stays below 8 e^|G|,
// so the fp16 range holds while that value stays below 9.
__device__ __forceinline__ float write_factors_rec(const unsigned char *rq, const unsigned char *rk,
                                                   const float *rb, const float G[8][4],
                                                   unsigned char *oWQ, unsigned char *oKh,
                                                   int warp, int lane) {
    uint2 qr[8], kr[8];
    float4 bv[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int r = 8 * warp + m;
        qr[m] = *reinterpret_cast<const uint2 *>(rq + r * 256 + lane * 8);
        kr[m] = *reinterpret_cast<const uint2 *>(rk + r * 256 + lane * 8);
        bv[m] = *reinterpret_cast<const float4 *>(rb + r * 128 + 4 * lane);
    }
    float gmax = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int r = 8 * warp + m;
        const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qr[m]);
        const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kr[m]);
        const float qf[4] = {__low2float(q2[0]), __high2float(q2[0]), __low2float(q2[1]), __high2float(q2[1])};
        const float kf[4] = {__low2float(k2[0]), __high2float(k2[0]), __low2float(k2[1]), __high2float(k2[1])};
        const float bf[4] = {bv[m].x, bv[m].y, bv[m].z, bv[m].w};
        float qb[4], kc[4], kh[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float e = __expf(G[m][i]), ei = __expf(-G[m][i]);
            qb[i] = qf[i] * e;
            kc[i] = bf[i] * kf[i] * e;
            kh[i] = kf[i] * ei;
            gmax = fmaxf(gmax, fabsf(G[m][i]));
        }
        st_h4(oWQ + sw128_off(r, 4 * lane, 128), kc[0], kc[1], kc[2], kc[3]);
        st_h4(oWQ + sw128_off(r + 64, 4 * lane, 128), qb[0], qb[1], qb[2], qb[3]);
        st_h4(oKh + sw128_off(r, 4 * lane, 64), kh[0], kh[1], kh[2], kh[3]);
    }
    return gmax;
}

}  // namespace tcc
}  // namespace gdn2
