// Pieces shared by the tensor-core forward and backward kernels: the chunk's
// decay frames, raw-tile addressing, fp16 store helpers and the warp-level
// tf32 tile product.
//
// Decay frames ("Gated DeltaNet-2", LIT-802 review, Key takeaways 2: the
// state is normalised by the cumulative decay so that D_t folds into the two
// factors of every rank-one erase).  Per chunk of 64 rows t and key channel c,
// G_t = sum_{i <= t} g_i (rows past the sequence's end hold g = 0), and the
// chunk splits into four 16-row blocks I with s_I = G_{16I-1} (s_0 = 0) and
// e_I = G_{16I+15}:
//   * state side, chunk-start frame, every factor <= 1 for any g <= 0:
//       E_t = e^G_t,  F_t = e^(G_63 - G_t),  gamma = e^G_63;
//   * pair factors e^(G_r - G_j) (r >= j) inside the chunk, which the chunk-
//     start frame would split into e^G_r and e^-G_j (the second unbounded):
//       - r and j in different blocks I > J: e^(G_r - s_I) * chi_IJ *
//         e^(e_J - G_j) with chi_IJ = e^(s_I - e_J); all three are <= 1, so an
//         fp16 operand can only underflow where the pair factor itself is
//         below fp16's resolution;
//       - r and j in the same block: l_r / l_j with l_t = e^(G'_t - G'_m),
//         m the block's row 7, in float32 (tf32 products), where G' sums
//         g' = max(g, -kClampG).  A clamped token lies between r and j only if
//         the true factor is below e^-kClampG, and then the computed one is
//         too; otherwise the two are equal.  Within a block |G' - G'_m| is at
//         most 8 kClampG, inside float32's range.
#pragma once

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {
namespace tcc {
using namespace tc;

// per-token floor of the log-decay inside the same-block pair factors
constexpr float kClampG = 9.0f;
// the kernels carry cumulative decays in log2 units (g log2 e), so that every
// factor is one ex2
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kClampG2 = kClampG * kLog2e;
// A tile is mild when every channel's cumulative log-decay stays within
// kMildG of its value at row 31 and |q|, |k|, |b k| <= kMildX: then every
// factor e^(+-(G - G_31)) x stays within kMildX e^kMildG (1.4e4, inside fp16)
// and no factor that matters falls below fp16's normal range, so one frame
// serves the whole chunk.  Other tiles take the block frames.
constexpr float kMildG = 4.0f;
constexpr float kMildG2 = kMildG * kLog2e;
constexpr float kMildX = 256.0f;

// 2^x (the special-function unit's ex2; flushes denormal results to zero)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float4 f4scale(float4 a, float s) { return make_float4(a.x * s, a.y * s, a.z * s, a.w * s); }
// 4 bf16 values of an 8-byte chunk, widened
__device__ __forceinline__ void ld_bf4(const unsigned char *p, float *x) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
__device__ __forceinline__ void st_h4v(unsigned char *p, const float *x) {
    *reinterpret_cast<uint2 *>(p) = make_uint2(pack_f16(x[0], x[1]), pack_f16(x[2], x[3]));
}

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

// Raw [64 rows][128 channels] tiles as TMA lands them with 128-byte swizzle:
// bf16 tiles as two boxes of 64 channels, float32 tiles as four boxes of 32
// channels, 8 KB per box.  Byte offset of element (t, c).
__host__ __device__ __forceinline__ uint32_t raw16(int t, int c) {
    return (uint32_t)((c >> 6) * 8192) + sw128_off(t, c & 63, 64);
}
__host__ __device__ __forceinline__ uint32_t raw32(int t, int c) {
    return (uint32_t)((c >> 5) * 8192) + sw128_chunk(t, (c & 31) >> 2, 64) + (uint32_t)((c & 3) * 4);
}

// Gate tiles (g, b, w and their gradients) come as float32 or bf16.  GB
// selects bf16: two 64-channel boxes (raw16) instead of four 32-channel ones
// (raw32), half the bytes.  Values are widened to float32 on load and rounded
// once on store.
template <bool GB> __host__ __device__ __forceinline__ uint32_t graw(int t, int c) {
    return GB ? raw16(t, c) : raw32(t, c);
}
template <bool GB> __host__ __device__ constexpr int gate_box_cols() { return GB ? 64 : 32; }
template <bool GB> __host__ __device__ constexpr uint32_t gate_tile_bytes() { return GB ? 16384u : 32768u; }
template <bool GB> __device__ __forceinline__ float gld1(const unsigned char *p) {
    if constexpr (GB) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
    else return *reinterpret_cast<const float *>(p);
}
template <bool GB> __device__ __forceinline__ float2 gld2(const unsigned char *p) {
    if constexpr (GB) return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
    else return *reinterpret_cast<const float2 *>(p);
}
template <bool GB> __device__ __forceinline__ float4 gld4(const unsigned char *p) {
    if constexpr (GB) {
        float x[4];
        ld_bf4(p, x);
        return make_float4(x[0], x[1], x[2], x[3]);
    } else {
        return *reinterpret_cast<const float4 *>(p);
    }
}
template <bool GB> __device__ __forceinline__ void gst1(unsigned char *p, float a) {
    if constexpr (GB) *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(a);
    else *reinterpret_cast<float *>(p) = a;
}
template <bool GB> __device__ __forceinline__ void gst2(unsigned char *p, float a, float b) {
    if constexpr (GB) *reinterpret_cast<uint32_t *>(p) = pack_bf16(a, b);
    else *reinterpret_cast<float2 *>(p) = make_float2(a, b);
}

// Zero rows L..63 of `boxes` consecutive 8 KB boxes of 64 rows x 128 B (the
// rows of a chunk past its sequence's end, which a packed layout fills with
// the next sequence's tokens).  A 128-byte swizzle permutes 16-byte chunks
// within a row only, so whole rows are zeroed the same way in any layout.
// Every thread of the block takes part; the caller supplies the barrier.
__device__ __forceinline__ void zero_rows(unsigned char *base, int boxes, int L, int tid, int nthreads) {
    const int per_box = (64 - L) * 8;
    for (int i = tid; i < boxes * per_box; i += nthreads) {
        const int box = i / per_box, rem = i - box * per_box;
        *reinterpret_cast<uint4 *>(base + box * 8192 + (L + (rem >> 3)) * 128 + (rem & 7) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
}

// Copy rows 0..L-1 of a [64 rows][128 channels] raw tile (8 KB boxes of
// 128-byte swizzled rows: es = 2 bytes per element, two boxes; es = 4, four)
// to global rows dst + r * stride, 128 channels each: the tail chunk of a
// packed sequence, whose TMA store would also write the next sequence's rows.
// Every thread of the block takes part; the caller supplies the barriers.
__device__ __forceinline__ void store_rows(unsigned char *dst, size_t stride, const unsigned char *tile,
                                           int es, int L, int tid, int nthreads) {
    const int per_row = es * 8;  // 16-byte chunks per row
    for (int i = tid; i < L * per_row; i += nthreads) {
        const int r = i / per_row, rem = i - r * per_row, x = rem >> 3, j = rem & 7;
        *reinterpret_cast<uint4 *>(dst + r * stride + x * 128 + j * 16) =
            *reinterpret_cast<const uint4 *>(tile + x * 8192 + sw128_chunk(r, j, 64));
    }
}

// Warp-level tf32 tile product D = A B + D (m16n8k8, f32 accumulate).
// Fragments (g = lane / 4, t = lane % 4): a0 (g, t), a1 (g + 8, t),
// a2 (g, t + 4), a3 (g + 8, t + 4); b0 (k = t, n = g), b1 (k = t + 4, n = g);
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
// Warp-level fp16 tile product D = A B + D (m16n8k16, f32 accumulate).
// Fragments: a0..a3 as f16 pairs: a0 (g, 2t..2t+1), a1 (g + 8, 2t..), a2 (g,
// 2t + 8..), a3 (g + 8, 2t + 8..); b0 (k = 2t..2t+1, n = g), b1 (k = 2t + 8..,
// n = g); c as for the tf32 product.
__device__ __forceinline__ void mma_f16_16x8x16(float *c, const uint32_t *a, const uint32_t *b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// ldmatrix: four 8x8 b16 matrices from shared memory (rows addressed by
// lanes 8i..8i+7 for matrix i), plain or transposed
__device__ __forceinline__ void ldsm_x4(uint32_t *r, uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t *r, uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr));
}
// two 8x8 b16 matrices, transposed (rows addressed by lanes 0..15)
__device__ __forceinline__ void ldsm_x2_t(uint32_t *r, uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(saddr));
}
// (x.lo s, x.hi s) for an f16 pair x, multiplied in float32 and rounded once
__device__ __forceinline__ uint32_t h2scale(uint32_t x, float s) {
    const float2 f = __half22float2(*reinterpret_cast<__half2 *>(&x));
    return pack_f16(f.x * s, f.y * s);
}

}  // namespace tcc
}  // namespace gdn2
