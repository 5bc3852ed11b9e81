// Shared device helpers, sizes and the workspace layout of libgdn2.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn2.h"

namespace gdn2 {

constexpr int kMaxD = 128;     // largest d_k / d_v
constexpr int kMaxChunk = 64;  // largest chunk

struct Dims {
    int B, T, H, dk, dv, C, NC;
    int gb;  // gate tensors g, b, w and dg, db, dw in bf16 (tensor-core path), else float32
    // gate logits (tensor-core path and decode): bit 0 set: g, b, w arrive as
    // pre-activation logits and are activated on load (GateAct below), and
    // dg, db, dw leave as gradients of the logits; bit 1: b = 2 sigmoid(x)
    int act;
    // Packed variable-length sequences (tensor-core path): N sequences whose
    // tokens lie at rows cu[n] .. cu[n + 1] - 1 of a B = 1 batch, cu (device,
    // N + 1 entries) as given by the caller, co (workspace, N + 1 entries) the
    // first chunk of each sequence in chunk order; NC then bounds the total
    // chunks.  cu == nullptr: B rows of T tokens each.
    const int *cu, *co;
    int N;
};

// One sequence as the kernels see it: its first row in the T axis of its
// batch row `brow`, its length, its chunks and the first of them (global).
struct Seq {
    int bos, len, nc, c0, brow;
};
__device__ __forceinline__ Seq seq_of(const Dims &d, int n) {
    if (!d.cu) return Seq{0, d.T, d.NC, n * d.NC, n};
    const int bos = __ldg(d.cu + n), c0 = __ldg(d.co + n);
    return Seq{bos, __ldg(d.cu + n + 1) - bos, __ldg(d.co + n + 1) - c0, c0, 0};
}
// sequences (rows of the batch, or packed sequences)
__host__ __device__ __forceinline__ int num_seqs(const Dims &d) { return d.N > 0 ? d.N : d.B; }
// chunk tiles of the call, in the order (sequence, head, chunk)
__device__ __forceinline__ int total_tiles(const Dims &d) {
    return d.cu ? d.H * __ldg(d.co + d.N) : d.B * d.H * d.NC;
}
// workspace tile index of chunk c of head h of sequence s (B rows: (b H + h) NC + c)
__device__ __forceinline__ int tile_of(const Dims &d, const Seq &s, int h, int c) {
    return s.c0 * d.H + h * s.nc + c;
}
// the sequence, head and chunk of tile `it`
__device__ __forceinline__ void tile_decode(const Dims &d, int it, int &n, int &h, int &c) {
    if (!d.cu) {
        c = it % d.NC;
        const int bhi = it / d.NC;
        h = bhi % d.H;
        n = bhi / d.H;
        return;
    }
    // the last sequence whose first tile is at or before it (it has chunks:
    // the next sequence, or the end, starts after it)
    int lo = 0, hi = d.N;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(d.co + mid) * d.H <= it) lo = mid;
        else hi = mid;
    }
    n = lo;
    const int c0 = __ldg(d.co + lo), nc = __ldg(d.co + lo + 1) - c0, rem = it - c0 * d.H;
    h = rem / nc;
    c = rem - h * nc;
}

// ---- gate activations ("Gated DeltaNet-2", LIT-802 review, Key takeaways 1:
// the erase and write gates are sigmoid outputs, 2 sigmoid for erase
// eigenvalues in [-1, 1]; the decay a log-sigmoid) for calls that pass logits
__device__ __forceinline__ float sigmoid_act(float x) { return 1.f / (1.f + __expf(-x)); }
// log(sigmoid(x)) = min(x, 0) - log(1 + e^-|x|), without overflow
__device__ __forceinline__ float logsigmoid_act(float x) { return fminf(x, 0.f) - log1pf(__expf(-fabsf(x))); }
struct GateAct {
    bool on;      // logits in, logit gradients out
    float bscale; // 1 or 2
    __device__ __forceinline__ float g(float x) const { return on ? logsigmoid_act(x) : x; }
    __device__ __forceinline__ float b(float x) const { return on ? bscale * sigmoid_act(x) : x; }
    __device__ __forceinline__ float w(float x) const { return on ? sigmoid_act(x) : x; }
    // d(activation)/dx at logit x: g' = sigmoid(-x), b' = s sigma (1 - sigma), w' = sigma (1 - sigma)
    __device__ __forceinline__ float dg(float x) const { return on ? sigmoid_act(-x) : 1.f; }
    __device__ __forceinline__ float db(float x) const {
        if (!on) return 1.f;
        const float s = sigmoid_act(x);
        return bscale * s * (1.f - s);
    }
    __device__ __forceinline__ float dw(float x) const {
        if (!on) return 1.f;
        const float s = sigmoid_act(x);
        return s * (1.f - s);
    }
};
__device__ __forceinline__ GateAct gate_act(int act) { return GateAct{(act & 1) != 0, (act & 2) ? 2.f : 1.f}; }
__device__ __forceinline__ float4 act_g4(const GateAct &a, float4 v) {
    return a.on ? make_float4(a.g(v.x), a.g(v.y), a.g(v.z), a.g(v.w)) : v;
}
__device__ __forceinline__ float4 act_b4(const GateAct &a, float4 v) {
    return a.on ? make_float4(a.b(v.x), a.b(v.y), a.b(v.z), a.b(v.w)) : v;
}
__device__ __forceinline__ float4 act_w4(const GateAct &a, float4 v) {
    return a.on ? make_float4(a.w(v.x), a.w(v.y), a.w(v.z), a.w(v.w)) : v;
}
__device__ __forceinline__ float2 act_g2(const GateAct &a, float2 v) { return a.on ? make_float2(a.g(v.x), a.g(v.y)) : v; }
__device__ __forceinline__ float2 act_b2(const GateAct &a, float2 v) { return a.on ? make_float2(a.b(v.x), a.b(v.y)) : v; }
__device__ __forceinline__ float2 act_w2(const GateAct &a, float2 v) { return a.on ? make_float2(a.w(v.x), a.w(v.y)) : v; }

// ---- element access in the io type (float or bf16), computing in float
template <typename E> __device__ __forceinline__ float ldx(const E *p, size_t i);
template <> __device__ __forceinline__ float ldx<float>(const float *p, size_t i) { return p[i]; }
template <> __device__ __forceinline__ float ldx<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
template <typename E> __device__ __forceinline__ void stx(E *p, size_t i, float x);
template <> __device__ __forceinline__ void stx<float>(float *p, size_t i, float x) { p[i] = x; }
template <> __device__ __forceinline__ void stx<__nv_bfloat16>(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// offset of element (bb, t, h, 0) in a [B, T, H, width] tensor
__device__ __forceinline__ size_t tok(const Dims &d, int bb, int t, int h, int width) {
    return (((size_t)bb * d.T + t) * d.H + h) * (size_t)width;
}
// offset of the (bb, h) state in a [B, H, dk, dv] tensor
__device__ __forceinline__ size_t st_off(const Dims &d, int bb, int h) {
    return ((size_t)bb * d.H + h) * (size_t)d.dk * d.dv;
}
// index of chunk tile (bb, h, c)
__device__ __forceinline__ size_t tile(const Dims &d, int bb, int h, int c) {
    return ((size_t)bb * d.H + h) * d.NC + c;
}

// ---- segment-parallel state passes.  A long sequence with few (b, h) leaves
// most SMs idle in the sequential state kernels; its chunks then split into P
// segments, and S_end = M_s S_begin + N_s over segment s (M_s the product of
// the chunks' transitions, N_s the state reached from zero):
//   phase 1: segment 0 for real; for every middle segment s = 1 .. P-2, N_s
//            (a run from a zero state) and M_s (a run from the identity with no
//            input), all in parallel;
//   link:    entries S_{s+1} = M_s S_s + N_s, s = 1 .. P-2 (a short scan);
//   phase 2: segments 1 .. P-1 for real from their entries, in parallel.
// The backward runs the same way in reverse with M_s^T (dS_entry = M_s^T
// dS_exit + R_s, R_s the gradient reached from a zero exit gradient).
// buf holds [bh][P][3][128 x 128] float32: entry (kind 0), zero-run result
// (kind 1) and map M_s (kind 2), rows of 128 like a state.
struct SegPass {
    int P;      // segments per sequence (1: one run over the whole sequence)
    int phase;  // 0: the whole sequence; 1, 2: the passes above
    float *buf;
};
enum SegKind { SEG_ENTRY = 0, SEG_ZERO = 1, SEG_MAP = 2 };
__host__ __device__ __forceinline__ float *seg_buf(const SegPass &sp, size_t bh, int s, int kind) {
    return sp.buf + ((bh * sp.P + s) * 3 + kind) * (size_t)(128 * 128);
}
// chunk range of segment s (P segments over nc chunks, every one non-empty)
__host__ __device__ __forceinline__ int seg_len(int nc, int P) { return (nc + P - 1) / P; }
// the largest useful P: every segment non-empty, at least 4 chunks each, and
// the first pass (2 + 4 (P - 2) CTAs per (b, h)) within one wave of 148 SMs
inline int seg_count(int B, int H, int nc) {
    int best = 1;
    for (int P = 3; P <= 8; ++P) {
        const int L = seg_len(nc, P);
        if (L < 4 || (P - 1) * L >= nc) break;
        if ((long long)(2 + 4 * (P - 2)) * B * H > 148) break;
        best = P;
    }
    return best;
}

// ---- the device status word (GDN2_OK or the first error recorded); kernels
// that can give up on a bounded wait receive its device address.
__device__ __forceinline__ void record_status(unsigned int *status, unsigned int s) {
    atomicCAS(status, 0u, s);
}

// ---- workspace of the CUDA-core (fp32) path: per-chunk float32 tiles
struct SimtWs {
    size_t gam;     // [B,H,NC,C,dk]  in-chunk cumulative log-decay
    size_t Tinv;    // [B,H,NC,C,C]   (I + A)^-1
    size_t P;       // [B,H,NC,C,C]   lower-incl(Qb Kh^T)
    size_t W;       // [B,H,NC,C,dk]  T Kc
    size_t Up;      // [B,H,NC,C,dv]  T U
    size_t Delta;   // [B,H,NC,C,dv]  U' - W S_c
    size_t Sc;      // [B,H,NC,dk,dv] chunk-entry states
    size_t fwd_end;
    size_t dSn;     // [B,H,NC,dk,dv] dL/dS at the chunk's exit
    size_t dDelta;  // [B,H,NC,C,dv]
    size_t dP;      // [B,H,NC,C,C]   lower-incl(dO Delta^T)
    size_t dA;      // [B,H,NC,C,C]   -strictly-lower(dU Delta^T)
    size_t X1;      // [B,H,NC,C,dk]  dO S_c^T
    size_t X2;      // [B,H,NC,C,dk]  dU S_c^T
    size_t X3;      // [B,H,NC,C,dk]  Delta dSn^T
    size_t X4;      // [B,H,NC,dk]    rowsum(dSn . S_c)
    size_t bwd_end;
};

// ---- host-side launch accounting: every launch site brackets its launch
// with launch_begin / launch_end (kernel kind ids below)
enum KernelKind {
    K_SIMT_PREP = 0, K_SIMT_STATE_FWD, K_SIMT_OUT, K_SIMT_STATE_BWD, K_SIMT_BWD_A, K_SIMT_BWD_B,
    K_DECODE, K_TC_PREP, K_TC_FWD, K_TC_BWD_STATE, K_TC_BWD_GRAD, K_SEQ_TABLE,
    K_PERMUTE_STATE, K_SEG_LINK, K_KINDS
};
void launch_begin(int kind, cudaStream_t s);
void launch_end(int kind, cudaStream_t s);

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// number of SMs of the current device (grid size of the persistent kernels)
inline int sm_count() {
    static int cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
        cached[dev] = n;
    }
    return cached[dev];
}

inline SimtWs simt_ws_layout(const Dims &d) {
    SimtWs w;
    size_t tiles = (size_t)d.B * d.H * d.NC;
    size_t o = 0;
    auto take = [&](size_t floats) { size_t at = o; o = align256(o + floats * sizeof(float)); return at; };
    w.gam = take(tiles * d.C * d.dk);
    w.Tinv = take(tiles * d.C * d.C);
    w.P = take(tiles * d.C * d.C);
    w.W = take(tiles * d.C * d.dk);
    w.Up = take(tiles * d.C * d.dv);
    w.Delta = take(tiles * d.C * d.dv);
    w.Sc = take(tiles * (size_t)d.dk * d.dv);
    w.fwd_end = o;
    w.dSn = take(tiles * (size_t)d.dk * d.dv);
    w.dDelta = take(tiles * d.C * d.dv);
    w.dP = take(tiles * d.C * d.C);
    w.dA = take(tiles * d.C * d.C);
    w.X1 = take(tiles * d.C * d.dk);
    w.X2 = take(tiles * d.C * d.dk);
    w.X3 = take(tiles * d.C * d.dk);
    w.X4 = take(tiles * d.dk);
    w.bwd_end = o;
    return w;
}

// ---- workspace of the tensor-core path (d_k = d_v = 128, chunk 64): fp16
// tiles in their 128-byte swizzled shared-memory layout, so that they move
// with plain bulk copies.  Offsets in bytes; bh = b * H + h.
//   rec   [bh][NC]        66560 B  the chunk's record, written by the chunk-
//                                  parallel prep kernel (layout REC_* below)
//   ckS   [bh][NC][2 halves]  16 KB  chunk-entry states in the chunk's frame, s S_c
//                                  (a copy of the forward's fp16 operand)
//   ckD   [bh][NC][2]          8 KB  Delta (columns of one d_v half)
//   ckdS  [bh][NC][2]         16 KB  dL/dS_{c+1}, the state gradient leaving chunk c
//   ckndU [bh][NC][2]          8 KB  -dU
// A forward that is not followed by a backward needs `rec` only.
//
// Chunk record: operands in the chunk's frame (fp16, 128-byte swizzled; see
// tc.cuh for the layouts and tc_common.cuh for the frames).  With the frame
// factor s (per key channel): s = 1 (the chunk-start frame) or, for a mild
// chunk, s = e^G_31 (the frame of row 31):
//   REC_WQ   [-W; Qb] as one [128 rows][128 key] K-major tile: rows 0..63
//            -W = -T Kc (Kc = b.k.e^G / s), rows 64..127 Qb = q.e^G / s (32 KB)
//   REC_KH   Kx: Kb = k.e^(G_63 - G) (s = 1), or Kh = k.e^(G_31 - G) (mild)
//            [64 pos][128 key] K-major (16 KB)
//   REC_T    T = (I + A)^-1             [64][64] K-major (8 KB)
//   REC_P    P                          [64][64] K-major (8 KB)
//   REC_FAC  gamma = e^G_63 [128] f32, then s [128] f32, stored as -1 where
//            s = 1 (a negative value marks the chunk-start frame)
// So that every consumer can handle both frames with per-channel scales:
//   S_next = gamma S + r Kx^T Delta,  r = 1 (s = 1) or gamma / s (mild);
//   the operand state is s S, the operand state gradient r dS'.
constexpr uint32_t REC_WQ = 0, REC_KH = 32768, REC_T = 49152, REC_P = 57344, REC_FAC = 65536,
                   REC_BYTES = 66560;
struct TcWs {
    size_t rec, rec_end, ckS, ckD, seg, fwd_end, ckdS, ckndU, bwd_end;
    int P;  // segments per sequence of the state passes (1: none)
};
inline TcWs tc_ws_layout(const Dims &d) {
    const size_t bh = (size_t)d.B * d.H, nc = (size_t)d.NC;
    TcWs w;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
    w.rec = take(bh * nc * REC_BYTES);
    w.rec_end = o;
    w.ckS = take(bh * nc * 2 * 16384);
    w.ckD = take(bh * nc * 2 * 8192);
    w.P = d.N > 0 ? 1 : seg_count(d.B, d.H, d.NC);
    w.seg = take(w.P > 1 ? bh * w.P * 3 * 128 * 128 * sizeof(float) : 0);
    w.fwd_end = o;
    w.ckdS = take(bh * nc * 2 * 16384);
    w.ckndU = take(bh * nc * 2 * 8192);
    w.bwd_end = o;
    return w;
}

template <typename T> __host__ __device__ __forceinline__ T *at(void *base, size_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(base) + off);
}

}  // namespace gdn2
