// Single-token recurrent decode of Gated Delta Rule-2.
//
// "Gated DeltaNet-2" abstract (linear-time sequence mixing with constant-memory
// decoding) and the update of the LIT-802 review, Key takeaways 1:
//   S' = diag(e^g) S;  delta = w.v - S'^T (b.k);  S <- S' + k delta^T;
//   o = S^T q = S'^T q + (k.q) delta.
// One block per (sequence, head).  The float32 state is read once into
// registers (each warp owns d_k/8 rows, each lane d_v/32 adjacent columns,
// so every warp load is one contiguous row segment), both value-axis
// reductions are formed from those registers, and the state is written back
// once: 2 * d_k * d_v * 4 bytes of state traffic per (sequence, head).

#include "common.cuh"

namespace gdn2 {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

template <int CL> __device__ __forceinline__ void vload(const float *p, float *x) {
    if constexpr (CL == 4) { float4 t = *reinterpret_cast<const float4 *>(p); x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w; }
    else if constexpr (CL == 2) { float2 t = *reinterpret_cast<const float2 *>(p); x[0] = t.x; x[1] = t.y; }
    else { x[0] = *p; }
}
template <int CL> __device__ __forceinline__ void vstore(float *p, const float *x) {
    if constexpr (CL == 4) { *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]); }
    else if constexpr (CL == 2) { *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]); }
    else { *p = x[0]; }
}

// E: the io type of q, k, v, o; GE: the gate type of g, b, w (float or bf16);
// ACT: gate logits (GateAct)
template <typename E, typename GE, bool ACT, int DK, int DV>
__global__ void __launch_bounds__(kDecThreads)
decode_step_kernel(const E *__restrict__ q, const E *__restrict__ k, const E *__restrict__ v,
                   const GE *__restrict__ g, const GE *__restrict__ b,
                   const GE *__restrict__ w, float *__restrict__ S, E *__restrict__ o, int H, int G, int act) {
    const GateAct ga = ACT ? gate_act(act) : GateAct{false, 1.f};  // logits in: activated on load
    constexpr int RW = DK / kDecWarps;  // rows per warp
    constexpr int CL = DV / 32;         // columns per lane
    __shared__ float sk[DK], sbk[DK], sq[DK], sa[DK], su[DV], sdelta[DV];
    __shared__ float red_r[kDecWarps][DV], red_p[kDecWarps][DV];
    __shared__ float s_kq;
    // block = (sequence n, value head hv); value head hv reads key head hv / G
    const int HV = H * G, hv = blockIdx.x % HV, n = blockIdx.x / HV, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const size_t hk = ((size_t)n * H + hv / G) * DK, hvo = ((size_t)n * HV + hv) * DV;
    float *Sp = S + ((size_t)n * HV + hv) * DK * DV;

    // issue the state loads first: they are the bulk of the traffic
    float x[RW][CL];
#pragma unroll
    for (int m = 0; m < RW; ++m) vload<CL>(Sp + (size_t)(warp * RW + m) * DV + lane * CL, x[m]);

    for (int i = tid; i < DK; i += kDecThreads) {
        float kv = ldx(k, hk + i), qv = ldx(q, hk + i);
        sk[i] = kv; sq[i] = qv; sbk[i] = ga.b(ldx(b, hk + i)) * kv; sa[i] = __expf(ga.g(ldx(g, hk + i)));
    }
    for (int j = tid; j < DV; j += kDecThreads) su[j] = ga.w(ldx(w, hvo + j)) * ldx(v, hvo + j);
    if (warp == 0) {
        float acc = 0.f;
        for (int i = lane; i < DK; i += 32) acc += ldx(k, hk + i) * ldx(q, hk + i);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) s_kq = acc;
    }
    __syncthreads();

    float pr[CL], pp[CL];
#pragma unroll
    for (int n2 = 0; n2 < CL; ++n2) { pr[n2] = 0.f; pp[n2] = 0.f; }
#pragma unroll
    for (int m = 0; m < RW; ++m) {
        const int i = warp * RW + m;
        const float a = sa[i], bk = sbk[i], qi = sq[i];
#pragma unroll
        for (int n2 = 0; n2 < CL; ++n2) {
            x[m][n2] *= a;
            pr[n2] += x[m][n2] * bk;
            pp[n2] += x[m][n2] * qi;
        }
    }
#pragma unroll
    for (int n2 = 0; n2 < CL; ++n2) {
        red_r[warp][lane * CL + n2] = pr[n2];
        red_p[warp][lane * CL + n2] = pp[n2];
    }
    __syncthreads();
    for (int j = tid; j < DV; j += kDecThreads) {
        float r = 0.f, p = 0.f;
#pragma unroll
        for (int wi = 0; wi < kDecWarps; ++wi) { r += red_r[wi][j]; p += red_p[wi][j]; }
        float dlt = su[j] - r;
        sdelta[j] = dlt;
        stx(o, hvo + j, p + s_kq * dlt);
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < RW; ++m) {
        const int i = warp * RW + m;
        const float ki = sk[i];
#pragma unroll
        for (int n2 = 0; n2 < CL; ++n2) x[m][n2] += ki * sdelta[lane * CL + n2];
        vstore<CL>(Sp + (size_t)i * DV + lane * CL, x[m]);
    }
}

template <typename E, typename GE, bool ACT, int DK, int DV>
static cudaError_t launch_dec(const void *q, const void *k, const void *v, const void *g,
                              const void *b, const void *w, float *S, void *o, int N, int H, int G,
                              int act, cudaStream_t s) {
    launch_begin(K_DECODE, s);
    decode_step_kernel<E, GE, ACT, DK, DV><<<(unsigned)N * (unsigned)(H * G), kDecThreads, 0, s>>>(
        (const E *)q, (const E *)k, (const E *)v, (const GE *)g, (const GE *)b, (const GE *)w, S,
        (E *)o, H, G, act);
    launch_end(K_DECODE, s);
    return cudaGetLastError();
}

template <typename E, typename GE, bool ACT>
static cudaError_t dispatch_dec(const void *q, const void *k, const void *v, const void *g,
                                const void *b, const void *w, float *S, void *o, int N, int H, int G,
                                int act, int dk, int dv, cudaStream_t s) {
#define GDN2_DEC(DK_, DV_) \
    if (dk == DK_ && dv == DV_) return launch_dec<E, GE, ACT, DK_, DV_>(q, k, v, g, b, w, S, o, N, H, G, act, s);
    GDN2_DEC(32, 32) GDN2_DEC(32, 64) GDN2_DEC(32, 128)
    GDN2_DEC(64, 32) GDN2_DEC(64, 64) GDN2_DEC(64, 128)
    GDN2_DEC(128, 32) GDN2_DEC(128, 64) GDN2_DEC(128, 128)
#undef GDN2_DEC
    return cudaErrorInvalidValue;
}

template <bool ACT>
static cudaError_t decode_types(const void *q, const void *k, const void *v, const void *g, const void *b,
                                const void *w, float *S, void *o, int N, int H, int G, int dk, int dv,
                                gdn2_io io, gdn2_io gate_io, int act, cudaStream_t s) {
    using BF = __nv_bfloat16;
    if (io == GDN2_IO_BF16)
        return gate_io == GDN2_IO_BF16
                   ? dispatch_dec<BF, BF, ACT>(q, k, v, g, b, w, S, o, N, H, G, act, dk, dv, s)
                   : dispatch_dec<BF, float, ACT>(q, k, v, g, b, w, S, o, N, H, G, act, dk, dv, s);
    return gate_io == GDN2_IO_BF16 ? dispatch_dec<float, BF, ACT>(q, k, v, g, b, w, S, o, N, H, G, act, dk, dv, s)
                                   : dispatch_dec<float, float, ACT>(q, k, v, g, b, w, S, o, N, H, G, act, dk, dv, s);
}

cudaError_t decode_launch(const void *q, const void *k, const void *v, const void *g,
                          const void *b, const void *w, float *S, void *o, int N, int H, int G,
                          int dk, int dv, gdn2_io io, gdn2_io gate_io, int act, cudaStream_t s) {
    return act ? decode_types<true>(q, k, v, g, b, w, S, o, N, H, G, dk, dv, io, gate_io, act, s)
               : decode_types<false>(q, k, v, g, b, w, S, o, N, H, G, dk, dv, io, gate_io, act, s);
}

}  // namespace gdn2
