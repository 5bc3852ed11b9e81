// Chunkwise forward of Gated Delta Rule-2 on CUDA cores in float32.
//
// "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
// (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4, Apps. A-B): within a
// chunk the state is normalised by the cumulative decay, so the recurrence
// becomes (I + A) Delta = U - Kc S with one unit-lower-triangular system shared
// by the erase side (W = T Kc) and the write side (U' = T U); only the state is
// carried between chunks.  Per chunk of L tokens entering with state S:
//   G = in-chunk inclusive cumsum of g (per key channel)
//   A[r][j] = sum_i b[r,i] k[r,i] k[j,i] e^(G[r,i]-G[j,i])      (j < r)
//   T = (I + A)^-1,  W = T Kc,  U' = T (w.v),  Kc = b.k.e^G
//   Delta = U' - W S
//   P[r][j] = sum_i q[r,i] k[j,i] e^(G[r,i]-G[j,i])             (j <= r)
//   O = (q.e^G) S + P Delta
//   S_next = diag(e^G_L) S + Kbar^T Delta,  Kbar = k.e^(G_L - G)
// This path forms every pairwise decay factor e^(G[r,i]-G[j,i]) directly,
// so it holds for any log-decay g <= 0 without overflow: it is the float32
// path (GDN2_IO_F32) and the path for every supported size.
//
// Three kernels: chunk_prep (all chunks in parallel), state_fwd (sequential
// over chunks, parallel over (b, h, 32-column slices of d_v)), out_fwd (all
// chunks in parallel).

#include "common.cuh"

namespace gdn2 {

constexpr int kThreads = 256;
constexpr int kSlice = 32;  // d_v columns per state_fwd / state_bwd block

// ------------------------------------------------------------- chunk_prep
template <typename E>
__global__ void __launch_bounds__(kThreads)
simt_chunk_prep(const E *__restrict__ q, const E *__restrict__ k, const E *__restrict__ v,
                const float *__restrict__ g, const float *__restrict__ b,
                const float *__restrict__ w, void *ws, SimtWs lay, Dims d) {
    extern __shared__ float sm[];
    const int C = d.C, dk = d.dk, dv = d.dv, LD = d.C + 1;
    float *sG = sm;               // [dk][LD]  channel-major
    float *sK = sG + dk * LD;     // [dk][LD]
    float *sX = sK + dk * LD;     // [dk][LD]  b, then Kc, then q
    float *sA = sX + dk * LD;     // [C][C]
    float *sT = sA + C * C;       // [C][C]
    float *sU = sT + C * C;       // [C][dv]
    const int c = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, tid = threadIdx.x;
    const int c0 = c * C, L = min(C, d.T - c0);
    const size_t ti = tile(d, bb, h, c);

    for (int idx = tid; idx < C * dk; idx += kThreads) {
        int r = idx / dk, i = idx % dk;
        float gv = 0.f, kv = 0.f, bv = 0.f;
        if (r < L) {
            size_t o = tok(d, bb, c0 + r, h, dk) + i;
            gv = g[o]; kv = ldx(k, o); bv = b[o];
        }
        sG[i * LD + r] = gv; sK[i * LD + r] = kv; sX[i * LD + r] = bv;
    }
    __syncthreads();
    for (int i = tid; i < dk; i += kThreads) {
        float acc = 0.f;
        for (int r = 0; r < L; ++r) { acc += sG[i * LD + r]; sG[i * LD + r] = acc; }
    }
    __syncthreads();
    float *gam = at<float>(ws, lay.gam) + ti * C * dk;
    for (int idx = tid; idx < L * dk; idx += kThreads) {
        int r = idx / dk, i = idx % dk;
        gam[idx] = sG[i * LD + r];
    }
    // A, strictly lower
    for (int p = tid; p < C * C; p += kThreads) {
        int r = p / C, j = p % C;
        float acc = 0.f;
        if (j < r && r < L) {
            for (int i = 0; i < dk; ++i)
                acc += sX[i * LD + r] * sK[i * LD + r] * sK[i * LD + j] *
                       __expf(sG[i * LD + r] - sG[i * LD + j]);
        }
        sA[p] = acc;
    }
    __syncthreads();
    // T = (I + A)^-1, row by row: T[i][c] = -sum_{j=c}^{i-1} A[i][j] T[j][c]
    for (int p = tid; p < C * C; p += kThreads) sT[p] = (p / C == p % C) ? 1.f : 0.f;
    __syncthreads();
    for (int i = 1; i < L; ++i) {
        for (int cc = tid; cc < i; cc += kThreads) {
            float acc = 0.f;
            for (int j = cc; j < i; ++j) acc += sA[i * C + j] * sT[j * C + cc];
            sT[i * C + cc] = -acc;
        }
        __syncthreads();
    }
    float *Tg = at<float>(ws, lay.Tinv) + ti * C * C;
    for (int p = tid; p < C * C; p += kThreads) Tg[p] = sT[p];
    // Kc = b.k.e^G in place of b
    for (int idx = tid; idx < dk * L; idx += kThreads) {
        int i = idx / L, r = idx % L;
        sX[i * LD + r] = sX[i * LD + r] * sK[i * LD + r] * __expf(sG[i * LD + r]);
    }
    for (int idx = tid; idx < C * dv; idx += kThreads) {
        int r = idx / dv, j = idx % dv;
        float u = 0.f;
        if (r < L) {
            size_t o = tok(d, bb, c0 + r, h, dv) + j;
            u = w[o] * ldx(v, o);
        }
        sU[idx] = u;
    }
    __syncthreads();
    float *Wg = at<float>(ws, lay.W) + ti * C * dk;
    for (int idx = tid; idx < L * dk; idx += kThreads) {
        int r = idx / dk, i = idx % dk;
        float acc = 0.f;
        for (int j = 0; j <= r; ++j) acc += sT[r * C + j] * sX[i * LD + j];
        Wg[idx] = acc;
    }
    float *Ug = at<float>(ws, lay.Up) + ti * C * dv;
    for (int idx = tid; idx < L * dv; idx += kThreads) {
        int r = idx / dv, j = idx % dv;
        float acc = 0.f;
        for (int s = 0; s <= r; ++s) acc += sT[r * C + s] * sU[s * dv + j];
        Ug[idx] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < C * dk; idx += kThreads) {
        int r = idx / dk, i = idx % dk;
        sX[i * LD + r] = r < L ? ldx(q, tok(d, bb, c0 + r, h, dk) + i) : 0.f;
    }
    __syncthreads();
    float *Pg = at<float>(ws, lay.P) + ti * C * C;
    for (int p = tid; p < C * C; p += kThreads) {
        int r = p / C, j = p % C;
        float acc = 0.f;
        if (j <= r && r < L) {
            for (int i = 0; i < dk; ++i)
                acc += sX[i * LD + r] * sK[i * LD + j] * __expf(sG[i * LD + r] - sG[i * LD + j]);
        }
        Pg[p] = acc;
    }
}

// -------------------------------------------------------------- state_fwd
__global__ void __launch_bounds__(kThreads)
simt_state_fwd_kernel(const float *__restrict__ S0, float *__restrict__ ST, const void *kptr,
                      int k_is_bf16, void *ws, SimtWs lay, Dims d) {
    extern __shared__ float sm[];
    const int C = d.C, dk = d.dk, dv = d.dv;
    float *sS = sm;              // [dk][kSlice]
    float *sW = sS + dk * kSlice;  // [C][dk]
    float *sKb = sW + C * dk;      // [C][dk]  Kbar
    float *sD = sKb + C * dk;      // [C][kSlice]
    float *sGL = sD + C * kSlice;  // [dk]      e^G_L
    const int v0 = blockIdx.x * kSlice, h = blockIdx.y, bb = blockIdx.z, tid = threadIdx.x;
    const size_t so = st_off(d, bb, h);
    for (int idx = tid; idx < dk * kSlice; idx += kThreads) {
        int i = idx / kSlice, j = idx % kSlice;
        sS[idx] = S0 ? S0[so + (size_t)i * dv + v0 + j] : 0.f;
    }
    __syncthreads();
    for (int c = 0; c < d.NC; ++c) {
        const int c0 = c * C, L = min(C, d.T - c0);
        const size_t ti = tile(d, bb, h, c);
        float *Sc = at<float>(ws, lay.Sc) + ti * dk * dv;
        for (int idx = tid; idx < dk * kSlice; idx += kThreads) {
            int i = idx / kSlice, j = idx % kSlice;
            Sc[(size_t)i * dv + v0 + j] = sS[idx];
        }
        const float *Wg = at<float>(ws, lay.W) + ti * C * dk;
        const float *gam = at<float>(ws, lay.gam) + ti * C * dk;
        for (int idx = tid; idx < L * dk; idx += kThreads) {
            int r = idx / dk, i = idx % dk;
            sW[idx] = Wg[idx];
            float kv = k_is_bf16 ? __bfloat162float(((const __nv_bfloat16 *)kptr)[tok(d, bb, c0 + r, h, dk) + i])
                                 : ((const float *)kptr)[tok(d, bb, c0 + r, h, dk) + i];
            sKb[idx] = kv * __expf(gam[(size_t)(L - 1) * dk + i] - gam[idx]);
        }
        for (int i = tid; i < dk; i += kThreads) sGL[i] = __expf(gam[(size_t)(L - 1) * dk + i]);
        __syncthreads();
        const float *Ug = at<float>(ws, lay.Up) + ti * C * dv;
        float *Dg = at<float>(ws, lay.Delta) + ti * C * dv;
        for (int idx = tid; idx < L * kSlice; idx += kThreads) {
            int r = idx / kSlice, j = idx % kSlice;
            float acc = Ug[(size_t)r * dv + v0 + j];
            for (int i = 0; i < dk; ++i) acc -= sW[r * dk + i] * sS[i * kSlice + j];
            sD[idx] = acc;
            Dg[(size_t)r * dv + v0 + j] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < dk * kSlice; idx += kThreads) {
            int i = idx / kSlice, j = idx % kSlice;
            float acc = sGL[i] * sS[idx];
            for (int r = 0; r < L; ++r) acc += sKb[r * dk + i] * sD[r * kSlice + j];
            sS[idx] = acc;
        }
        __syncthreads();
    }
    if (ST)
        for (int idx = tid; idx < dk * kSlice; idx += kThreads) {
            int i = idx / kSlice, j = idx % kSlice;
            ST[so + (size_t)i * dv + v0 + j] = sS[idx];
        }
}

// ---------------------------------------------------------------- out_fwd
template <typename E>
__global__ void __launch_bounds__(kThreads)
simt_out_fwd(const E *__restrict__ q, E *__restrict__ o, void *ws, SimtWs lay, Dims d) {
    extern __shared__ float sm[];
    const int C = d.C, dk = d.dk, dv = d.dv;
    float *sQ = sm;              // [C][dk] q.e^G
    float *sS = sQ + C * dk;     // [dk][dv]
    float *sP = sS + dk * dv;    // [C][C]
    float *sD = sP + C * C;      // [C][dv]
    const int c = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, tid = threadIdx.x;
    const int c0 = c * C, L = min(C, d.T - c0);
    const size_t ti = tile(d, bb, h, c);
    const float *gam = at<float>(ws, lay.gam) + ti * C * dk;
    for (int idx = tid; idx < L * dk; idx += kThreads) {
        int r = idx / dk, i = idx % dk;
        sQ[idx] = ldx(q, tok(d, bb, c0 + r, h, dk) + i) * __expf(gam[idx]);
    }
    const float *Sc = at<float>(ws, lay.Sc) + ti * dk * dv;
    for (int idx = tid; idx < dk * dv; idx += kThreads) sS[idx] = Sc[idx];
    const float *Pg = at<float>(ws, lay.P) + ti * C * C;
    for (int idx = tid; idx < C * C; idx += kThreads) sP[idx] = Pg[idx];
    const float *Dg = at<float>(ws, lay.Delta) + ti * C * dv;
    for (int idx = tid; idx < L * dv; idx += kThreads) sD[idx] = Dg[idx];
    __syncthreads();
    for (int idx = tid; idx < L * dv; idx += kThreads) {
        int r = idx / dv, j = idx % dv;
        float acc = 0.f;
        for (int i = 0; i < dk; ++i) acc += sQ[r * dk + i] * sS[i * dv + j];
        for (int s = 0; s <= r; ++s) acc += sP[r * C + s] * sD[s * dv + j];
        stx(o, tok(d, bb, c0 + r, h, dv) + j, acc);
    }
}

// ---------------------------------------------------------------- launchers
static size_t prep_smem(const Dims &d) {
    return sizeof(float) * (3 * (size_t)d.dk * (d.C + 1) + 2 * d.C * d.C + (size_t)d.C * d.dv);
}
static size_t state_smem(const Dims &d) {
    return sizeof(float) * ((size_t)d.dk * kSlice + 2 * (size_t)d.C * d.dk + d.C * kSlice + d.dk);
}
static size_t out_smem(const Dims &d) {
    return sizeof(float) * ((size_t)d.C * d.dk + (size_t)d.dk * d.dv + d.C * d.C + (size_t)d.C * d.dv);
}

template <typename K> static cudaError_t allow_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename E>
cudaError_t simt_prep_launch(const void *q, const void *k, const void *v, const float *g,
                             const float *b, const float *w, void *ws, const Dims &d,
                             cudaStream_t s) {
    SimtWs lay = simt_ws_layout(d);
    size_t sm = prep_smem(d);
    cudaError_t e = allow_smem(simt_chunk_prep<E>, sm);
    if (e != cudaSuccess) return e;
    launch_begin(K_SIMT_PREP, s);
    simt_chunk_prep<E><<<dim3(d.NC, d.H, d.B), kThreads, sm, s>>>(
        (const E *)q, (const E *)k, (const E *)v, g, b, w, ws, lay, d);
    launch_end(K_SIMT_PREP, s);
    return cudaGetLastError();
}

cudaError_t simt_state_fwd_launch(const float *S0, float *ST, const void *k, int k_is_bf16, void *ws,
                                  const Dims &d, cudaStream_t s) {
    SimtWs lay = simt_ws_layout(d);
    size_t sm = state_smem(d);
    cudaError_t e = allow_smem(simt_state_fwd_kernel, sm);
    if (e != cudaSuccess) return e;
    launch_begin(K_SIMT_STATE_FWD, s);
    simt_state_fwd_kernel<<<dim3(d.dv / kSlice, d.H, d.B), kThreads, sm, s>>>(S0, ST, k, k_is_bf16,
                                                                              ws, lay, d);
    launch_end(K_SIMT_STATE_FWD, s);
    return cudaGetLastError();
}

template <typename E>
cudaError_t simt_out_launch(const void *q, void *o, void *ws, const Dims &d, cudaStream_t s) {
    SimtWs lay = simt_ws_layout(d);
    size_t sm = out_smem(d);
    cudaError_t e = allow_smem(simt_out_fwd<E>, sm);
    if (e != cudaSuccess) return e;
    launch_begin(K_SIMT_OUT, s);
    simt_out_fwd<E><<<dim3(d.NC, d.H, d.B), kThreads, sm, s>>>((const E *)q, (E *)o, ws, lay, d);
    launch_end(K_SIMT_OUT, s);
    return cudaGetLastError();
}

template cudaError_t simt_prep_launch<float>(const void *, const void *, const void *, const float *,
                                             const float *, const float *, void *, const Dims &,
                                             cudaStream_t);
template cudaError_t simt_prep_launch<__nv_bfloat16>(const void *, const void *, const void *,
                                                     const float *, const float *, const float *,
                                                     void *, const Dims &, cudaStream_t);
template cudaError_t simt_out_launch<float>(const void *, void *, void *, const Dims &, cudaStream_t);
template cudaError_t simt_out_launch<__nv_bfloat16>(const void *, void *, void *, const Dims &,
                                                    cudaStream_t);

}  // namespace gdn2
