// Gate-aware chunkwise backward of Gated Delta Rule-2 on CUDA cores, float32.
//
// "Gated DeltaNet-2" (LIT-802 review, Key takeaways 2; paper Secs. 3.3-3.4,
// Apps. A-B, D.6; digg thread 11/): the per-channel erase gate b sits inside
// the dot products that accumulate the gradient of the strictly-lower A, so
// it cannot be pulled outside as a scalar beta would be.
//
// Reverse mode of the chunk step (forward in simt_fwd.cu), for a chunk with
// entering state S, exit gradient dSn = dL/dS_next and upstream dO:
//   dDelta = P^T dO + Kbar dSn                      (state_bwd, sequential)
//   dS     = (q.e^G)^T dO - W^T dDelta + diag(e^G_L) dSn
//   dU     = T^T dDelta,    dw = dU.v,  dv = dU.w
// and, because (I + A) Delta = U - Kc S, the gradient of T collapses:
//   dT = dDelta Delta^T (I + A)^T  =>  dA = -T^T dT T^T = -strictly-lower(dU Delta^T)
//   dKc = -dU S^T + dA Kh            (b inside Kc and inside every term of dA)
//   dQb = dO S^T + dP Kh,            dP = lower-incl(dO Delta^T)
//   dKh = dP^T Qb + dA^T Kc + (Delta dSn^T) diag(e^G_L)
// then, channel by channel (pairwise decay factors formed directly):
//   dq = dQb.e^G,  db = dKc.k.e^G,  dk = dKc.b.e^G + dKh.e^-G
//   dG = dQb.Qb + dKc.Kc - dKh.Kh,  plus at the chunk's last row
//        e^G_L rowsum(dSn . S) + sum_j (Delta dSn^T)_j . Kbar_j
//   dg = reverse in-chunk cumsum of dG.

#include "common.cuh"

namespace gdn2 {

constexpr int kThreadsB = 256;
constexpr int kSliceB = 32;

// -------------------------------------------------------------- state_bwd
template <typename E>
__global__ void __launch_bounds__(kThreadsB)
simt_state_bwd(const E *__restrict__ q, const E *__restrict__ k, const E *__restrict__ dO,
               const float *__restrict__ dST, float *__restrict__ dS0, void *ws, SimtWs lay,
               Dims d) {
    extern __shared__ float sm[];
    const int C = d.C, dk = d.dk, dv = d.dv;
    float *sdS = sm;                  // [dk][kSliceB]
    float *sQ = sdS + dk * kSliceB;   // [C][dk]  q.e^G
    float *sW = sQ + C * dk;          // [C][dk]
    float *sKb = sW + C * dk;         // [C][dk]  Kbar
    float *sP = sKb + C * dk;         // [C][C]
    float *sdO = sP + C * C;          // [C][kSliceB]
    float *sdD = sdO + C * kSliceB;   // [C][kSliceB]
    float *sGL = sdD + C * kSliceB;   // [dk]
    const int v0 = blockIdx.x * kSliceB, h = blockIdx.y, bb = blockIdx.z, tid = threadIdx.x;
    const size_t so = st_off(d, bb, h);
    for (int idx = tid; idx < dk * kSliceB; idx += kThreadsB) {
        int i = idx / kSliceB, j = idx % kSliceB;
        sdS[idx] = dST ? dST[so + (size_t)i * dv + v0 + j] : 0.f;
    }
    __syncthreads();
    for (int c = d.NC - 1; c >= 0; --c) {
        const int c0 = c * C, L = min(C, d.T - c0);
        const size_t ti = tile(d, bb, h, c);
        float *dSn = at<float>(ws, lay.dSn) + ti * dk * dv;
        for (int idx = tid; idx < dk * kSliceB; idx += kThreadsB) {
            int i = idx / kSliceB, j = idx % kSliceB;
            dSn[(size_t)i * dv + v0 + j] = sdS[idx];
        }
        const float *gam = at<float>(ws, lay.gam) + ti * C * dk;
        const float *Wg = at<float>(ws, lay.W) + ti * C * dk;
        for (int idx = tid; idx < L * dk; idx += kThreadsB) {
            int r = idx / dk, i = idx % dk;
            size_t o = tok(d, bb, c0 + r, h, dk) + i;
            float G = gam[idx], GL = gam[(size_t)(L - 1) * dk + i];
            sQ[idx] = ldx(q, o) * __expf(G);
            sW[idx] = Wg[idx];
            sKb[idx] = ldx(k, o) * __expf(GL - G);
        }
        for (int i = tid; i < dk; i += kThreadsB) sGL[i] = __expf(gam[(size_t)(L - 1) * dk + i]);
        const float *Pg = at<float>(ws, lay.P) + ti * C * C;
        for (int idx = tid; idx < C * C; idx += kThreadsB) sP[idx] = Pg[idx];
        for (int idx = tid; idx < L * kSliceB; idx += kThreadsB) {
            int r = idx / kSliceB, j = idx % kSliceB;
            sdO[idx] = ldx(dO, tok(d, bb, c0 + r, h, dv) + v0 + j);
        }
        __syncthreads();
        float *dDg = at<float>(ws, lay.dDelta) + ti * C * dv;
        for (int idx = tid; idx < L * kSliceB; idx += kThreadsB) {
            int r = idx / kSliceB, j = idx % kSliceB;
            float acc = 0.f;
            for (int s = r; s < L; ++s) acc += sP[s * C + r] * sdO[s * kSliceB + j];
            for (int i = 0; i < dk; ++i) acc += sKb[r * dk + i] * sdS[i * kSliceB + j];
            sdD[idx] = acc;
            dDg[(size_t)r * dv + v0 + j] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < dk * kSliceB; idx += kThreadsB) {
            int i = idx / kSliceB, j = idx % kSliceB;
            float acc = sGL[i] * sdS[idx];
            for (int r = 0; r < L; ++r)
                acc += sQ[r * dk + i] * sdO[r * kSliceB + j] - sW[r * dk + i] * sdD[r * kSliceB + j];
            sdS[idx] = acc;
        }
        __syncthreads();
    }
    if (dS0)
        for (int idx = tid; idx < dk * kSliceB; idx += kThreadsB) {
            int i = idx / kSliceB, j = idx % kSliceB;
            dS0[so + (size_t)i * dv + v0 + j] = sdS[idx];
        }
}

// ------------------------------------------------------------ chunk_bwd_a
// Per chunk: dU (and dw, dv), dP, dA and the value-axis sums X1..X4.
template <typename E>
__global__ void __launch_bounds__(kThreadsB)
simt_chunk_bwd_a(const E *__restrict__ v, const float *__restrict__ w, const E *__restrict__ dO,
                 E *__restrict__ dvout, float *__restrict__ dwout, void *ws, SimtWs lay, Dims d) {
    extern __shared__ float sm[];
    const int C = d.C, dk = d.dk, dv = d.dv, LV = d.dv + 1;
    float *sT = sm;               // [C][C]
    float *sD = sT + C * C;       // [C][LV] Delta
    float *sdD = sD + C * LV;     // [C][LV] dDelta
    float *sdU = sdD + C * LV;    // [C][LV] dU
    float *sdO = sdU + C * LV;    // [C][LV]
    float *sS = sdO + C * LV;     // [dk][LV] S_c, then dSn
    const int c = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, tid = threadIdx.x;
    const int c0 = c * C, L = min(C, d.T - c0);
    const size_t ti = tile(d, bb, h, c);
    const float *Tg = at<float>(ws, lay.Tinv) + ti * C * C;
    for (int idx = tid; idx < C * C; idx += kThreadsB) sT[idx] = Tg[idx];
    const float *Dg = at<float>(ws, lay.Delta) + ti * C * dv;
    const float *dDg = at<float>(ws, lay.dDelta) + ti * C * dv;
    for (int idx = tid; idx < L * dv; idx += kThreadsB) {
        int r = idx / dv, j = idx % dv;
        sD[r * LV + j] = Dg[idx];
        sdD[r * LV + j] = dDg[idx];
        sdO[r * LV + j] = ldx(dO, tok(d, bb, c0 + r, h, dv) + j);
    }
    const float *Sc = at<float>(ws, lay.Sc) + ti * dk * dv;
    for (int idx = tid; idx < dk * dv; idx += kThreadsB) sS[(idx / dv) * LV + idx % dv] = Sc[idx];
    __syncthreads();
    for (int idx = tid; idx < L * dv; idx += kThreadsB) {
        int r = idx / dv, j = idx % dv;
        float acc = 0.f;
        for (int s = r; s < L; ++s) acc += sT[s * C + r] * sdD[s * LV + j];
        sdU[r * LV + j] = acc;
        size_t o = tok(d, bb, c0 + r, h, dv) + j;
        dwout[o] = acc * ldx(v, o);
        stx(dvout, o, acc * w[o]);
    }
    __syncthreads();
    float *dPg = at<float>(ws, lay.dP) + ti * C * C;
    float *dAg = at<float>(ws, lay.dA) + ti * C * C;
    for (int p = tid; p < C * C; p += kThreadsB) {
        int r = p / C, j = p % C;
        float ap = 0.f, aa = 0.f;
        if (r < L && j <= r) {
            for (int x = 0; x < dv; ++x) {
                ap += sdO[r * LV + x] * sD[j * LV + x];
                aa += sdU[r * LV + x] * sD[j * LV + x];
            }
        }
        dPg[p] = ap;
        dAg[p] = (j < r) ? -aa : 0.f;
    }
    float *X1 = at<float>(ws, lay.X1) + ti * C * dk;
    float *X2 = at<float>(ws, lay.X2) + ti * C * dk;
    for (int idx = tid; idx < L * dk; idx += kThreadsB) {
        int r = idx / dk, i = idx % dk;
        float a1 = 0.f, a2 = 0.f;
        for (int x = 0; x < dv; ++x) {
            float s = sS[i * LV + x];
            a1 += sdO[r * LV + x] * s;
            a2 += sdU[r * LV + x] * s;
        }
        X1[idx] = a1;
        X2[idx] = a2;
    }
    const float *dSn = at<float>(ws, lay.dSn) + ti * dk * dv;
    float *X4 = at<float>(ws, lay.X4) + ti * dk;
    for (int i = tid; i < dk; i += kThreadsB) {
        float acc = 0.f;
        for (int x = 0; x < dv; ++x) acc += dSn[(size_t)i * dv + x] * sS[i * LV + x];
        X4[i] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < dk * dv; idx += kThreadsB) sS[(idx / dv) * LV + idx % dv] = dSn[idx];
    __syncthreads();
    float *X3 = at<float>(ws, lay.X3) + ti * C * dk;
    for (int idx = tid; idx < L * dk; idx += kThreadsB) {
        int r = idx / dk, i = idx % dk;
        float acc = 0.f;
        for (int x = 0; x < dv; ++x) acc += sD[r * LV + x] * sS[i * LV + x];
        X3[idx] = acc;
    }
}

// ------------------------------------------------------------ chunk_bwd_b
// Per chunk and key channel: dq, dk, db, dg (pairwise decay factors).
template <typename E>
__global__ void __launch_bounds__(kThreadsB)
simt_chunk_bwd_b(const E *__restrict__ q, const E *__restrict__ k, const float *__restrict__ b,
                 E *__restrict__ dqout, E *__restrict__ dkout, float *__restrict__ dbout,
                 float *__restrict__ dgout, void *ws, SimtWs lay, Dims d) {
    extern __shared__ float sm[];
    const int C = d.C, dk = d.dk, LD = d.C + 1;
    float *sG = sm;             // [dk][LD]
    float *sK = sG + dk * LD;   // [dk][LD]
    float *sQ = sK + dk * LD;   // [dk][LD]
    float *sB = sQ + dk * LD;   // [dk][LD]
    float *sdG = sB + dk * LD;  // [dk][LD]
    float *sdP = sdG + dk * LD; // [C][C]
    float *sdA = sdP + C * C;   // [C][C]
    const int c = blockIdx.x, h = blockIdx.y, bb = blockIdx.z, tid = threadIdx.x;
    const int c0 = c * C, L = min(C, d.T - c0);
    const size_t ti = tile(d, bb, h, c);
    const float *gam = at<float>(ws, lay.gam) + ti * C * dk;
    for (int idx = tid; idx < L * dk; idx += kThreadsB) {
        int r = idx / dk, i = idx % dk;
        size_t o = tok(d, bb, c0 + r, h, dk) + i;
        sG[i * LD + r] = gam[idx];
        sK[i * LD + r] = ldx(k, o);
        sQ[i * LD + r] = ldx(q, o);
        sB[i * LD + r] = b[o];
    }
    const float *dPg = at<float>(ws, lay.dP) + ti * C * C;
    const float *dAg = at<float>(ws, lay.dA) + ti * C * C;
    for (int p = tid; p < C * C; p += kThreadsB) { sdP[p] = dPg[p]; sdA[p] = dAg[p]; }
    __syncthreads();
    const float *X1 = at<float>(ws, lay.X1) + ti * C * dk;
    const float *X2 = at<float>(ws, lay.X2) + ti * C * dk;
    const float *X3 = at<float>(ws, lay.X3) + ti * C * dk;
    for (int idx = tid; idx < L * dk; idx += kThreadsB) {
        int r = idx / dk, i = idx % dk;
        const float *G = sG + i * LD, *kk = sK + i * LD, *qq = sQ + i * LD, *bb_ = sB + i * LD;
        float Gr = G[r], eG = __expf(Gr), GL = G[L - 1];
        float dqE = eG * X1[idx], dKcE = -eG * X2[idx];
        for (int j = 0; j <= r; ++j) {
            float f = kk[j] * __expf(Gr - G[j]);
            dqE += sdP[r * C + j] * f;
            dKcE += sdA[r * C + j] * f;   // dA is zero on the diagonal
        }
        float dKhE = __expf(GL - Gr) * X3[idx];
        for (int s = r; s < L; ++s) {
            float f = __expf(G[s] - Gr);
            dKhE += (sdP[s * C + r] * qq[s] + sdA[s * C + r] * bb_[s] * kk[s]) * f;
        }
        size_t o = tok(d, bb, c0 + r, h, dk) + i;
        stx(dqout, o, dqE);
        stx(dkout, o, dKcE * bb_[r] + dKhE);
        dbout[o] = dKcE * kk[r];
        sdG[i * LD + r] = dqE * qq[r] + dKcE * bb_[r] * kk[r] - dKhE * kk[r];
    }
    __syncthreads();
    const float *X4 = at<float>(ws, lay.X4) + ti * dk;
    for (int i = tid; i < dk; i += kThreadsB) {
        const float *G = sG + i * LD, *kk = sK + i * LD;
        float GL = G[L - 1];
        float end = __expf(GL) * X4[i];
        for (int j = 0; j < L; ++j) end += X3[(size_t)j * dk + i] * kk[j] * __expf(GL - G[j]);
        float acc = end;
        for (int r = L - 1; r >= 0; --r) {
            acc += sdG[i * LD + r];
            dgout[tok(d, bb, c0 + r, h, dk) + i] = acc;
        }
    }
}

// ---------------------------------------------------------------- launchers
template <typename K> static cudaError_t allow_smem_b(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename E>
cudaError_t simt_bwd_launch(const void *q, const void *k, const void *v, const float *b,
                            const float *w, const void *dO, const float *dST, void *dq, void *dk,
                            void *dv, float *dg, float *db, float *dw, float *dS0, void *ws,
                            const Dims &d, cudaStream_t s) {
    SimtWs lay = simt_ws_layout(d);
    cudaError_t e;
    size_t sm1 = sizeof(float) * ((size_t)d.dk * kSliceB + 3 * (size_t)d.C * d.dk + d.C * d.C +
                                  2 * d.C * kSliceB + d.dk);
    if ((e = allow_smem_b(simt_state_bwd<E>, sm1)) != cudaSuccess) return e;
    launch_begin(K_SIMT_STATE_BWD, s);
    simt_state_bwd<E><<<dim3(d.dv / kSliceB, d.H, d.B), kThreadsB, sm1, s>>>(
        (const E *)q, (const E *)k, (const E *)dO, dST, dS0, ws, lay, d);
    launch_end(K_SIMT_STATE_BWD, s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    size_t sm2 = sizeof(float) * ((size_t)d.C * d.C + 4 * (size_t)d.C * (d.dv + 1) +
                                  (size_t)d.dk * (d.dv + 1));
    if ((e = allow_smem_b(simt_chunk_bwd_a<E>, sm2)) != cudaSuccess) return e;
    launch_begin(K_SIMT_BWD_A, s);
    simt_chunk_bwd_a<E><<<dim3(d.NC, d.H, d.B), kThreadsB, sm2, s>>>(
        (const E *)v, w, (const E *)dO, (E *)dv, dw, ws, lay, d);
    launch_end(K_SIMT_BWD_A, s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    size_t sm3 = sizeof(float) * (5 * (size_t)d.dk * (d.C + 1) + 2 * (size_t)d.C * d.C);
    if ((e = allow_smem_b(simt_chunk_bwd_b<E>, sm3)) != cudaSuccess) return e;
    launch_begin(K_SIMT_BWD_B, s);
    simt_chunk_bwd_b<E><<<dim3(d.NC, d.H, d.B), kThreadsB, sm3, s>>>(
        (const E *)q, (const E *)k, b, (E *)dq, (E *)dk, db, dg, ws, lay, d);
    launch_end(K_SIMT_BWD_B, s);
    return cudaGetLastError();
}

template cudaError_t simt_bwd_launch<float>(const void *, const void *, const void *, const float *,
                                            const float *, const void *, const float *, void *,
                                            void *, void *, float *, float *, float *, float *,
                                            void *, const Dims &, cudaStream_t);
template cudaError_t simt_bwd_launch<__nv_bfloat16>(const void *, const void *, const void *,
                                                    const float *, const float *, const void *,
                                                    const float *, void *, void *, void *, float *,
                                                    float *, float *, float *, void *, const Dims &,
                                                    cudaStream_t);

}  // namespace gdn2
