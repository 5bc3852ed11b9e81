// The link step of the segment-parallel state passes (SegPass in common.cuh):
// entry states S_{s+1} = M_s S_s + N_s forward, exit gradients
// E_s = M_{s+1}^T E_{s+1} + R_{s+1} backward, for every (b, h) of a split call.
// Only the state crosses chunk borders ("Gated DeltaNet-2", digg thread 9/),
// so a segment of chunks acts on it as one affine map.
//
// Grid (8, B H): a CTA owns 16 of the 128 columns of one (b, h) and keeps them
// in shared memory from step to step; the map M is staged in shared memory 32
// rows (or columns) at a time with coalesced loads.  Thread t computes row
// t / 2, 8 columns.  float32 throughout.

#include "common.cuh"

namespace gdn2 {

template <bool TRANSPOSE>
__global__ void __launch_bounds__(256) seg_link_kernel(SegPass sp) {
    __shared__ float Es[128][17];  // the carried columns
    __shared__ float Ms[32][129];  // 32 k-rows of M (TRANSPOSE: M[k][i]) or of M^T (M[i][k] at [k][i])
    const int tid = threadIdx.x, i = tid >> 1, j0 = 8 * (tid & 1), c0 = 16 * blockIdx.x;
    const size_t bh = blockIdx.y;
    const int first = TRANSPOSE ? sp.P - 2 : 1;
    {
        const float *E = seg_buf(sp, bh, first, SEG_ENTRY);
        for (int e = tid; e < 128 * 16; e += 256) Es[e >> 4][e & 15] = E[(e >> 4) * 128 + c0 + (e & 15)];
    }
    __syncthreads();
    for (int step = 0; step < sp.P - 2; ++step) {
        // forward: from segment s = 1 + step to s + 1; backward: from s + 1 = P - 2 - step to s
        const int s_map = TRANSPOSE ? sp.P - 2 - step : 1 + step;
        const int s_out = TRANSPOSE ? s_map - 1 : s_map + 1;
        const float *M = seg_buf(sp, bh, s_map, SEG_MAP);
        const float *A = seg_buf(sp, bh, s_map, SEG_ZERO) + (size_t)i * 128 + c0 + j0;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = A[j];
        for (int k0 = 0; k0 < 128; k0 += 32) {
            // Ms[kk][r] = the factor of E[k0 + kk] in output row r
            for (int e = tid; e < 32 * 128; e += 256) {
                const int a = e >> 7, b = e & 127;  // coalesced over b
                if (TRANSPOSE) Ms[a][b] = M[(size_t)(k0 + a) * 128 + b];  // M[k][i], k = k0 + a, i = b
                else Ms[e & 31][e >> 5] = M[(size_t)(e >> 5) * 128 + k0 + (e & 31)];  // M[i][k]
            }
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < 32; ++kk) {
                const float m = Ms[kk][i];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = fmaf(m, Es[k0 + kk][j0 + j], acc[j]);
            }
            __syncthreads();
        }
        float *out = seg_buf(sp, bh, s_out, SEG_ENTRY) + (size_t)i * 128 + c0 + j0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            Es[i][j0 + j] = acc[j];
            out[j] = acc[j];
        }
        __syncthreads();
    }
}

cudaError_t seg_link_launch(const SegPass &sp, int nbh, bool backward, cudaStream_t s) {
    launch_begin(K_SEG_LINK, s);
    if (backward) seg_link_kernel<true><<<dim3(8, nbh), 256, 0, s>>>(sp);
    else seg_link_kernel<false><<<dim3(8, nbh), 256, 0, s>>>(sp);
    launch_end(K_SEG_LINK, s);
    return cudaGetLastError();
}

}  // namespace gdn2
