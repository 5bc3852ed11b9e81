// The link step of the segment-parallel state passes (SegPass in common.cuh):
// entry states S_{s+1} = M_s S_s + N_s forward, exit gradients
// E_s = M_{s+1}^T E_{s+1} + R_{s+1} backward, for every (b, h) of a split call.
// Only the state crosses chunk borders ("Gated DeltaNet-2", digg thread 9/),
// so a segment of chunks acts on it as one affine map.
//
// Grid (8, B H): a CTA owns 16 of the 128 columns of one (b, h) and keeps them
// in shared memory from step to step.  The whole map M (64 KB) is staged in
// dynamic shared memory per step, each thread's sixteen 16-byte loads issued
// before any is stored, so that a step waits for one round trip to L2.
// Thread t computes row t / 2, 8 columns.  float32 throughout.

#include "common.cuh"

namespace gdn2 {

constexpr int kLinkMs = 128 * 129;                         // floats of the staged map
constexpr int kLinkSmem = (kLinkMs + 128 * 17) * 4;        // + the carried columns

template <bool TRANSPOSE>
__global__ void __launch_bounds__(256) seg_link_kernel(SegPass sp) {
    extern __shared__ float link_sm[];
    float(*Ms)[129] = reinterpret_cast<float(*)[129]>(link_sm);             // Ms[k][i]: factor of E[k] in row i
    float(*Es)[17] = reinterpret_cast<float(*)[17]>(link_sm + kLinkMs);    // the carried columns
    const int tid = threadIdx.x, i = tid >> 1, j0 = 8 * (tid & 1), c0 = 16 * blockIdx.x;
    const size_t bh = blockIdx.y;
    const int first = TRANSPOSE ? sp.P - 2 : 1;
    {
        const float *E = seg_buf(sp, bh, first, SEG_ENTRY);
        float4 ev[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {  // 128 rows x 4 float4 of this CTA's 16 columns
            const int q = tid + 256 * m;
            ev[m] = *reinterpret_cast<const float4 *>(E + (q >> 2) * 128 + c0 + 4 * (q & 3));
        }
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int q = tid + 256 * m, r = q >> 2, c = 4 * (q & 3);
            Es[r][c] = ev[m].x;
            Es[r][c + 1] = ev[m].y;
            Es[r][c + 2] = ev[m].z;
            Es[r][c + 3] = ev[m].w;
        }
    }
    for (int step = 0; step < sp.P - 2; ++step) {
        // forward: from segment s = 1 + step to s + 1; backward: from s + 1 = P - 2 - step to s
        const int s_map = TRANSPOSE ? sp.P - 2 - step : 1 + step;
        const int s_out = TRANSPOSE ? s_map - 1 : s_map + 1;
        const float *M = seg_buf(sp, bh, s_map, SEG_MAP);
        const float *A = seg_buf(sp, bh, s_map, SEG_ZERO) + (size_t)i * 128 + c0 + j0;
        float acc[8];
        {
            const float4 a0 = *reinterpret_cast<const float4 *>(A), a1 = *reinterpret_cast<const float4 *>(A + 4);
            acc[0] = a0.x; acc[1] = a0.y; acc[2] = a0.z; acc[3] = a0.w;
            acc[4] = a1.x; acc[5] = a1.y; acc[6] = a1.z; acc[7] = a1.w;
        }
        // the whole map, 128 rows of 32 float4: row q / 32, float4 q % 32, with
        // q = tid + 256 m; stored as Ms[k][i]
        float4 mv[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int q = tid + 256 * m;
            mv[m] = *reinterpret_cast<const float4 *>(M + (size_t)(q >> 5) * 128 + 4 * (q & 31));
        }
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int q = tid + 256 * m, row = q >> 5, col = 4 * (q & 31);
            const float v[4] = {mv[m].x, mv[m].y, mv[m].z, mv[m].w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                if (TRANSPOSE) Ms[row][col + x] = v[x];  // M[k][i]: k = row, i = col + x
                else Ms[col + x][row] = v[x];            // M[i][k]: i = row, k = col + x
            }
        }
        __syncthreads();  // the map and the carried columns are in place
#pragma unroll 8
        for (int k = 0; k < 128; ++k) {
            const float mk = Ms[k][i];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = fmaf(mk, Es[k][j0 + j], acc[j]);
        }
        __syncthreads();  // every thread has read the carried columns and the map
        float *out = seg_buf(sp, bh, s_out, SEG_ENTRY) + (size_t)i * 128 + c0 + j0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            Es[i][j0 + j] = acc[j];
            out[j] = acc[j];
        }
    }
}

cudaError_t seg_link_launch(const SegPass &sp, int nbh, bool backward, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(seg_link_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinkSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(seg_link_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinkSmem);
    if (e != cudaSuccess) return e;
    launch_begin(K_SEG_LINK, s);
    if (backward) seg_link_kernel<true><<<dim3(8, nbh), 256, kLinkSmem, s>>>(sp);
    else seg_link_kernel<false><<<dim3(8, nbh), 256, kLinkSmem, s>>>(sp);
    launch_end(K_SEG_LINK, s);
    return cudaGetLastError();
}

}  // namespace gdn2
