// gdn2_fwd_noalloc: the chunkwise forward for callers that cannot allocate
// device memory (see include/gdn2.h).  Its scratch is a file-scope device
// array of GDN2_NOALLOC_SCRATCH_BYTES that every GPU which loads this library
// holds until the process exits.  All calls share it.

#include "common.cuh"

namespace gdn2 {

template <typename E>
cudaError_t simt_prep_launch(const void *, const void *, const void *, const float *, const float *,
                             const float *, void *, const Dims &, cudaStream_t);
cudaError_t simt_state_fwd_launch(const float *, float *, const void *, int, void *, const Dims &,
                                  cudaStream_t);
template <typename E>
cudaError_t simt_out_launch(const void *, void *, void *, const Dims &, cudaStream_t);

// The scratch itself.  In host code this name is only a stand-in for the
// symbol; kernels must receive the device address that cudaGetSymbolAddress
// returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN2_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch in the current device's context.  It is
// looked up on every call (cudaGetSymbolAddress allocates nothing), so a call
// made after cudaDeviceReset, or in a new primary context, never receives an
// address from a context that no longer exists.  The first lookup in a
// context also loads the library's device code there, which is why the first
// call on a device should come before any stream capture.
static cudaError_t scratch_address(void **out) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    *out = p;
    return cudaSuccess;
}

}  // namespace gdn2

using namespace gdn2;

extern "C" gdn2_status gdn2_fwd_noalloc(const void *q, const void *k, const void *v,
                                        const float *g, const float *b, const float *w,
                                        const float *S0, void *o, float *ST, int B, int T, int H,
                                        int d_k, int d_v, int chunk, gdn2_io io,
                                        gdn2_stream_t stream) {
    if (B < 1 || T < 1 || H < 1 || (io != GDN2_IO_F32 && io != GDN2_IO_BF16))
        return GDN2_ERR_INVALID_ARG;
    auto supported_d = [](int x) { return x == 32 || x == 64 || x == 128; };
    if (!supported_d(d_k) || !supported_d(d_v) || !(chunk == 16 || chunk == 32 || chunk == 64))
        return GDN2_ERR_UNSUPPORTED;
    if (H > 65535 || B > 65535) return GDN2_ERR_UNSUPPORTED;
    for (const void *p : {q, k, v, (const void *)g, (const void *)b, (const void *)w, (const void *)o})
        if (!p || ((uintptr_t)p & 15u)) return GDN2_ERR_INVALID_ARG;
    for (const void *p : {(const void *)S0, (const void *)ST})
        if (p && ((uintptr_t)p & 15u)) return GDN2_ERR_INVALID_ARG;
    // size check before any CUDA call: problems whose scratch exceeds the
    // array are rejected
    if ((long long)B * H * ((T + chunk - 1) / chunk) > (1LL << 31)) return GDN2_ERR_WORKSPACE;
    Dims d{B, T, H, d_k, d_v, chunk, (T + chunk - 1) / chunk};
    if (simt_ws_layout(d).fwd_end > (size_t)GDN2_NOALLOC_SCRATCH_BYTES) return GDN2_ERR_WORKSPACE;

    void *ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return GDN2_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    // Every scratch element the three kernels read is written earlier in the
    // same call, so nothing needs clearing between calls.
    if (io == GDN2_IO_BF16)
        e = simt_prep_launch<__nv_bfloat16>(q, k, v, g, b, w, ws, d, s);
    else
        e = simt_prep_launch<float>(q, k, v, g, b, w, ws, d, s);
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    if (simt_state_fwd_launch(S0, ST, k, io == GDN2_IO_BF16, ws, d, s) != cudaSuccess)
        return GDN2_ERR_CUDA;
    e = io == GDN2_IO_BF16 ? simt_out_launch<__nv_bfloat16>(q, o, ws, d, s)
                           : simt_out_launch<float>(q, o, ws, d, s);
    return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}
