// Host side of the C ABI in include/gdn2.h: argument checks, workspace sizing
// and kernel dispatch.  No allocation, no synchronisation (except
// gdn2_get_device_status), no CPU fallback.

#include <stdint.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {

// kernels and launchers of the other translation units
template <typename E>
cudaError_t simt_prep_launch(const void *, const void *, const void *, const float *, const float *,
                             const float *, void *, const Dims &, cudaStream_t);
cudaError_t simt_state_fwd_launch(const float *, float *, const void *, int, void *, const Dims &,
                                  cudaStream_t);
template <typename E>
cudaError_t simt_out_launch(const void *, void *, void *, const Dims &, cudaStream_t);
template <typename E>
cudaError_t simt_bwd_launch(const void *, const void *, const void *, const float *, const float *,
                            const void *, const float *, void *, void *, void *, float *, float *,
                            float *, float *, void *, const Dims &, cudaStream_t);
cudaError_t decode_launch(const void *, const void *, const void *, const void *, const void *,
                          const void *, float *, void *, int, int, int, int, gdn2_io, gdn2_io,
                          cudaStream_t);
cudaError_t tc_fwd_launch(const void *, const void *, const void *, const void *, const void *,
                          const void *, const float *, void *, float *, void *, int,
                          unsigned int *, const Dims &, cudaStream_t);
cudaError_t tc_bwd_launch(const void *, const void *, const void *, const void *, const void *,
                          const void *, const void *, const float *, void *, void *, void *,
                          void *, void *, void *, float *, void *, unsigned int *, const Dims &,
                          cudaStream_t);

// The device status word (GDN2_OK or the first error a kernel recorded), and
// the slot that gdn2_get_device_status moves it into.  One pair per device,
// shared by every stream.
__device__ unsigned int g_status_word;
__device__ unsigned int g_status_taken;

// device address of g_status_word in the current device's context, looked up
// on every call (cheap, allocates nothing, and never stale after a reset)
static unsigned int *status_word() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    return static_cast<unsigned int *>(p);
}

// reads and clears the status word in one atomic step, after the work
// enqueued on the stream before it
static __global__ void status_take_kernel() { g_status_taken = atomicExch(&g_status_word, 0u); }
static std::mutex g_status_mu;

// the tensor-core path: bf16 I/O, d_k = d_v = 128, chunk 64
static bool use_tc(const Dims &d, gdn2_io io) {
    return io == GDN2_IO_BF16 && d.dk == 128 && d.dv == 128 && d.C == 64;
}

static std::atomic<unsigned long long> g_launches{0};

// ---- optional per-kernel event timing (gdn2_set_kernel_timer)
struct PendingTiming {
    int kind;
    cudaEvent_t start, end;
};
static std::mutex g_timer_mu;
static std::atomic<bool> g_timer_on{false};
static std::vector<PendingTiming> g_pending;
static cudaEvent_t g_open_start[K_KINDS];
static unsigned long long g_kind_count[K_KINDS];
static double g_kind_ms[K_KINDS];
static const char *const g_kind_names[K_KINDS] = {
    "simt_chunk_prep", "simt_state_fwd", "simt_out_fwd", "simt_state_bwd", "simt_chunk_bwd_a",
    "simt_chunk_bwd_b", "decode_step", "tc_prep", "tc_fwd", "tc_bwd_state", "tc_bwd_grad", "seq_table"};

void launch_begin(int kind, cudaStream_t s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (!g_timer_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_timer_mu);
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) == cudaSuccess) cudaEventRecord(e, s);
    g_open_start[kind] = e;
}

void launch_end(int kind, cudaStream_t s) {
    if (!g_timer_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_timer_mu);
    cudaEvent_t st = g_open_start[kind], e = nullptr;
    g_open_start[kind] = nullptr;
    if (!st) return;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaEventDestroy(st);
        return;
    }
    cudaEventRecord(e, s);
    g_pending.push_back({kind, st, e});
}

static bool supported_d(int x) { return x == 32 || x == 64 || x == 128; }
static bool supported_chunk(int c) { return c == 16 || c == 32 || c == 64; }
static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

static gdn2_status check_dims(int B, int T, int H, int dk, int dv, int chunk, gdn2_io io) {
    if (B < 1 || T < 1 || H < 1) return GDN2_ERR_INVALID_ARG;
    if (io != GDN2_IO_F32 && io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    if (!supported_d(dk) || !supported_d(dv) || !supported_chunk(chunk)) return GDN2_ERR_UNSUPPORTED;
    // grid limits: chunks per sequence in grid.x, H in grid.y, B in grid.z
    if (H > 65535 || B > 65535) return GDN2_ERR_UNSUPPORTED;
    if ((long long)B * T * H * (dk > dv ? dk : dv) > (1LL << 40)) return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}

static Dims make_dims(int B, int T, int H, int dk, int dv, int chunk) {
    return Dims{B, T, H, dk, dv, chunk, (T + chunk - 1) / chunk, 0};
}

// every required pointer non-null and 16-byte aligned; optional ones aligned
static gdn2_status check_ptrs(std::initializer_list<const void *> required,
                              std::initializer_list<const void *> optional) {
    for (const void *p : required)
        if (!p || !aligned16(p)) return GDN2_ERR_INVALID_ARG;
    for (const void *p : optional)
        if (p && !aligned16(p)) return GDN2_ERR_INVALID_ARG;
    return GDN2_OK;
}

static gdn2_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA; }

static cudaError_t run_forward(const void *q, const void *k, const void *v, const float *g,
                               const float *b, const float *w, const float *S0, void *o, float *ST,
                               void *ws, const Dims &d, gdn2_io io, cudaStream_t s) {
    cudaError_t e;
    if (io == GDN2_IO_BF16) {
        if ((e = simt_prep_launch<__nv_bfloat16>(q, k, v, g, b, w, ws, d, s)) != cudaSuccess) return e;
    } else {
        if ((e = simt_prep_launch<float>(q, k, v, g, b, w, ws, d, s)) != cudaSuccess) return e;
    }
    if ((e = simt_state_fwd_launch(S0, ST, k, io == GDN2_IO_BF16, ws, d, s)) != cudaSuccess) return e;
    if (o) {
        if (io == GDN2_IO_BF16) return simt_out_launch<__nv_bfloat16>(q, o, ws, d, s);
        return simt_out_launch<float>(q, o, ws, d, s);
    }
    return cudaSuccess;
}

}  // namespace gdn2

using namespace gdn2;

extern "C" {

static size_t ws_bytes_for(const Dims &d, gdn2_io io, int for_bwd) {
    SimtWs lay = simt_ws_layout(d);
    if (use_tc(d, io)) {
        const TcWs t = tc_ws_layout(d);
        return for_bwd ? t.bwd_end : t.rec_end;
    }
    return for_bwd ? lay.bwd_end : lay.fwd_end;
}

size_t gdn2_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk, gdn2_io io,
                            int for_bwd) {
    if (check_dims(B, T, H, d_k, d_v, chunk, io) != GDN2_OK) return 0;
    return ws_bytes_for(make_dims(B, T, H, d_k, d_v, chunk), io, for_bwd);
}

// gate tensors in bf16 need the tensor-core path
static gdn2_status check_gate_io(const Dims &d, gdn2_io io, gdn2_io gate_io) {
    if (gate_io != GDN2_IO_F32 && gate_io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    if (gate_io == GDN2_IO_BF16 && !use_tc(d, io)) return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}

gdn2_status gdn2_fwd_ex(const void *q, const void *k, const void *v, const void *g, const void *b,
                        const void *w, const float *S0, void *o, float *ST, void *ws,
                        size_t ws_bytes, int B, int T, int H, int d_k, int d_v, int chunk,
                        gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    gdn2_status st = check_dims(B, T, H, d_k, d_v, chunk, io);
    if (st != GDN2_OK) return st;
    Dims d = make_dims(B, T, H, d_k, d_v, chunk);
    if ((st = check_gate_io(d, io, gate_io)) != GDN2_OK) return st;
    st = check_ptrs({q, k, v, g, b, w, o}, {S0, ST});
    if (st != GDN2_OK) return st;
    if (!ws || !aligned16(ws) || ws_bytes < ws_bytes_for(d, io, 0)) return GDN2_ERR_WORKSPACE;
    d.gb = gate_io == GDN2_IO_BF16;
    if (use_tc(d, io)) {
        unsigned int *status = status_word();
        if (!status) return GDN2_ERR_CUDA;
        const int keep = ws_bytes >= ws_bytes_for(d, io, 1);
        return cuda_status(tc_fwd_launch(q, k, v, g, b, w, S0, o, ST, ws, keep, status, d,
                                         (cudaStream_t)stream));
    }
    return cuda_status(run_forward(q, k, v, static_cast<const float *>(g), static_cast<const float *>(b),
                                   static_cast<const float *>(w), S0, o, ST, ws, d, io,
                                   (cudaStream_t)stream));
}

gdn2_status gdn2_fwd(const void *q, const void *k, const void *v, const float *g, const float *b,
                     const float *w, const float *S0, void *o, float *ST, void *ws,
                     size_t ws_bytes, int B, int T, int H, int d_k, int d_v, int chunk,
                     gdn2_io io, gdn2_stream_t stream) {
    return gdn2_fwd_ex(q, k, v, g, b, w, S0, o, ST, ws, ws_bytes, B, T, H, d_k, d_v, chunk, io,
                       GDN2_IO_F32, stream);
}

gdn2_status gdn2_bwd_ex(const void *q, const void *k, const void *v, const void *g, const void *b,
                        const void *w, const float *S0, const void *dO, const float *dST, void *dq,
                        void *dk, void *dv, void *dg, void *db, void *dw, float *dS0, void *ws,
                        size_t ws_bytes, int ws_has_fwd, int B, int T, int H, int d_k, int d_v,
                        int chunk, gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    gdn2_status st = check_dims(B, T, H, d_k, d_v, chunk, io);
    if (st != GDN2_OK) return st;
    Dims d = make_dims(B, T, H, d_k, d_v, chunk);
    if ((st = check_gate_io(d, io, gate_io)) != GDN2_OK) return st;
    st = check_ptrs({q, k, v, g, b, w, dO, dq, dk, dv, dg, db, dw}, {S0, dST, dS0});
    if (st != GDN2_OK) return st;
    if (!ws || !aligned16(ws) || ws_bytes < ws_bytes_for(d, io, 1)) return GDN2_ERR_WORKSPACE;
    d.gb = gate_io == GDN2_IO_BF16;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (use_tc(d, io)) {
        unsigned int *status = status_word();
        if (!status) return GDN2_ERR_CUDA;
        if (!ws_has_fwd) {
            e = tc_fwd_launch(q, k, v, g, b, w, S0, nullptr, nullptr, ws, 1, status, d, s);
            if (e != cudaSuccess) return GDN2_ERR_CUDA;
        }
        return cuda_status(tc_bwd_launch(q, k, v, g, b, w, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws,
                                         status, d, s));
    }
    const float *gf = static_cast<const float *>(g), *bf = static_cast<const float *>(b),
                *wf = static_cast<const float *>(w);
    float *dgf = static_cast<float *>(dg), *dbf = static_cast<float *>(db), *dwf = static_cast<float *>(dw);
    if (!ws_has_fwd) {
        e = run_forward(q, k, v, gf, bf, wf, S0, nullptr, nullptr, ws, d, io, s);
        if (e != cudaSuccess) return GDN2_ERR_CUDA;
    }
    if (io == GDN2_IO_BF16)
        e = simt_bwd_launch<__nv_bfloat16>(q, k, v, bf, wf, dO, dST, dq, dk, dv, dgf, dbf, dwf, dS0, ws,
                                           d, s);
    else
        e = simt_bwd_launch<float>(q, k, v, bf, wf, dO, dST, dq, dk, dv, dgf, dbf, dwf, dS0, ws, d, s);
    return cuda_status(e);
}

gdn2_status gdn2_bwd(const void *q, const void *k, const void *v, const float *g, const float *b,
                     const float *w, const float *S0, const void *dO, const float *dST, void *dq,
                     void *dk, void *dv, float *dg, float *db, float *dw, float *dS0, void *ws,
                     size_t ws_bytes, int ws_has_fwd, int B, int T, int H, int d_k, int d_v,
                     int chunk, gdn2_io io, gdn2_stream_t stream) {
    return gdn2_bwd_ex(q, k, v, g, b, w, S0, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, ws_bytes,
                       ws_has_fwd, B, T, H, d_k, d_v, chunk, io, GDN2_IO_F32, stream);
}

// ---------------------------------------------------------- packed sequences
// Chunk offsets co[0..N] of the sequences cu[0..N] (chunk C): one block,
// a block-wide scan in steps of its 1024 threads.  A table that is not
// non-decreasing from 0 to T gets co = 0 throughout (every sequence empty)
// and records GDN2_ERR_INVALID_ARG.
static __global__ void __launch_bounds__(1024) seq_table_kernel(const int *cu, int N, int T, int C, int *co,
                                                               unsigned int *status) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    __shared__ int bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        carry = 0;
        bad = (cu[0] != 0 || cu[N] != T);
    }
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int n = base + tid;
        int cnt = 0;
        if (n < N) {
            const int len = cu[n + 1] - cu[n];
            if (len < 0) bad = 1;
            cnt = len > 0 ? (len + C - 1) / C : 0;
        }
        int x = cnt;  // inclusive scan: warps, then warp totals
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int t = warp_tot[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, off);
                if (lane >= off) t += y;
            }
            warp_tot[lane] = t;
        }
        __syncthreads();
        const int incl = carry + x + (warp > 0 ? warp_tot[warp - 1] : 0);
        if (n < N) co[n + 1] = incl;
        __syncthreads();
        if (tid == 1023) carry = incl;
        __syncthreads();
    }
    if (tid == 0) co[0] = 0;
    __syncthreads();
    if (bad) {
        for (int n = tid; n <= N; n += 1024) co[n] = 0;
        if (tid == 0) record_status(status, GDN2_ERR_INVALID_ARG);
    }
}

// a packed call: B = 1 row of T tokens holding N sequences, the chunk bound
// ceil(T / C) + N, and the chunk table at the end of the workspace
static Dims varlen_dims(int N, int T, int H, int dk, int dv, int chunk) {
    Dims d = make_dims(1, T, H, dk, dv, chunk);
    d.NC = (T + chunk - 1) / chunk + N;
    d.N = N;
    return d;
}
// the chunk table follows the records (a forward-only workspace) or the whole
// layout (a workspace that keeps the forward for the backward)
static size_t varlen_table_at(const Dims &d, int for_bwd) {
    const TcWs t = tc_ws_layout(d);
    return for_bwd ? t.bwd_end : t.rec_end;
}
static size_t varlen_ws_bytes(const Dims &d, int for_bwd) {
    return varlen_table_at(d, for_bwd) + align256((size_t)(d.N + 1) * sizeof(int));
}
static gdn2_status check_varlen(int N, int T, int H, int dk, int dv, int chunk, gdn2_io io, gdn2_io gate_io,
                                const int *cu) {
    if (N < 1 || !cu || !aligned16(cu)) return GDN2_ERR_INVALID_ARG;
    gdn2_status st = check_dims(1, T, H, dk, dv, chunk, io);
    if (st != GDN2_OK) return st;
    if (gate_io != GDN2_IO_F32 && gate_io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    if (!use_tc(make_dims(1, T, H, dk, dv, chunk), io)) return GDN2_ERR_UNSUPPORTED;
    if (N > 65535 || (long long)H * ((T + chunk - 1) / chunk + N) > 0x7fffffffLL) return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}
static cudaError_t seq_table_launch(Dims &d, void *ws, int for_bwd, unsigned int *status, cudaStream_t s) {
    int *co = reinterpret_cast<int *>(static_cast<char *>(ws) + varlen_table_at(d, for_bwd));
    launch_begin(K_SEQ_TABLE, s);
    seq_table_kernel<<<1, 1024, 0, s>>>(d.cu, d.N, d.T, d.C, co, status);
    launch_end(K_SEQ_TABLE, s);
    d.co = co;
    return cudaGetLastError();
}

size_t gdn2_workspace_bytes_varlen(int N, int T, int H, int d_k, int d_v, int chunk, gdn2_io io, int for_bwd) {
    if (N < 1 || check_dims(1, T, H, d_k, d_v, chunk, io) != GDN2_OK) return 0;
    if (!use_tc(make_dims(1, T, H, d_k, d_v, chunk), io)) return 0;
    return varlen_ws_bytes(varlen_dims(N, T, H, d_k, d_v, chunk), for_bwd);
}

gdn2_status gdn2_fwd_varlen(const void *q, const void *k, const void *v, const void *g, const void *b,
                            const void *w, const float *S0, void *o, float *ST, void *ws, size_t ws_bytes,
                            const int *cu_seqlens, int N, int T, int H, int d_k, int d_v, int chunk,
                            gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    gdn2_status st = check_varlen(N, T, H, d_k, d_v, chunk, io, gate_io, cu_seqlens);
    if (st != GDN2_OK) return st;
    st = check_ptrs({q, k, v, g, b, w, o}, {S0, ST});
    if (st != GDN2_OK) return st;
    Dims d = varlen_dims(N, T, H, d_k, d_v, chunk);
    d.cu = cu_seqlens;
    d.gb = gate_io == GDN2_IO_BF16;
    if (!ws || !aligned16(ws) || ws_bytes < varlen_ws_bytes(d, 0)) return GDN2_ERR_WORKSPACE;
    unsigned int *status = status_word();
    if (!status) return GDN2_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const int keep = ws_bytes >= varlen_ws_bytes(d, 1);
    cudaError_t e = seq_table_launch(d, ws, keep, status, s);
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    return cuda_status(tc_fwd_launch(q, k, v, g, b, w, S0, o, ST, ws, keep, status, d, s));
}

gdn2_status gdn2_bwd_varlen(const void *q, const void *k, const void *v, const void *g, const void *b,
                            const void *w, const float *S0, const void *dO, const float *dST, void *dq,
                            void *dk, void *dv, void *dg, void *db, void *dw, float *dS0, void *ws,
                            size_t ws_bytes, int ws_has_fwd, const int *cu_seqlens, int N, int T, int H,
                            int d_k, int d_v, int chunk, gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    gdn2_status st = check_varlen(N, T, H, d_k, d_v, chunk, io, gate_io, cu_seqlens);
    if (st != GDN2_OK) return st;
    st = check_ptrs({q, k, v, g, b, w, dO, dq, dk, dv, dg, db, dw}, {S0, dST, dS0});
    if (st != GDN2_OK) return st;
    Dims d = varlen_dims(N, T, H, d_k, d_v, chunk);
    d.cu = cu_seqlens;
    d.gb = gate_io == GDN2_IO_BF16;
    if (!ws || !aligned16(ws) || ws_bytes < varlen_ws_bytes(d, 1)) return GDN2_ERR_WORKSPACE;
    unsigned int *status = status_word();
    if (!status) return GDN2_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = seq_table_launch(d, ws, 1, status, s);
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    if (!ws_has_fwd) {
        e = tc_fwd_launch(q, k, v, g, b, w, S0, nullptr, nullptr, ws, 1, status, d, s);
        if (e != cudaSuccess) return GDN2_ERR_CUDA;
    }
    return cuda_status(tc_bwd_launch(q, k, v, g, b, w, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, status,
                                     d, s));
}

gdn2_status gdn2_decode_step_ex(const void *q, const void *k, const void *v, const void *g,
                                const void *b, const void *w, float *S, void *o, int N, int H,
                                int d_k, int d_v, gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    if (N < 1 || H < 1 || (io != GDN2_IO_F32 && io != GDN2_IO_BF16)) return GDN2_ERR_INVALID_ARG;
    if (gate_io != GDN2_IO_F32 && gate_io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    if (!supported_d(d_k) || !supported_d(d_v)) return GDN2_ERR_UNSUPPORTED;
    if ((long long)N * H > 0x7fffffffLL) return GDN2_ERR_UNSUPPORTED;
    gdn2_status st = check_ptrs({q, k, v, g, b, w, S, o}, {});
    if (st != GDN2_OK) return st;
    return cuda_status(decode_launch(q, k, v, g, b, w, S, o, N, H, d_k, d_v, io, gate_io,
                                     (cudaStream_t)stream));
}

gdn2_status gdn2_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *b, const float *w, float *S, void *o, int N, int H,
                             int d_k, int d_v, gdn2_io io, gdn2_stream_t stream) {
    return gdn2_decode_step_ex(q, k, v, g, b, w, S, o, N, H, d_k, d_v, io, GDN2_IO_F32, stream);
}

// One block, one waiting thread: an mbarrier that no copy or product will
// complete, waited on with the same bounded wait the kernels use.
static __global__ void selftest_timeout_kernel(unsigned int *status, long long limit) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, limit)) record_status(status, GDN2_ERR_TIMEOUT);
}

gdn2_status gdn2_selftest_timeout(long long limit_cycles, gdn2_stream_t stream) {
    unsigned int *st = status_word();
    if (!st) return GDN2_ERR_CUDA;
    const long long lim = limit_cycles < 1000 ? 1000 : (limit_cycles > 4000000000LL ? 4000000000LL : limit_cycles);
    selftest_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(st, lim);
    return cuda_status(cudaGetLastError());
}

gdn2_status gdn2_get_device_status(gdn2_stream_t stream) {
    // one reader at a time: the taken value goes through one device slot
    std::lock_guard<std::mutex> lock(g_status_mu);
    cudaStream_t s = (cudaStream_t)stream;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    status_take_kernel<<<1, 1, 0, s>>>();
    unsigned int word = 0;
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&word, g_status_taken, sizeof(word), 0, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return GDN2_ERR_CUDA;
    return (gdn2_status)word;
}

const char *gdn2_status_string(gdn2_status status) {
    switch (status) {
        case GDN2_OK: return "ok";
        case GDN2_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size)";
        case GDN2_ERR_UNSUPPORTED: return "unsupported size (d_k, d_v in {32,64,128}; chunk in {16,32,64})";
        case GDN2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case GDN2_ERR_CUDA: return "CUDA error";
        case GDN2_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
        case GDN2_ERR_RANGE: return "an fp16 operand of the tensor-core path overflowed (see gdn2.h)";
    }
    return "unknown status";
}

int gdn2_version(void) { return 200; }

unsigned long long gdn2_kernel_launches(void) { return g_launches.load(); }

void gdn2_set_kernel_timer(int enable) {
    std::lock_guard<std::mutex> lock(g_timer_mu);
    for (auto &p : g_pending) {
        cudaEventDestroy(p.start);
        cudaEventDestroy(p.end);
    }
    g_pending.clear();
    for (int i = 0; i < K_KINDS; ++i) {
        g_kind_count[i] = 0;
        g_kind_ms[i] = 0.0;
    }
    g_timer_on.store(enable != 0);
}

int gdn2_kernel_kinds(void) { return K_KINDS; }

const char *gdn2_kernel_name(int id) { return id >= 0 && id < K_KINDS ? g_kind_names[id] : nullptr; }

gdn2_status gdn2_kernel_times(unsigned long long *count, double *ms, int n) {
    std::lock_guard<std::mutex> lock(g_timer_mu);
    gdn2_status st = GDN2_OK;
    for (auto &p : g_pending) {
        float t = 0.f;
        if (cudaEventSynchronize(p.end) != cudaSuccess ||
            cudaEventElapsedTime(&t, p.start, p.end) != cudaSuccess)
            st = GDN2_ERR_CUDA;
        else {
            g_kind_count[p.kind] += 1;
            g_kind_ms[p.kind] += t;
        }
        cudaEventDestroy(p.start);
        cudaEventDestroy(p.end);
    }
    g_pending.clear();
    for (int i = 0; i < n && i < K_KINDS; ++i) {
        if (count) count[i] = g_kind_count[i];
        if (ms) ms[i] = g_kind_ms[i];
    }
    return st;
}

}  // extern "C"
