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
                          const void *, float *, void *, int, int, int, int, int, gdn2_io, gdn2_io, int,
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
    "simt_chunk_bwd_b", "decode_step", "tc_prep", "tc_fwd", "tc_bwd_state", "tc_bwd_grad", "seq_table",
    "permute_state", "seg_link"};

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
    return Dims{B, T, H, dk, dv, chunk, (T + chunk - 1) / chunk, 0, 0};
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

// gate_io: the gate tensors' type in its low byte, GDN2_GATE_* flags above it
static gdn2_io gate_type(gdn2_io gate_io) { return (gdn2_io)((int)gate_io & 0xff); }
static int gate_flags(gdn2_io gate_io) { return ((int)gate_io >> 8) & 3; }
static bool gate_io_valid(gdn2_io gate_io) {
    const int t = (int)gate_io & 0xff, f = (int)gate_io >> 8;
    return (t == GDN2_IO_F32 || t == GDN2_IO_BF16) && (f & ~3) == 0 && (f != 2);  // B_X2 needs LOGITS
}
// gate tensors in bf16, and gate logits, need the tensor-core path
static gdn2_status check_gate_io(const Dims &d, gdn2_io io, gdn2_io gate_io) {
    if (!gate_io_valid(gate_io)) return GDN2_ERR_INVALID_ARG;
    if ((gate_type(gate_io) == GDN2_IO_BF16 || gate_flags(gate_io) != 0) && !use_tc(d, io))
        return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}

// ------------------------------------------------------ grouped value heads
// H_v value heads over H key heads, G = H_v / H consecutive value heads per
// key head.  Value head h G + j reads q, k, g, b of key head h, so the G
// states of a key head evolve as one state of G d_v columns: the kernels run
// that wide problem (d_v' = G d_v) on v, w, o, dO, dv, dw unchanged in memory
// ([.., H_v, d_v] is [.., H, G d_v]).  Only the states are laid out per value
// head, [S, H_v, d_k, d_v]; they pass through the wide layout [S, H, d_k, G d_v]
// in two workspace buffers.
static int value_groups(int H, int H_v) {
    if (H_v == 0 || H_v == H) return 1;
    if (H_v < H || H_v % H != 0) return 0;
    return H_v / H;
}

// state layouts: per value head [S][H G][dk][dvh]  <->  wide [S][H][dk][G dvh]
static __global__ void permute_state_kernel(const float *src, float *dst, long long total, int G, int dk,
                                            int dvh, int to_wide) {
    const int dvw = G * dvh;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int col = (int)(i % dvw), key = (int)((i / dvw) % dk);
        const long long sh = i / ((long long)dvw * dk);  // s H + h
        const long long j = ((sh * G + col / dvh) * dk + key) * dvh + col % dvh;
        if (to_wide) dst[i] = src[j];
        else dst[j] = src[i];
    }
}
static cudaError_t permute_state(const float *src, float *dst, const Dims &d, int G, int to_wide, cudaStream_t s) {
    const long long total = (long long)num_seqs(d) * d.H * d.dk * d.dv;
    const int blocks = (int)((total + 255) / 256 < 4 * sm_count() ? (total + 255) / 256 : 4 * sm_count());
    launch_begin(K_PERMUTE_STATE, s);
    permute_state_kernel<<<blocks, 256, 0, s>>>(src, dst, total, G, d.dk, d.dv / G, to_wide);
    launch_end(K_PERMUTE_STATE, s);
    return cudaGetLastError();
}
static size_t state_bytes(const Dims &d) { return align256((size_t)num_seqs(d) * d.H * d.dk * d.dv * sizeof(float)); }

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

// ------------------------------------------------------------ one call
// The problem after the host checks: the (wide) sizes, the path, and the
// workspace regions that follow the path's own layout: the packed
// sequences' chunk table, then two wide state buffers when G > 1.
struct Call {
    Dims d;
    gdn2_io io;
    int G;
    int for_bwd;
    size_t table_at, states_at, total;
};

// packed: N sequences of the table cu (which only a launch reads; sizing
// passes none)
static gdn2_status plan_call(Call &c, int B, int T, int H, int H_v, int dk, int dv, int chunk, gdn2_io io,
                             gdn2_io gate_io, bool packed, int N, const int *cu, int for_bwd) {
    c.G = value_groups(H, H_v);
    if (c.G == 0 || H < 1) return GDN2_ERR_INVALID_ARG;
    if (c.G > 1 && !supported_d(dv)) return GDN2_ERR_UNSUPPORTED;
    const int dvw = c.G * dv;
    gdn2_status st = check_dims(packed ? 1 : B, T, H, dk, dvw, chunk, io);
    if (st != GDN2_OK) return st;
    c.io = io;
    c.for_bwd = for_bwd;
    c.d = make_dims(packed ? 1 : B, T, H, dk, dvw, chunk);
    if ((st = check_gate_io(c.d, io, gate_io)) != GDN2_OK) return st;
    c.d.gb = gate_type(gate_io) == GDN2_IO_BF16;
    c.d.act = gate_flags(gate_io);
    size_t o;
    if (packed) {
        if (N < 1 || ((uintptr_t)cu & 3u) != 0) return GDN2_ERR_INVALID_ARG;
        if (!use_tc(c.d, io)) return GDN2_ERR_UNSUPPORTED;
        if (N > 65535 || (long long)H * ((T + chunk - 1) / chunk + N) > 0x7fffffffLL) return GDN2_ERR_UNSUPPORTED;
        c.d.NC = (T + chunk - 1) / chunk + N;  // bounds the chunks of N sequences over T tokens
        c.d.N = N;
        c.d.cu = cu;
        const TcWs t = tc_ws_layout(c.d);
        c.table_at = for_bwd ? t.bwd_end : t.rec_end;
        o = c.table_at + align256((size_t)(N + 1) * sizeof(int));
    } else {
        c.table_at = 0;
        o = ws_bytes_for(c.d, io, for_bwd);
    }
    c.states_at = align256(o);
    c.total = c.G > 1 ? c.states_at + 2 * state_bytes(c.d) : o;
    return GDN2_OK;
}

static cudaError_t seq_table_launch(Call &c, void *ws, unsigned int *status, cudaStream_t s) {
    if (c.d.N == 0) return cudaSuccess;
    int *co = reinterpret_cast<int *>(static_cast<char *>(ws) + c.table_at);
    launch_begin(K_SEQ_TABLE, s);
    seq_table_kernel<<<1, 1024, 0, s>>>(c.d.cu, c.d.N, c.d.T, c.d.C, co, status);
    launch_end(K_SEQ_TABLE, s);
    c.d.co = co;
    return cudaGetLastError();
}
static float *state_buf(const Call &c, void *ws, int i) {
    return reinterpret_cast<float *>(static_cast<char *>(ws) + c.states_at + i * state_bytes(c.d));
}

static gdn2_status fwd_call(Call &c, const void *q, const void *k, const void *v, const void *g,
                            const void *b, const void *w, const float *S0, void *o, float *ST, void *ws,
                            size_t ws_bytes, gdn2_stream_t stream) {
    gdn2_status st = check_ptrs({q, k, v, g, b, w, o}, {S0, ST});
    if (st != GDN2_OK) return st;
    if (!ws || !aligned16(ws) || ws_bytes < c.total) return GDN2_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    // keep the forward for the backward when the workspace is the backward's
    Call full = c;
    if (!c.for_bwd) {
        Call cb;
        if (plan_call(cb, c.d.B, c.d.T, c.d.H, c.d.H * c.G, c.d.dk, c.d.dv / c.G, c.d.C, c.io,
                      (gdn2_io)((c.d.gb ? GDN2_IO_BF16 : GDN2_IO_F32) | (c.d.act << 8)), c.d.N > 0, c.d.N,
                      c.d.cu, 1) == GDN2_OK &&
            ws_bytes >= cb.total)
            full = cb;
    }
    const int keep = full.for_bwd;
    const float *wS0 = S0;
    float *wST = ST;
    cudaError_t e = cudaSuccess;
    if (full.G > 1) {
        if (S0) {
            wS0 = state_buf(full, ws, 0);
            if ((e = permute_state(S0, state_buf(full, ws, 0), full.d, full.G, 1, s)) != cudaSuccess) return GDN2_ERR_CUDA;
        }
        if (ST) wST = state_buf(full, ws, 1);
    }
    if (use_tc(full.d, full.io)) {
        unsigned int *status = status_word();
        if (!status) return GDN2_ERR_CUDA;
        if ((e = seq_table_launch(full, ws, status, s)) != cudaSuccess) return GDN2_ERR_CUDA;
        e = tc_fwd_launch(q, k, v, g, b, w, wS0, o, wST, ws, keep, status, full.d, s);
    } else {
        e = run_forward(q, k, v, static_cast<const float *>(g), static_cast<const float *>(b),
                        static_cast<const float *>(w), wS0, o, wST, ws, full.d, full.io, s);
    }
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    if (full.G > 1 && ST) e = permute_state(wST, ST, full.d, full.G, 0, s);
    return cuda_status(e);
}

static gdn2_status bwd_call(Call &c, const void *q, const void *k, const void *v, const void *g,
                            const void *b, const void *w, const float *S0, const void *dO, const float *dST,
                            void *dq, void *dk, void *dv, void *dg, void *db, void *dw, float *dS0, void *ws,
                            size_t ws_bytes, int ws_has_fwd, gdn2_stream_t stream) {
    gdn2_status st = check_ptrs({q, k, v, g, b, w, dO, dq, dk, dv, dg, db, dw}, {S0, dST, dS0});
    if (st != GDN2_OK) return st;
    if (!ws || !aligned16(ws) || ws_bytes < c.total) return GDN2_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const float *wS0 = S0, *wdST = dST;
    float *wdS0 = dS0;
    cudaError_t e = cudaSuccess;
    if (c.G > 1) {
        // S0 (read by a recomputed forward) and then dS0 share buffer 0: the
        // stream runs the forward's reads before the backward's writes
        if (S0 && !ws_has_fwd) {
            wS0 = state_buf(c, ws, 0);
            if ((e = permute_state(S0, state_buf(c, ws, 0), c.d, c.G, 1, s)) != cudaSuccess) return GDN2_ERR_CUDA;
        }
        if (dST) {
            wdST = state_buf(c, ws, 1);
            if ((e = permute_state(dST, state_buf(c, ws, 1), c.d, c.G, 1, s)) != cudaSuccess) return GDN2_ERR_CUDA;
        }
        if (dS0) wdS0 = state_buf(c, ws, 0);
    }
    if (use_tc(c.d, c.io)) {
        unsigned int *status = status_word();
        if (!status) return GDN2_ERR_CUDA;
        if ((e = seq_table_launch(c, ws, status, s)) != cudaSuccess) return GDN2_ERR_CUDA;
        if (!ws_has_fwd) {
            e = tc_fwd_launch(q, k, v, g, b, w, wS0, nullptr, nullptr, ws, 1, status, c.d, s);
            if (e != cudaSuccess) return GDN2_ERR_CUDA;
        }
        e = tc_bwd_launch(q, k, v, g, b, w, dO, wdST, dq, dk, dv, dg, db, dw, wdS0, ws, status, c.d, s);
    } else {
        const float *gf = static_cast<const float *>(g), *bf = static_cast<const float *>(b),
                    *wf = static_cast<const float *>(w);
        float *dgf = static_cast<float *>(dg), *dbf = static_cast<float *>(db), *dwf = static_cast<float *>(dw);
        if (!ws_has_fwd) {
            e = run_forward(q, k, v, gf, bf, wf, wS0, nullptr, nullptr, ws, c.d, c.io, s);
            if (e != cudaSuccess) return GDN2_ERR_CUDA;
        }
        if (c.io == GDN2_IO_BF16)
            e = simt_bwd_launch<__nv_bfloat16>(q, k, v, bf, wf, dO, wdST, dq, dk, dv, dgf, dbf, dwf, wdS0, ws,
                                               c.d, s);
        else
            e = simt_bwd_launch<float>(q, k, v, bf, wf, dO, wdST, dq, dk, dv, dgf, dbf, dwf, wdS0, ws, c.d, s);
    }
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    if (c.G > 1 && dS0) e = permute_state(wdS0, dS0, c.d, c.G, 0, s);
    return cuda_status(e);
}

size_t gdn2_workspace_bytes_ex(int B, int T, int H, int H_v, int d_k, int d_v, int chunk, gdn2_io io,
                               gdn2_io gate_io, int for_bwd) {
    Call c;
    if (plan_call(c, B, T, H, H_v, d_k, d_v, chunk, io, gate_io, false, 0, nullptr, for_bwd) != GDN2_OK) return 0;
    return c.total;
}

gdn2_status gdn2_fwd_ex(const void *q, const void *k, const void *v, const void *g, const void *b,
                        const void *w, const float *S0, void *o, float *ST, void *ws,
                        size_t ws_bytes, int B, int T, int H, int H_v, int d_k, int d_v, int chunk,
                        gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    Call c;
    gdn2_status st = plan_call(c, B, T, H, H_v, d_k, d_v, chunk, io, gate_io, false, 0, nullptr, 0);
    if (st != GDN2_OK) return st;
    return fwd_call(c, q, k, v, g, b, w, S0, o, ST, ws, ws_bytes, stream);
}

gdn2_status gdn2_fwd(const void *q, const void *k, const void *v, const float *g, const float *b,
                     const float *w, const float *S0, void *o, float *ST, void *ws,
                     size_t ws_bytes, int B, int T, int H, int d_k, int d_v, int chunk,
                     gdn2_io io, gdn2_stream_t stream) {
    return gdn2_fwd_ex(q, k, v, g, b, w, S0, o, ST, ws, ws_bytes, B, T, H, H, d_k, d_v, chunk, io,
                       GDN2_IO_F32, stream);
}

gdn2_status gdn2_bwd_ex(const void *q, const void *k, const void *v, const void *g, const void *b,
                        const void *w, const float *S0, const void *dO, const float *dST, void *dq,
                        void *dk, void *dv, void *dg, void *db, void *dw, float *dS0, void *ws,
                        size_t ws_bytes, int ws_has_fwd, int B, int T, int H, int H_v, int d_k, int d_v,
                        int chunk, gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    Call c;
    gdn2_status st = plan_call(c, B, T, H, H_v, d_k, d_v, chunk, io, gate_io, false, 0, nullptr, 1);
    if (st != GDN2_OK) return st;
    return bwd_call(c, q, k, v, g, b, w, S0, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, ws_bytes, ws_has_fwd,
                    stream);
}

gdn2_status gdn2_bwd(const void *q, const void *k, const void *v, const float *g, const float *b,
                     const float *w, const float *S0, const void *dO, const float *dST, void *dq,
                     void *dk, void *dv, float *dg, float *db, float *dw, float *dS0, void *ws,
                     size_t ws_bytes, int ws_has_fwd, int B, int T, int H, int d_k, int d_v,
                     int chunk, gdn2_io io, gdn2_stream_t stream) {
    return gdn2_bwd_ex(q, k, v, g, b, w, S0, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, ws_bytes,
                       ws_has_fwd, B, T, H, H, d_k, d_v, chunk, io, GDN2_IO_F32, stream);
}

size_t gdn2_workspace_bytes_varlen(int N, int T, int H, int H_v, int d_k, int d_v, int chunk, gdn2_io io,
                                   gdn2_io gate_io, int for_bwd) {
    Call c;
    if (plan_call(c, 1, T, H, H_v, d_k, d_v, chunk, io, gate_io, true, N, nullptr, for_bwd) != GDN2_OK) return 0;
    return c.total;
}

gdn2_status gdn2_fwd_varlen(const void *q, const void *k, const void *v, const void *g, const void *b,
                            const void *w, const float *S0, void *o, float *ST, void *ws, size_t ws_bytes,
                            const int *cu_seqlens, int N, int T, int H, int H_v, int d_k, int d_v, int chunk,
                            gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    if (!cu_seqlens) return GDN2_ERR_INVALID_ARG;
    Call c;
    gdn2_status st = plan_call(c, 1, T, H, H_v, d_k, d_v, chunk, io, gate_io, true, N, cu_seqlens, 0);
    if (st != GDN2_OK) return st;
    return fwd_call(c, q, k, v, g, b, w, S0, o, ST, ws, ws_bytes, stream);
}

gdn2_status gdn2_bwd_varlen(const void *q, const void *k, const void *v, const void *g, const void *b,
                            const void *w, const float *S0, const void *dO, const float *dST, void *dq,
                            void *dk, void *dv, void *dg, void *db, void *dw, float *dS0, void *ws,
                            size_t ws_bytes, int ws_has_fwd, const int *cu_seqlens, int N, int T, int H,
                            int H_v, int d_k, int d_v, int chunk, gdn2_io io, gdn2_io gate_io,
                            gdn2_stream_t stream) {
    if (!cu_seqlens) return GDN2_ERR_INVALID_ARG;
    Call c;
    gdn2_status st = plan_call(c, 1, T, H, H_v, d_k, d_v, chunk, io, gate_io, true, N, cu_seqlens, 1);
    if (st != GDN2_OK) return st;
    return bwd_call(c, q, k, v, g, b, w, S0, dO, dST, dq, dk, dv, dg, db, dw, dS0, ws, ws_bytes, ws_has_fwd,
                    stream);
}

gdn2_status gdn2_decode_step_ex(const void *q, const void *k, const void *v, const void *g,
                                const void *b, const void *w, float *S, void *o, int N, int H, int H_v,
                                int d_k, int d_v, gdn2_io io, gdn2_io gate_io, gdn2_stream_t stream) {
    if (N < 1 || H < 1 || (io != GDN2_IO_F32 && io != GDN2_IO_BF16)) return GDN2_ERR_INVALID_ARG;
    if (!gate_io_valid(gate_io)) return GDN2_ERR_INVALID_ARG;
    const int G = value_groups(H, H_v);
    if (G == 0) return GDN2_ERR_INVALID_ARG;
    if (!supported_d(d_k) || !supported_d(d_v)) return GDN2_ERR_UNSUPPORTED;
    if ((long long)N * H * G > 0x7fffffffLL) return GDN2_ERR_UNSUPPORTED;
    gdn2_status st = check_ptrs({q, k, v, g, b, w, S, o}, {});
    if (st != GDN2_OK) return st;
    return cuda_status(decode_launch(q, k, v, g, b, w, S, o, N, H, G, d_k, d_v, io, gate_type(gate_io),
                                     gate_flags(gate_io), (cudaStream_t)stream));
}

gdn2_status gdn2_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *b, const float *w, float *S, void *o, int N, int H,
                             int d_k, int d_v, gdn2_io io, gdn2_stream_t stream) {
    return gdn2_decode_step_ex(q, k, v, g, b, w, S, o, N, H, H, d_k, d_v, io, GDN2_IO_F32, stream);
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
