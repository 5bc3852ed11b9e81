"""Throughput of the Gated Delta Rule-2 operator on B200: one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one chunkwise forward (gdn2_fwd) plus one gate-aware backward
(gdn2_bwd, reusing the forward's workspace) over the training workload
B=4, T=4096, H=16, d_k=d_v=128, chunk 64, bf16 q/k/v/o/dO and float32 gates
and state, on seeded synthetic inputs already resident in HBM.  The metric is
tokens/s (B*T per step).  With N > 1 (torchrun, one rank per GPU, NCCL) every
rank runs its own batch of that shape (weak scaling: the (batch, head) units
are independent, so no data-path collective exists); ranks only meet at
barriers and at the max-over-ranks of the device time.

--impl reference times the fp64 CPU oracle (the only other implementation of
the operator: a token-by-token recurrence with reverse mode) on a bounded
sample of the same workload, on this host's cores.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD_INDEX = 2
METRIC = "GDR-2 fwd+bwd tokens/s (H16, dk=dv=128) and % of HBM/tensor roofline"
NAMES = ("q", "k", "v", "g", "b", "w", "S0")
def byte_model(gs: int = 4):
    """Algorithmic bytes per token-head at d = 128: bf16 q, k, v, o, dO, dq, dk,
    dv and gates g, b, w, dg, db, dw of gs bytes (4 float32, 2 bf16).  Returns
    (forward, backward, per-kernel), the per-kernel figures attributing each
    tensor to the kernel that first reads (or writes) it."""
    fwd = 3 * 128 * 2 + 3 * 128 * gs + 128 * 2
    bwd = 3 * 128 * 2 + 3 * 128 * gs + 128 * 2 + 3 * 128 * 2 + 3 * 128 * gs
    kern = {
        # q, k, g, b read
        "tc_prep": 2 * 128 * 2 + 2 * 128 * gs,
        # v, w read; o written
        "tc_fwd": 128 * 2 + 128 * gs + 128 * 2,
        # q, k, g, b, dO, v, w read; dv, dw written
        "tc_bwd_state": 2 * 128 * 2 + 2 * 128 * gs + 128 * 2 + 128 * 2 + 128 * gs + 128 * 2 + 128 * gs,
        # dq, dk, db, dg written
        "tc_bwd_grad": 2 * 128 * 2 + 2 * 128 * gs,
    }
    assert kern["tc_prep"] + kern["tc_fwd"] == fwd and kern["tc_bwd_state"] + kern["tc_bwd_grad"] == bwd
    return fwd, bwd, kern


# float32 gates: 2560 + 4864 = 7424; bf16 gates: 1792 + 3328 = 5120
FWD_BYTES, BWD_BYTES, KERNEL_BYTES = byte_model(4)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=8)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-sub", action="store_true",
                   help="skip the workload 1 and 3 sub-objects of the default line")
    p.add_argument("--batch", type=int, default=None,
                   help="override B (smaller cases for profiling captures only)")
    p.add_argument("--workload", type=int, choices=[1, 2, 3], default=2,
                   help="2 = fwd+bwd B4 T4096 (the default line), 3 = fwd+bwd B1 T16384, "
                        "1 = forward only B8 T2048 (a line of its own metric)")
    return p.parse_args()


def cores() -> int:
    return max(1, len(os.sched_getaffinity(0)))


# ------------------------------------------------------------ clock sampling

class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for t, line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((t, parts))
        inside = [r for t, r in rows if self.t0 - 0.15 <= t <= self.t1 + 0.15] or [r for _, r in rows]
        mhz = [float(r[1]) for r in inside if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in inside if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in inside for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(inside)}


# ------------------------------------------------------------------ our arm

def traffic_from_profiles(kernel_key: str, src_hash: str):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.json),
    only if the kernel's sources are unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(kernel_key)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("src_sha256") != src_hash:
        return None
    return rec.get("dram_bytes_per_launch")


# the files that make up each tensor-core kernel whose DRAM traffic
# profiles/traffic.json records; a kernel's captured figure applies while these
# match (the shared headers count for every kernel)
TC_SHARED_SOURCES = ("common.cuh", "tc.cuh", "tc_common.cuh", "tmap.cuh")
TC_KERNEL_SOURCES = {"tc_prep": ("tc_prep.cu",), "tc_fwd": ("tc_fwd.cu",),
                     "tc_bwd_state": ("tc_bwd.cu",), "tc_bwd_grad": ("tc_bwd_grad.cu",)}


def sources_hash(kernel_key: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_128_b200", "csrc")
    for n in TC_KERNEL_SOURCES[kernel_key] + TC_SHARED_SOURCES:
        h.update(open(os.path.join(csrc, n), "rb").read())
    return h.hexdigest()


def _peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peaks = json.load(open(path)) if os.path.exists(path) else {}
    return peaks.get("hbm_gbs", 6650.0), ("of measured" if "hbm_gbs" in peaks else "of fallback")


def kernel_split(gdn, run_steps, steps, token_heads, peak, stream, kernel_bytes=None):
    """Per-kernel device time from the library's event timer, taken in a pass
    of its own (the timer records two events around every launch, so it is
    never on while a headline number is timed)."""
    import torch

    torch.cuda.synchronize()
    gdn.gdn2_set_kernel_timer(True)
    run_steps(steps)
    torch.cuda.synchronize()
    ktimes = gdn.gdn2_kernel_times()
    gdn.gdn2_set_kernel_timer(False)
    kernels = {}
    for name, (cnt, tot) in ktimes.items():
        # a kernel may launch more than once a step (the split state passes):
        # its algorithmic bytes are per step, so its rate is taken per step
        ent = {"launches": cnt, "avg_ms": tot / cnt, "ms_per_step": tot / steps}
        per = (kernel_bytes or KERNEL_BYTES).get(name)
        if per is not None:
            gbs = per * token_heads / (tot / steps * 1e-3) / 1e9
            ent.update(alg_bytes_per_step=per * token_heads, achieved_gbs=gbs, frac=gbs / peak)
        kernels[name] = ent
    return kernels


class FwdBwdCase:
    """Device buffers and the fwd+bwd step of one workload shape (bf16 I/O,
    float32 or bf16 gates, float32 state), inputs resident in HBM."""

    def __init__(self, wl, B, seed, dev, with_bwd=True, gates="f32"):
        import torch

        import gated_delta_rule_128_b200 as gdn
        from gated_delta_rule_128_b200 import workloads

        self.gdn, self.wl, self.dev = gdn, wl, dev
        self.B, self.T, self.H, self.dk, self.dv, self.C = B, wl.T, wl.H, wl.dk, wl.dv, wl.chunk
        self.with_bwd = with_bwd
        x = workloads.draw(B, wl.T, wl.H, wl.dk, wl.dv, seed, s0_std=wl.s0_std,
                           erase_scale=wl.erase_scale, with_dO=with_bwd)
        bf = torch.bfloat16
        io_names = ("q", "k", "v", "dO")
        gate_t = bf if gates == "bf16" else torch.float32
        self.host = {n: (t.to(bf) if n in io_names else t.to(gate_t) if n in ("g", "b", "w") else t)
                     .contiguous() for n, t in x.items()}
        self.gate_io = gdn.GDN2_IO_BF16 if gates == "bf16" else gdn.GDN2_IO_F32
        self.fwd_bytes, self.bwd_bytes, self.kernel_bytes = byte_model(2 if gates == "bf16" else 4)
        self.d = {n: t.to(dev) for n, t in self.host.items()}
        self.io = gdn.GDN2_IO_BF16
        self.ws = gdn.workspace(B, wl.T, wl.H, wl.dk, wl.dv, wl.chunk, self.io, with_bwd, dev)
        self.o = torch.empty(B, wl.T, wl.H, wl.dv, dtype=bf, device=dev)
        self.ST = None if with_bwd else torch.empty(B, wl.H, wl.dk, wl.dv, device=dev)
        d = self.d
        self.grads = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]),
                          dv=torch.empty_like(d["v"]), dg=torch.empty_like(d["g"]),
                          db=torch.empty_like(d["b"]), dw=torch.empty_like(d["w"])) if with_bwd else {}
        self.stream = torch.cuda.current_stream(dev)

    @property
    def token_heads(self):
        return self.B * self.T * self.H

    def fwd(self, inp=None, out=None):
        inp, out = inp or self.d, out or dict(o=self.o, **self.grads)
        g = self.gdn
        g.gdn2_fwd_ex(*(inp[n] for n in NAMES), out["o"], self.ST, self.ws, self.ws.numel(), self.B,
                      self.T, self.H, self.H, self.dk, self.dv, self.C, self.io, self.gate_io, self.stream)

    def bwd(self, inp=None, out=None):
        inp, out = inp or self.d, out or dict(o=self.o, **self.grads)
        self.gdn.gdn2_bwd_ex(*(inp[n] for n in NAMES), inp["dO"], None, out["dq"], out["dk"],
                             out["dv"], out["dg"], out["db"], out["dw"], None, self.ws,
                             self.ws.numel(), 1, self.B, self.T, self.H, self.H, self.dk, self.dv,
                             self.C, self.io, self.gate_io, self.stream)

    def step(self, inp=None, out=None):
        self.fwd(inp, out)
        if self.with_bwd:
            self.bwd(inp, out)

    def run(self, n):
        for _ in range(n):
            self.step()

    def timed(self, steps, warmup, barrier=lambda: None):
        """(ms per step, fwd ms, bwd ms, launches) over `steps` device-timed
        steps after `warmup` untimed ones; the kernel timer is off."""
        import torch

        for _ in range(max(3, warmup)):
            self.step()
        torch.cuda.synchronize(self.dev)
        if self.gdn.gdn2_get_device_status(self.stream) != 0:
            raise RuntimeError("device status reports an error after warm-up")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(self.dev)
        launches0 = self.gdn.gdn2_kernel_launches()
        start.record(self.stream)
        for i in range(steps):
            e0, e1, e2 = ev[i]
            e0.record(self.stream)
            self.fwd()
            e1.record(self.stream)
            if self.with_bwd:
                self.bwd()
            e2.record(self.stream)
        end.record(self.stream)
        torch.cuda.synchronize(self.dev)
        launches = self.gdn.gdn2_kernel_launches() - launches0
        barrier()
        if self.gdn.gdn2_get_device_status(self.stream) != 0:
            raise RuntimeError("device status reports an error after the timed region")
        fwd_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
        bwd_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
        return start.elapsed_time(end) / steps, fwd_ms, bwd_ms, launches


def sub_workload(index, args, rank, dev, peak, peak_src, gates="f32"):
    """A secondary workload of the default line (1: forward only B8 T2048;
    3: fwd+bwd B1 T16384 with b in [0, 2]; 2 with bf16 gates), device-timed
    like the headline."""
    import torch

    from gated_delta_rule_128_b200 import dist as gd
    from gated_delta_rule_128_b200 import workloads

    wl = workloads.WORKLOADS[index]
    case = FwdBwdCase(wl, wl.B, gd.rank_seed(wl.seed, rank), dev, with_bwd=wl.backward, gates=gates)
    steps = max(5, args.steps // 2)
    ms, fwd_ms, bwd_ms, _ = case.timed(steps, args.warmup, gd.barrier)
    kernels = kernel_split(case.gdn, case.run, steps, case.token_heads, peak, case.stream,
                           case.kernel_bytes)
    ms = gd.max_over_ranks([ms], dev)[0]
    if wl.backward:
        alg = case.token_heads * (case.fwd_bytes + case.bwd_bytes)
    else:  # the forward's bytes per token-head plus S0 read and S_T written
        alg = case.token_heads * case.fwd_bytes + 2 * wl.B * wl.H * wl.dk * wl.dv * 4
    gbs = alg / (ms * 1e-3) / 1e9
    name = wl.name + (" bf16 gates" if gates == "bf16" else "")
    out = {"workload": name, "ms_per_step": ms, "steps": steps,
           "tokens_per_s": wl.B * wl.T / (ms * 1e-3),
           "roofline_step": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                             "frac": gbs / peak, "alg_bytes_per_step": alg,
                             "peak_source": peak_src},
           "kernels": kernels}
    if wl.backward:
        out.update(fwd_ms=fwd_ms, bwd_ms=bwd_ms)
    del case
    torch.cuda.empty_cache()
    return out


def sub_packed(args, rank, dev, peak, peak_src):
    """Workload 2's 16384 tokens per head as one packed row of sequences of
    mixed lengths (uniform in [1, 2048], seeded), fwd+bwd through the packed
    entry points: the step a training run on packed documents takes."""
    import torch

    import gated_delta_rule_128_b200 as gdn
    from gated_delta_rule_128_b200 import dist as gd
    from gated_delta_rule_128_b200 import workloads

    wl = workloads.WORKLOADS[2]
    T, H, dk, dv, C = wl.B * wl.T, wl.H, wl.dk, wl.dv, wl.chunk
    seed = gd.rank_seed(1005, rank)
    lens = workloads.packed_lengths(T, seed)
    N = len(lens)
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32, device=dev)
    x = workloads.draw(1, T, H, dk, dv, seed)
    bf = torch.bfloat16
    d = {n: (t.to(bf) if n in ("q", "k", "v", "dO") else t).contiguous().to(dev) for n, t in x.items()}
    io, gio = gdn.GDN2_IO_BF16, gdn.GDN2_IO_F32
    ws = torch.empty(gdn.gdn2_workspace_bytes_varlen(N, T, H, H, dk, dv, C, io, gio, 1), dtype=torch.uint8,
                     device=dev)
    o = torch.empty(1, T, H, dv, dtype=bf, device=dev)
    gr = {n: torch.empty_like(d[m]) for n, m in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"),
                                                 ("db", "b"), ("dw", "w"))}
    stream = torch.cuda.current_stream(dev)
    names = ("q", "k", "v", "g", "b", "w")

    def step():
        gdn.gdn2_fwd_varlen(*(d[n] for n in names), None, o, None, ws, ws.numel(), cu, N, T, H, H, dk, dv,
                            C, io, gio, stream)
        gdn.gdn2_bwd_varlen(*(d[n] for n in names), None, d["dO"], None, gr["dq"], gr["dk"], gr["dv"],
                            gr["dg"], gr["db"], gr["dw"], None, ws, ws.numel(), 1, cu, N, T, H, H, dk, dv,
                            C, io, gio, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if gdn.gdn2_get_device_status(stream) != 0:
        raise RuntimeError("device status reports an error in the packed workload")
    steps = max(5, args.steps // 2)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gd.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    gd.barrier()
    ms = gd.max_over_ranks([start.elapsed_time(end) / steps], dev)[0]
    alg = T * H * (FWD_BYTES + BWD_BYTES)
    gbs = alg / (ms * 1e-3) / 1e9
    out = {"workload": f"fwd+bwd packed {N} sequences (lengths 1..2048, {T} tokens) H{H} d{dk} C{C} bf16",
           "ms_per_step": ms, "steps": steps, "tokens_per_s": T / (ms * 1e-3),
           "sequences": N, "longest": max(lens), "shortest": min(lens),
           "roofline_step": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                             "frac": gbs / peak, "alg_bytes_per_step": alg, "peak_source": peak_src}}
    del ws, d, gr
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch

    import gated_delta_rule_128_b200 as gdn
    from gated_delta_rule_128_b200 import dist as gd
    from gated_delta_rule_128_b200 import workloads

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workloads.WORKLOADS[WORKLOAD_INDEX]
    B = args.batch or wl.B
    case = FwdBwdCase(wl, B, gd.rank_seed(wl.seed, rank), dev)
    T, H, dk, dv = wl.T, wl.H, wl.dk, wl.dv
    peak, peak_src = _peak()
    host = {n: t.pin_memory() for n, t in case.host.items()}

    sampler = ClockSampler(local_rank)
    sampler.start()
    sampler.mark_start()
    ms_step, fwd_ms, bwd_ms, launches = case.timed(args.steps, args.warmup, gd.barrier)
    sampler.mark_end()
    # the per-kernel split, in a pass of its own
    kernels = kernel_split(gdn, case.run, args.steps, case.token_heads, peak, case.stream)
    kernel_steps = args.steps

    # end-to-end through host buffers: every step copies its inputs H2D from
    # pinned memory and its outputs D2H.  The input copies run on one stream,
    # the step on the launch stream and the output copies on a third, with two
    # sets of device buffers, so that step i's D2H overlaps step i+1's H2D
    # (PCIe moves both directions at once).  The timed region spans the first
    # H2D to the last D2H.
    d, stream = case.d, case.stream
    outs = [dict(o=torch.empty_like(case.o), **{n: torch.empty_like(t) for n, t in case.grads.items()})
            for _ in range(2)]
    host_out = [{n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in ob.items()}
                for ob in outs]
    h2d = sum(t.numel() * t.element_size() for n, t in host.items() if n != "S0")
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    stage = [{n: (d[n] if n == "S0" else torch.empty_like(t)) for n, t in d.items()} for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ev_in, ev_done, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    gd.barrier()
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(args.e2e_steps):
        k = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[k])  # step i - 2 has read this stage
            for n, t in host.items():
                if n != "S0":
                    stage[k][n].copy_(t, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if i >= 2:
            stream.wait_event(ev_out[k])  # step i - 2's outputs have left these buffers
        case.step(stage[k], outs[k])
        ev_done[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[k])
            for n, t in outs[k].items():
                host_out[k][n].copy_(t, non_blocking=True)
            ev_out[k].record(s_out)
    stream.wait_stream(s_out)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e_start.elapsed_time(e_end) / args.e2e_steps
    gd.barrier()
    clocks = sampler.stop()
    if gdn.gdn2_get_device_status(stream) != 0:
        raise RuntimeError("device status reports an error after the end-to-end steps")
    del outs, host_out, stage
    token_heads = case.token_heads
    del case
    torch.cuda.empty_cache()

    decode = run_decode(args, rank, dev) if not args.no_decode else None
    subs = {} if (args.no_sub or WORKLOAD_INDEX != 2) else {
        f"workload{i}": sub_workload(i, args, rank, dev, peak, peak_src) for i in (1, 3)}
    if subs:
        subs["workload2_bf16_gates"] = sub_workload(2, args, rank, dev, peak, peak_src, gates="bf16")
        subs["packed"] = sub_packed(args, rank, dev, peak, peak_src)
    ms_step, e2e_ms, fwd_ms, bwd_ms = gd.max_over_ranks([ms_step, e2e_ms, fwd_ms, bwd_ms], dev)
    if decode is not None:
        decode["us_per_step"] = gd.max_over_ranks([decode["us_per_step"]], dev)[0]
    tokens = B * T * world
    value = tokens / (ms_step * 1e-3)
    alg_bytes = token_heads * (FWD_BYTES + BWD_BYTES)
    for n, kd in kernels.items():
        kd["traffic"] = (traffic_from_profiles(n, sources_hash(n)) if n in TC_KERNEL_SOURCES else None)
    dom = max(kernels, key=lambda n: kernels[n]["ms_per_step"])
    dk_ = kernels[dom]
    per_step = dk_["launches"] / max(1, kernel_steps)  # launches of the kernel in one step
    roofline = {"bound": "hbm", "kernel": dom, "achieved": dk_.get("achieved_gbs"), "peak": peak,
                "unit": "GB/s", "frac": dk_.get("frac"), "peak_source": peak_src,
                "alg_bytes_per_launch": (dk_["alg_bytes_per_step"] / per_step
                                         if dk_.get("alg_bytes_per_step") is not None else None),
                "avg_launch_ms": dk_["avg_ms"],
                "traffic": dk_["traffic"]}
    step_achieved = alg_bytes / (ms_step * 1e-3) / 1e9
    roofline_step = {"bound": "hbm", "achieved": step_achieved, "peak": peak, "unit": "GB/s",
                     "frac": step_achieved / peak, "alg_bytes_per_step": alg_bytes,
                     "peak_source": peak_src}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic (seeded workload generators)",
        "config": {"workload": wl.name if B == wl.B else f"{wl.name}, B overridden to {B}",
                   "B": B, "T": T, "H": H, "d_k": dk, "d_v": dv,
                   "chunk": wl.chunk, "io": "bf16 q/k/v/o/dO/dq/dk/dv, f32 g/b/w/state",
                   "global_batch": B * world, "seq_len": T, "parallelism": f"dp{world}",
                   "l2": f"inputs {h2d / 1e9:.2f} GB per step (> 126 MB L2), no flush",
                   "arithmetic": "fp16 and tf32 tensor-core operands, fp32 accumulation and state"},
        "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
        "roofline": roofline,
        "roofline_step": roofline_step,
        "kernels": kernels,
        "kernel_timing": "per-kernel split from a separate pass of the same steps with the "
                         "library's event timer on; the headline region runs with it off",
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "copies": "pinned host buffers; H2D, step and D2H on three streams with two "
                          "device buffer sets, step i's D2H overlapping step i+1's H2D"},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if decode is not None:
        us = decode["us_per_step"]
        dec_bytes = decode["bytes_per_step"]
        gbs = dec_bytes / (us * 1e-6) / 1e9
        decode.update(tokens_per_s=decode["N"] * world / (us * 1e-6),
                      roofline={"bound": "hbm", "kernel": "decode_step", "achieved": gbs,
                                "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                                "alg_bytes_per_launch": dec_bytes, "peak_source": peak_src})
        line["decode"] = decode
    line.update(subs)
    return line


def run_decode(args, rank, dev):
    """Recurrent decode, workload 4 (256 sequences x 16 heads, d = 128, bf16
    q/k/v/o, f32 gates and state): 1024 consecutive steps captured in one CUDA
    graph and replayed on the stream the events are recorded on, inputs of 8
    seeded steps cycled, state resident in HBM."""
    import torch

    import gated_delta_rule_128_b200 as gdn
    from gated_delta_rule_128_b200 import dist as gd
    from gated_delta_rule_128_b200 import workloads

    wl = workloads.WORKLOADS[4]
    N, H, dk, dv = wl.B, wl.H, wl.dk, wl.dv
    seed = gd.rank_seed(wl.seed, rank)
    S = workloads.decode_state(N, H, dk, dv, seed, wl.s0_std).to(dev)
    steps = []
    for st in range(8):
        x = workloads.decode_step_inputs(N, H, dk, dv, seed, st)
        steps.append({n: (t.to(torch.bfloat16) if n in ("q", "k", "v") else t).to(dev)
                      for n, t in x.items()})
    o = torch.empty(N, H, dv, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)
    io = gdn.GDN2_IO_BF16

    def run(n):
        for i in range(n):
            d = steps[i % 8]
            gdn.gdn2_decode_step(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S, o, N, H, dk,
                                 dv, io, stream)

    nsteps = wl.decode_steps
    with torch.cuda.stream(stream):
        run(16)  # warm-up, eager
    torch.cuda.synchronize(dev)
    # thread-local capture: other threads' CUDA calls (a process group's
    # watchdog under torchrun) cannot invalidate it
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    how = "1024 consecutive steps in one CUDA graph"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
            run(nsteps)
        with torch.cuda.stream(stream):
            graph.replay()  # warm-up replay
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        del graph
    except RuntimeError as err:
        torch.cuda.synchronize(dev)
        how = f"1024 consecutive launches on one stream (graph capture failed: {str(err)[:80]})"
        e0.record(stream)
        run(nsteps)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / nsteps
    if gdn.gdn2_get_device_status() != 0:
        raise RuntimeError("device status reports an error after decode")
    per_head = 2 * dk * dv * 4 + (2 * dk + dv) * 2 + (2 * dk + dv) * 4 + dv * 2
    return {"workload": wl.name, "N": N, "H": H, "steps": nsteps,
            "us_per_step": us, "bytes_per_step": per_head * N * H,
            "inputs": "8 seeded steps cycled; " + how}


def run_forward_only(args, rank, world, local_rank):
    """Workload 1 as a line of its own: the forward alone (bf16 q/k/v/o, f32
    gates and state, S0 ~ N(0, 0.02), B8 T2048 H16 d128 C64), device-timed per
    call; algorithmic bytes are the forward's per token-head plus S0 read and
    S_T written."""
    import torch

    from gated_delta_rule_128_b200 import dist as gd
    from gated_delta_rule_128_b200 import workloads

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workloads.WORKLOADS[1]
    B = args.batch or wl.B
    case = FwdBwdCase(wl, B, gd.rank_seed(wl.seed, rank), dev, with_bwd=False)
    peak, _ = _peak()
    ms, _, _, launches = case.timed(args.steps, args.warmup, gd.barrier)
    kernels = kernel_split(case.gdn, case.run, args.steps, case.token_heads, peak, case.stream)
    ms = gd.max_over_ranks([ms], dev)[0]
    alg = case.token_heads * FWD_BYTES + 2 * B * wl.H * wl.dk * wl.dv * 4
    gbs = alg / (ms * 1e-3) / 1e9
    return {
        "metric": "GDR-2 fwd tokens/s (H16, dk=dv=128) and % of HBM roofline", "value": B * wl.T * world / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic (seeded workload generators)",
        "config": {"workload": wl.name, "B": B, "T": wl.T, "H": wl.H, "d_k": wl.dk, "d_v": wl.dv,
                   "chunk": wl.chunk},
        "roofline_step": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                          "alg_bytes_per_step": alg},
        "kernels": kernels, "gpu_launches": launches,
    }


# -------------------------------------------------------------- oracle arm

def oracle_sample(seconds_budget: float, nthreads: int):
    """Time the fp64 oracle (forward + reverse mode) on whole sequences of
    (batch, head) pairs of the workload: about `seconds_budget` of work on
    `nthreads` threads.  Returns (tokens/s scaled to the workload's H heads,
    sample text, seconds)."""
    import numpy as np

    import oracle
    from gated_delta_rule_128_b200 import workloads

    wl = workloads.WORKLOADS[WORKLOAD_INDEX]
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    global _ORACLE_INPUTS
    if _ORACLE_INPUTS is None:
        x = workloads.draw_workload(WORKLOAD_INDEX)
        for n in ("q", "k", "v", "dO"):
            x[n] = workloads.round_bf16(x[n])
        # (b, h) pairs as heads of one batch row: [1, T, B*H, D]
        _ORACLE_INPUTS = {n: t.permute(1, 0, 2, 3).reshape(T, B * H, -1)[None].contiguous()
                          for n, t in x.items() if n != "S0"}
    x = _ORACLE_INPUTS

    def run(npairs, threads):
        sl = {n: np.ascontiguousarray(t[:, :, :npairs].double().numpy()) for n, t in x.items()}
        S0 = np.zeros((1, npairs, dk, dv))
        t0 = time.perf_counter()
        oracle.forward(sl["q"], sl["k"], sl["v"], sl["g"], sl["b"], sl["w"], S0, nthreads=threads)
        oracle.backward(sl["q"], sl["k"], sl["v"], sl["g"], sl["b"], sl["w"], S0, sl["dO"], None,
                        nthreads=threads)
        return time.perf_counter() - t0

    per_pair = run(1, 1)                       # one whole sequence, one thread
    waves = max(1, int(seconds_budget / per_pair))
    pairs = int(min(B * H, max(1, nthreads) * waves))
    elapsed = run(pairs, nthreads)
    tokens_per_s = pairs * T / H / elapsed
    sample = (f"{pairs} of the {B * H} (batch, head) sequences of {wl.name} (all {T} tokens), "
              f"fp64 forward + reverse mode, {nthreads} threads, {elapsed:.1f} s")
    return tokens_per_s, sample, elapsed


_ORACLE_INPUTS = None


def run_reference(args, rank, world):
    """The oracle arm: rank 0 only."""
    if rank != 0:
        return None
    n = cores()
    total = max(1, args.steps + max(3, args.warmup))
    per_step = max(0.5, min(20.0, 150.0 / total))
    vals = []
    sample = ""
    for i in range(total):
        v, sample, _ = oracle_sample(per_step, n)
        if i >= max(3, args.warmup):
            vals.append(v)
    value = statistics.mean(vals)
    from gated_delta_rule_128_b200 import workloads
    wl = workloads.WORKLOADS[WORKLOAD_INDEX]
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded workload generators)",
        "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "H": wl.H, "d_k": wl.dk,
                   "d_v": wl.dv, "chunk": wl.chunk, "global_batch": wl.B * world,
                   "seq_len": wl.T, "parallelism": f"dp{world}"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": n, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    global WORKLOAD_INDEX
    args = parse()
    WORKLOAD_INDEX = args.workload
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    from gated_delta_rule_128_b200 import dist as gd
    gd.init("nccl", gd.rank_info(), timeout_s=120)
    if args.workload == 1:
        try:
            line = run_forward_only(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(line), flush=True)
        finally:
            gd.shutdown()
        return
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v, sample, _ = oracle_sample(15.0, cores())
            line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores(),
                                    "kind": "oracle", "sample": sample}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        gd.shutdown()


if __name__ == "__main__":
    main()
