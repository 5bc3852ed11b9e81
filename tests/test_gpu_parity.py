"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs.

Tolerances (max|gpu - ref| / max|ref| per output tensor): float32 path 1e-4;
bf16-I/O path 5e-3 on o and S_T, 1e-2 on gradients.  bf16 inputs are rounded
once on the host and the oracle consumes exactly the rounded values.

Small cases span several chunks and a ragged tail; the five workloads run at
full size on the GPU and are compared on sampled (batch, head) pairs that the
oracle computes one by one.
"""

import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_128_b200 as gdn
from gated_delta_rule_128_b200 import workloads
from _util import TOL_BF16_GRAD, TOL_BF16_OUT, TOL_F32, io_round, rel, to_device, to_np64

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "g", "b", "w", "S0")
GRADS = ("dq", "dk", "dv", "dg", "db", "dw", "dS0")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gdn.lib()


def tols(io):
    return (TOL_F32, TOL_F32) if io == "f32" else (TOL_BF16_OUT, TOL_BF16_GRAD)


def gpu_fwd_bwd(x, io, chunk, backward=True, use_dST=True, gates="f32", encoding="activated"):
    d = to_device(x, io, gates=gates)
    o, ST, ws = gdn.forward(*(d[n] for n in NAMES), chunk=chunk, for_bwd=backward, gates=encoding)
    out = {"o": o, "ST": ST}
    if backward:
        gr = gdn.backward(*(d[n] for n in NAMES), d["dO"], d.get("dST") if use_dST else None,
                          chunk=chunk, ws=ws, ws_has_fwd=True, gates=encoding)
        out.update(gr)
    torch.cuda.synchronize()
    assert gdn.gdn2_get_device_status() == 0
    return {n: t.float().cpu().numpy() for n, t in out.items() if t is not None}


def oracle_fwd_bwd(x, io, backward=True, use_dST=True, pairs=None, gates="f32"):
    """Oracle on all (b, h) pairs, or on the listed ones (results stacked in
    the order given, as batch 1 with len(pairs) heads)."""
    if pairs is not None:
        x = {n: (torch.stack([t[bb, h] for bb, h in pairs])[None] if n in ("S0", "dST")
                 else torch.stack([t[bb, :, h] for bb, h in pairs], dim=1)[None]).contiguous()
             for n, t in x.items() if t.dim() == 4}
    r = to_np64(io_round(x, io, gates))
    o, ST = oracle.forward(*(r[n] for n in NAMES))
    out = {"o": o, "ST": ST}
    if backward:
        out.update(oracle.backward(*(r[n] for n in NAMES), r["dO"],
                                   r.get("dST") if use_dST else None, ckpt=64))
    return out


def compare(gpu, ref, io, names, pairs=None):
    tol_out, tol_grad = tols(io)
    errs = {}
    for n in names:
        a = gpu[n]
        if pairs is not None:
            if n in ("ST", "dS0"):
                a = np.stack([a[bb, h] for bb, h in pairs])[None]
            else:
                a = np.stack([a[bb, :, h] for bb, h in pairs], axis=1)[None]
        assert np.isfinite(a).all(), n
        errs[n] = rel(a, ref[n])
    bad = {n: e for n, e in errs.items()
           if e > (tol_out if n in ("o", "ST") else tol_grad)}
    assert not bad, f"parity failures {bad} (all: {errs})"
    return errs


# ------------------------------------------------------------- workload 0

def test_workload0_fp32_forward_backward():
    x = workloads.draw_workload(0)
    gpu = gpu_fwd_bwd(x, "f32", 64, use_dST=False)
    ref = oracle_fwd_bwd(x, "f32", use_dST=False)
    compare(gpu, ref, "f32", ("o", "ST") + GRADS)


@pytest.mark.parametrize("tie", ["kda", "gdn"])
def test_workload0_fp32_tied_gates(tie):
    """b = w = beta 1 gives KDA; a scalar decay as well gives Gated DeltaNet."""
    x = workloads.draw_workload(0, tie=tie)
    gpu = gpu_fwd_bwd({n: t for n, t in x.items() if n not in ("beta", "alpha_log")}, "f32", 64,
                      use_dST=False)
    r = to_np64(x)
    if tie == "kda":
        o, ST = oracle.kda_forward(r["q"], r["k"], r["v"], r["g"], r["beta"], r["S0"])
    else:
        o, ST = oracle.gdn_forward(r["q"], r["k"], r["v"], r["alpha_log"], r["beta"], r["S0"])
    assert rel(gpu["o"], o) < TOL_F32 and rel(gpu["ST"], ST) < TOL_F32
    ref = oracle.backward(*(r[n] for n in NAMES), r["dO"], None)
    compare(gpu, ref, "f32", GRADS)
    # the tied scalar's gradient: dbeta = sum_c db + sum_c dw
    dbeta = gpu["db"].sum(-1) + gpu["dw"].sum(-1)
    assert rel(dbeta, ref["db"].sum(-1) + ref["dw"].sum(-1)) < TOL_F32


@pytest.mark.parametrize("tie", ["kda", "gdn"])
def test_tensor_core_path_tied_gates(tie):
    """The ties on the tensor-core path (bf16, d = 128, chunk 64): b = w = beta 1
    reproduces KDA, and a scalar decay as well reproduces Gated DeltaNet, at the
    bf16 tolerances; the tied scalar's gradient is sum_c db + sum_c dw."""
    x = workloads.draw(1, 256, 2, 128, 128, 810 + len(tie), tie=tie, s0_std=0.1)
    xr = io_round({n: t for n, t in x.items() if n not in ("beta", "alpha_log")}, "bf16")
    gpu = gpu_fwd_bwd({n: t for n, t in x.items() if n not in ("beta", "alpha_log")}, "bf16", 64,
                      use_dST=False)
    r = to_np64(xr)
    beta, alpha = x["beta"].double().numpy(), x.get("alpha_log")
    if tie == "kda":
        o, ST = oracle.kda_forward(r["q"], r["k"], r["v"], r["g"], beta, r["S0"])
    else:
        o, ST = oracle.gdn_forward(r["q"], r["k"], r["v"], alpha.double().numpy(), beta, r["S0"])
    assert rel(gpu["o"], o) < TOL_BF16_OUT and rel(gpu["ST"], ST) < TOL_BF16_OUT
    ref = oracle.backward(*(r[n] for n in NAMES), r["dO"], None)
    compare(gpu, ref, "bf16", GRADS)
    dbeta = gpu["db"].sum(-1) + gpu["dw"].sum(-1)
    assert rel(dbeta, ref["db"].sum(-1) + ref["dw"].sum(-1)) < TOL_BF16_GRAD


# ------------------------------------------------------ small grids, ragged

CASES = [
    # B, T, H, dk, dv, chunk
    (2, 200, 2, 128, 128, 64),
    (1, 77, 3, 64, 128, 32),
    (2, 33, 2, 32, 64, 16),
    (1, 64, 2, 128, 32, 64),
    (1, 65, 1, 64, 64, 64),
    (3, 1, 2, 128, 128, 64),
    (1, 130, 2, 32, 32, 16),
]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}T{}H{}k{}v{}C{}".format(*c))
def test_small_grids(case, io):
    B, T, H, dk, dv, chunk = case
    x = workloads.draw(B, T, H, dk, dv, 500 + T + dk, s0_std=0.3, with_dST=True)
    gpu = gpu_fwd_bwd(x, io, chunk)
    ref = oracle_fwd_bwd(x, io)
    compare(gpu, ref, io, ("o", "ST") + GRADS)


# The tensor-core path (bf16, d = 128, chunk 64): one and two chunks, a ragged
# tail, more tiles than SMs with one chunk each, and several tiles per
# persistent CTA; non-zero S0 and dS_T throughout.
TC_CASES = [
    # B, T, H
    (1, 64, 1),
    (1, 128, 1),
    (1, 127, 3),
    (2, 64, 80),
    (3, 700, 11),
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "B{}T{}H{}".format(*c))
def test_tensor_core_path_tiles(case):
    B, T, H = case
    x = workloads.draw(B, T, H, 128, 128, 700 + T + H, s0_std=0.3, with_dST=True)
    gpu = gpu_fwd_bwd(x, "bf16", 64)
    ref = oracle_fwd_bwd(x, "bf16")
    compare(gpu, ref, "bf16", ("o", "ST") + GRADS)


def test_forward_only_workspace_gives_the_same_outputs():
    """A workspace sized for the forward alone (chunk records only) and one
    sized for the backward run the same products: o and S_T agree bit for bit."""
    x = workloads.draw(2, 300, 3, 128, 128, 94, s0_std=0.2, with_dO=False)
    d = to_device(x, "bf16")
    o1, ST1, ws1 = gdn.forward(*(d[n] for n in NAMES), chunk=64, for_bwd=False)
    o2, ST2, ws2 = gdn.forward(*(d[n] for n in NAMES), chunk=64, for_bwd=True)
    torch.cuda.synchronize()
    assert ws1.numel() < ws2.numel()
    assert gdn.gdn2_get_device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(ST1, ST2)


def test_negative_eigenvalue_erase_range():
    x = workloads.draw(1, 150, 2, 64, 64, 77, erase_scale=2.0, s0_std=0.1, with_dST=True)
    for io in ("f32", "bf16"):
        compare(gpu_fwd_bwd(x, io, 64), oracle_fwd_bwd(x, io), io, ("o", "ST") + GRADS)


def test_backward_recompute_equals_reuse_and_is_deterministic():
    x = workloads.draw(2, 150, 2, 128, 128, 91, s0_std=0.1, with_dST=True)
    d = to_device(x, "bf16")
    o, ST, ws = gdn.forward(*(d[n] for n in NAMES), chunk=64, for_bwd=True)
    a = gdn.backward(*(d[n] for n in NAMES), d["dO"], d["dST"], chunk=64, ws=ws, ws_has_fwd=True)
    b = gdn.backward(*(d[n] for n in NAMES), d["dO"], d["dST"], chunk=64)  # fresh ws, recompute
    o2, ST2, _ = gdn.forward(*(d[n] for n in NAMES), chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(ST, ST2)
    for n in GRADS:
        assert torch.equal(a[n], b[n]), n


def test_tensor_core_path_repeats_bit_for_bit_at_scale():
    """Two runs of the forward and backward at a size where every persistent
    CTA walks many tiles and the state kernels run more CTAs than SMs give
    identical bits: no copy, product or readout races another."""
    x = workloads.draw(8, 1024, 16, 128, 128, 95, s0_std=0.02, with_dST=True)
    d = to_device(x, "bf16")
    runs = []
    for _ in range(2):
        o, ST, ws = gdn.forward(*(d[n] for n in NAMES), chunk=64, for_bwd=True)
        gr = gdn.backward(*(d[n] for n in NAMES), d["dO"], d["dST"], chunk=64, ws=ws, ws_has_fwd=True)
        runs.append(dict(o=o, ST=ST, **gr))
    torch.cuda.synchronize()
    for n in runs[0]:
        assert torch.equal(runs[0][n], runs[1][n]), n


@pytest.mark.parametrize("dk,chunk", [(64, 32), (128, 64)])
def test_every_output_written_and_no_nan_read(dk, chunk):
    """Outputs and workspace pre-filled with NaN: every output element must be
    written, and nothing uninitialised may reach an output."""
    B, T, H, dv = 1, 100, 2, dk
    x = workloads.draw(B, T, H, dk, dv, 92, s0_std=0.1, with_dST=True)
    d = to_device(x, "bf16")
    ws = gdn.workspace(B, T, H, dk, dv, chunk, 1, True)
    ws.view(torch.uint8).fill_(0xFF)   # NaN pattern in every float32 slot
    o = torch.full((B, T, H, dv), float("nan"), dtype=torch.bfloat16, device="cuda")
    ST = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    gdn.gdn2_fwd(*(d[n] for n in NAMES), o, ST, ws, ws.numel(), B, T, H, dk, dv, chunk, 1)
    outs = {n: torch.full_like(d[m], float("nan")) for n, m in
            (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"), ("db", "b"), ("dw", "w"))}
    outs["dS0"] = torch.full_like(ST, float("nan"))
    gdn.gdn2_bwd(*(d[n] for n in NAMES), d["dO"], d["dST"], outs["dq"], outs["dk"], outs["dv"],
                 outs["dg"], outs["db"], outs["dw"], outs["dS0"], ws, ws.numel(), 1,
                 B, T, H, dk, dv, chunk, 1)
    torch.cuda.synchronize()
    for n, t in list(outs.items()) + [("o", o), ("ST", ST)]:
        assert torch.isfinite(t.float()).all(), n


# --------------------------------------------- full-size workloads, sampled

# eight (batch, head) pairs per workload, the first and the last pair included
SAMPLE = {1: [(0, 0), (7, 15), (3, 9), (1, 4), (5, 12), (6, 1), (2, 14), (4, 7)],
          2: [(0, 0), (3, 15), (1, 7), (2, 3), (0, 12), (3, 0), (1, 14), (2, 9)],
          3: [(0, 0), (0, 15), (0, 6), (0, 3), (0, 9), (0, 12), (0, 1), (0, 13)]}


@pytest.mark.parametrize("index", [1, 2, 3])
def test_full_workload_sampled_heads(index):
    wl = workloads.WORKLOADS[index]
    x = workloads.draw_workload(index)
    if wl.backward:
        x["dST"] = torch.zeros(wl.B, wl.H, wl.dk, wl.dv)   # training: no gradient on S_T
    gpu = gpu_fwd_bwd(x, wl.io, wl.chunk, backward=wl.backward)
    ref = oracle_fwd_bwd(x, wl.io, backward=wl.backward, pairs=SAMPLE[index])
    names = ("o", "ST") + (GRADS if wl.backward else ())
    compare(gpu, ref, wl.io, names, pairs=SAMPLE[index])


# ------------------------------------------- segment-parallel state passes

@pytest.mark.parametrize("T,H", [(768, 2), (837, 2), (1024, 2), (4096, 1)])
def test_split_state_passes(T, H):
    """Few (b, h) and many chunks: the state passes split each sequence into
    segments (maps M_s, N_s in parallel, a link, then the segments' real runs).
    T = 768, 837 and 1024 with B = 1, H = 2 take 3, 4 and 4 segments (837: a
    short last segment with a ragged tail); T = 4096 with H = 1 takes the
    largest count, 8, whose link runs six steps.  Against the oracle."""
    x = workloads.draw(1, T, H, 128, 128, 980 + T, s0_std=0.1, with_dST=True)
    gpu = gpu_fwd_bwd(x, "bf16", 64)
    ref = oracle_fwd_bwd(x, "bf16")
    compare(gpu, ref, "bf16", ("o", "ST") + GRADS)


def test_split_state_passes_steep_decay_and_bf16_gates():
    """The split passes under a steep decay (g = 4 logsigmoid) with bf16 gates."""
    x = workloads.draw(1, 1024, 2, 128, 128, 985, s0_std=0.1, with_dST=True)
    gen = torch.Generator().manual_seed(986)
    x["g"] = torch.nn.functional.logsigmoid(torch.randn(x["g"].shape, generator=gen)) * 4
    gpu = gpu_fwd_bwd(x, "bf16", 64, gates="bf16")
    ref = oracle_fwd_bwd(x, "bf16", gates="bf16")
    compare(gpu, ref, "bf16", ("o", "ST") + GRADS)


# --------------------------------------------------------------- bf16 gates

@pytest.mark.parametrize("index", [1, 2])
def test_bf16_gates_full_workload_sampled_heads(index):
    """g, b, w in bf16 (and dg, db, dw returned in bf16) on the tensor-core
    path at full size: the oracle takes the same bf16-rounded gate values."""
    wl = workloads.WORKLOADS[index]
    x = workloads.draw_workload(index)
    if wl.backward:
        x["dST"] = torch.zeros(wl.B, wl.H, wl.dk, wl.dv)
    gpu = gpu_fwd_bwd(x, wl.io, wl.chunk, backward=wl.backward, gates="bf16")
    ref = oracle_fwd_bwd(x, wl.io, backward=wl.backward, pairs=SAMPLE[index], gates="bf16")
    names = ("o", "ST") + (GRADS if wl.backward else ())
    compare(gpu, ref, wl.io, names, pairs=SAMPLE[index])


@pytest.mark.parametrize("kind", ["ragged", "steep_then_mild"])
def test_bf16_gates_small(kind):
    """bf16 gates on a ragged length (T = 200: three full chunks and a short
    one) and on a call that takes both the steep and the mild tile paths."""
    if kind == "ragged":
        x = workloads.draw(2, 200, 2, 128, 128, 77, s0_std=0.1, with_dST=True)
    else:
        x = _steep(kind, 931)
    gpu = gpu_fwd_bwd(x, "bf16", 64, gates="bf16")
    ref = oracle_fwd_bwd(x, "bf16", gates="bf16")
    compare(gpu, ref, "bf16", ("o", "ST") + GRADS)


def test_bf16_gates_match_f32_gates_on_rounded_values():
    """The two gate types give the same results when the float32 gates hold
    the bf16-rounded values: the bf16 path only changes the storage."""
    x = io_round(workloads.draw(1, 256, 2, 128, 128, 58, s0_std=0.1, with_dST=True), "f32", "bf16")
    a = gpu_fwd_bwd(x, "bf16", 64, gates="f32")
    b = gpu_fwd_bwd(x, "bf16", 64, gates="bf16")
    for n in ("o", "ST", "dq", "dk", "dv", "dS0"):
        assert np.array_equal(a[n], b[n]), n
    for n in ("dg", "db", "dw"):   # rounded once more to bf16
        assert rel(b[n], a[n]) < 4e-3, n


# -------------------------------------------------------- packed sequences

VARLEN_LENS = [65, 1, 200, 64, 0, 3, 130, 17]


def _varlen_inputs(lens, H, seed):
    cu = [0] + list(np.cumsum(lens))
    N, T = len(lens), int(cu[-1])
    x = workloads.draw(1, T, H, 128, 128, seed)
    x["S0"] = workloads.draw(N, 1, H, 128, 128, seed + 1, s0_std=0.1)["S0"]
    x["dST"] = workloads.draw(N, 1, H, 128, 128, seed + 2, s0_std=0.1)["S0"]
    return x, [int(c) for c in cu]


def gpu_varlen(x, cu, gates="f32"):
    d = to_device(x, "bf16", gates=gates)
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    o, ST, ws = gdn.forward_varlen(*(d[n] for n in NAMES[:-1]), cu_d, d["S0"], for_bwd=True)
    gr = gdn.backward_varlen(*(d[n] for n in NAMES[:-1]), cu_d, d["S0"], d["dO"], d["dST"], ws=ws,
                             ws_has_fwd=True)
    torch.cuda.synchronize()
    assert gdn.gdn2_get_device_status() == 0
    out = {"o": o, "ST": ST, **gr}
    return {n: t.float().cpu().numpy() for n, t in out.items()}


@pytest.mark.parametrize("gates", ["f32", "bf16"])
def test_varlen_mixed_lengths(gates):
    """Packed sequences of lengths 65, 1, 200, 64, 0, 3, 130 and 17 (short
    tails, a sequence of one token, an empty one) against the oracle run on
    each sequence alone from its own S0."""
    from oracle import varlen
    x, cu = _varlen_inputs(VARLEN_LENS, 2, 950)
    gpu = gpu_varlen(x, cu, gates)
    r = to_np64(io_round(x, "bf16", gates))
    names = ("q", "k", "v", "g", "b", "w")
    o, ST = varlen.forward(*(r[n] for n in names), cu, r["S0"])
    ref = {"o": o, "ST": ST, **varlen.backward(*(r[n] for n in names), cu, r["S0"], r["dO"], r["dST"])}
    compare(gpu, ref, "bf16", ("o", "ST") + GRADS)


def test_varlen_equal_lengths_match_the_batch_bit_for_bit():
    """Three sequences of 200 tokens packed back to back give exactly the
    batch call's results: the same tiles, masked tails instead of the
    tensor's end."""
    B, T, H = 3, 200, 2
    x = workloads.draw(B, T, H, 128, 128, 951, s0_std=0.1, with_dST=True)
    dense = gpu_fwd_bwd(x, "bf16", 64)
    packed = {n: (t.reshape(1, B * T, *t.shape[2:]) if n not in ("S0", "dST") else t) for n, t in x.items()}
    pv = gpu_varlen(packed, [0, T, 2 * T, 3 * T])
    for n in ("o", "dq", "dk", "dv", "dg", "db", "dw"):
        assert np.array_equal(pv[n], dense[n].reshape(pv[n].shape)), n
    for n in ("ST", "dS0"):
        assert np.array_equal(pv[n], dense[n]), n


def test_varlen_rejects_a_bad_table_on_the_device():
    """A table that falls (0, 30, 20, 64) is caught on the device: the call
    records GDN2_ERR_INVALID_ARG, treats every sequence as empty, and the
    next valid call runs clean."""
    x, cu = _varlen_inputs([30, 0, 44], 1, 952)
    d = to_device(x, "bf16")
    bad = torch.tensor([0, 30, 20, 74], dtype=torch.int32, device="cuda")
    o, ST, _ = gdn.forward_varlen(*(d[n] for n in NAMES[:-1]), bad, d["S0"], check=False)
    torch.cuda.synchronize()
    assert gdn.gdn2_get_device_status() == 1
    assert torch.equal(ST, d["S0"])
    gpu = gpu_varlen(x, cu)          # asserts a clean status itself
    assert np.isfinite(gpu["o"]).all()


# ------------------------------------------------------ fused gate prologue

def _logit_inputs(B, T, H, seed, g_shift):
    """Gate logits: x_g ~ N(g_shift, 1) (g = log sigmoid(x_g): shift 3 gives a
    mild decay near -0.05 per token, shift 0 a steep one near -0.8), x_b, x_w ~ N(0, 1.5)."""
    x = workloads.draw(B, T, H, 128, 128, seed, s0_std=0.1, with_dST=True)
    gen = torch.Generator().manual_seed(seed + 1)
    x["g"] = torch.randn(x["g"].shape, generator=gen) + g_shift
    x["b"] = torch.randn(x["b"].shape, generator=gen) * 1.5
    x["w"] = torch.randn(x["w"].shape, generator=gen) * 1.5
    return x


@pytest.mark.parametrize("encoding,gates,T,g_shift", [
    ("logits", "f32", 200, 3.0),        # mild tiles, ragged
    ("logits_b2", "bf16", 200, 0.0),    # steep tiles, b = 2 sigmoid, bf16 logits
    ("logits", "f32", 1024, 3.0),       # the split state passes (B1 H2: 4 segments)
])
def test_gate_logits(encoding, gates, T, g_shift):
    """The fused gate prologue: g, b, w arrive as logits, the kernels activate
    them on load, and dg, db, dw leave as gradients of the logits.  Against
    the oracle's gate layer (fp64 activations, chain rule) on the same
    (rounded) logits."""
    from oracle import gates as ogates
    B = 2 if T == 200 else 1
    x = _logit_inputs(B, T, 2, 990 + T, g_shift)
    gpu = gpu_fwd_bwd(x, "bf16", 64, gates=gates, encoding=encoding)
    r = to_np64(io_round(x, "bf16", gates))
    bs = 2.0 if encoding == "logits_b2" else 1.0
    args = (r["q"], r["k"], r["v"], r["g"], r["b"], r["w"], r["S0"])
    o, ST = ogates.forward(*args, b_scale=bs)
    ref = {"o": o, "ST": ST, **ogates.backward(*args, r["dO"], r["dST"], b_scale=bs)}
    compare(gpu, ref, "bf16", ("o", "ST") + GRADS)


def test_gate_logits_packed():
    """Gate logits with packed sequences (65, 1, 130 tokens): the rows past each
    sequence's end keep no decay, as a zero logit would otherwise activate to
    log 1/2."""
    from oracle import gates as ogates, varlen
    cu = [0, 65, 66, 196]
    x = _logit_inputs(1, 196, 2, 995, 1.0)
    x["S0"] = workloads.draw(3, 1, 2, 128, 128, 996, s0_std=0.1)["S0"]
    x["dST"] = workloads.draw(3, 1, 2, 128, 128, 997, s0_std=0.1)["S0"]
    d = to_device(x, "bf16")
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    o, ST, ws = gdn.forward_varlen(*(d[n] for n in NAMES[:-1]), cu_d, d["S0"], for_bwd=True, gates="logits")
    gr = gdn.backward_varlen(*(d[n] for n in NAMES[:-1]), cu_d, d["S0"], d["dO"], d["dST"], ws=ws,
                             ws_has_fwd=True, gates="logits")
    torch.cuda.synchronize()
    assert gdn.gdn2_get_device_status() == 0
    gpu = {n: t.float().cpu().numpy() for n, t in {"o": o, "ST": ST, **gr}.items()}
    r = to_np64(io_round(x, "bf16"))
    ga, gb_, gw = ogates.activate(r["g"], r["b"], r["w"])
    names = ("q", "k", "v")
    o_ref, ST_ref = varlen.forward(*(r[n] for n in names), ga, gb_, gw, cu, r["S0"])
    ref = varlen.backward(*(r[n] for n in names), ga, gb_, gw, cu, r["S0"], r["dO"], r["dST"])
    sig = lambda z: 0.5 * (1.0 + np.tanh(0.5 * z))  # noqa: E731
    ref["dg"] = ref["dg"] * sig(-r["g"])
    ref["db"] = ref["db"] * sig(r["b"]) * (1 - sig(r["b"]))
    ref["dw"] = ref["dw"] * sig(r["w"]) * (1 - sig(r["w"]))
    compare(gpu, {"o": o_ref, "ST": ST_ref, **ref}, "bf16", ("o", "ST") + GRADS)


def test_gate_logits_decode():
    """The decode step with gate logits (b = 2 sigmoid) against the oracle's gate layer."""
    from oracle import gates as ogates
    N, H, dk, dv = 3, 2, 64, 64
    S_gpu = workloads.decode_state(N, H, dk, dv, 21, 0.3).cuda()
    S_ref = S_gpu.double().cpu().numpy()
    for s_ in range(6):
        x = workloads.decode_step_inputs(N, H, dk, dv, 22, s_)
        gen = torch.Generator().manual_seed(23 + s_)
        for n in ("g", "b", "w"):
            x[n] = torch.randn(x[n].shape, generator=gen) + (2.0 if n == "g" else 0.0)
        d = {n: t.cuda() for n, t in x.items()}
        o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S_gpu, gates="logits_b2")
        r = {n: t.double().numpy()[:, None] for n, t in x.items()}
        o_ref, S_ref = ogates.forward(r["q"], r["k"], r["v"], r["g"], r["b"], r["w"], S_ref, b_scale=2.0)
        assert rel(o.cpu().numpy(), o_ref[:, 0]) < TOL_F32, s_
        assert rel(S_gpu.cpu().numpy(), S_ref) < TOL_F32, s_


# ------------------------------------------------------ grouped value heads

def _grouped_inputs(B, T, H, Hv, dk, dv, seed):
    x = workloads.draw(B, T, H, dk, dv, seed)
    xv = workloads.draw(B, T, Hv, dk, dv, seed + 1, s0_std=0.1, with_dST=True)
    for n in ("v", "w", "S0", "dO", "dST"):
        x[n] = xv[n]
    return x


@pytest.mark.parametrize("io,H,Hv,dk,dv,chunk", [
    ("bf16", 2, 4, 128, 64, 64),     # tensor cores: G d_v = 128
    ("f32", 1, 2, 64, 32, 32),       # CUDA cores: G d_v = 64
    ("bf16", 1, 4, 32, 32, 16),      # CUDA cores, bf16 I/O: G d_v = 128
])
def test_grouped_value_heads(io, H, Hv, dk, dv, chunk):
    """H_v value heads over H key heads: value head j reads key head
    j / (H_v / H); states per value head.  Against the oracle's grouped form
    (the token loop on repeated q, k, g, b, key-side gradients summed)."""
    from oracle import grouped
    x = _grouped_inputs(2, 150, H, Hv, dk, dv, 960 + Hv)
    gpu = gpu_fwd_bwd(x, io, chunk)
    r = to_np64(io_round(x, io))
    names = ("q", "k", "v", "g", "b", "w", "S0")
    o, ST = grouped.forward(*(r[n] for n in names))
    ref = {"o": o, "ST": ST, **grouped.backward(*(r[n] for n in names), r["dO"], r["dST"])}
    compare(gpu, ref, io, ("o", "ST") + GRADS)


def test_grouped_value_heads_packed():
    """Grouped value heads and packed sequences together (tensor cores)."""
    from oracle import varlen
    cu = [0, 70, 71, 200]       # lengths 70, 1, 129
    x = _grouped_inputs(1, 200, 1, 2, 128, 64, 970)
    x["S0"] = workloads.draw(3, 1, 2, 128, 64, 971, s0_std=0.1)["S0"]
    x["dST"] = workloads.draw(3, 1, 2, 128, 64, 972, s0_std=0.1)["S0"]
    gpu = gpu_varlen(x, cu)
    r = to_np64(io_round(x, "bf16"))
    rep = {n: (np.repeat(r[n], 2, axis=2) if n in ("q", "k", "g", "b") else r[n]) for n in r}
    names = ("q", "k", "v", "g", "b", "w")
    o, ST = varlen.forward(*(rep[n] for n in names), cu, rep["S0"])
    gr = varlen.backward(*(rep[n] for n in names), cu, rep["S0"], rep["dO"], rep["dST"])
    for n in ("q", "k", "g", "b"):
        gr["d" + n] = gr["d" + n].reshape(1, 200, 1, 2, 128).sum(axis=3)
    compare(gpu, {"o": o, "ST": ST, **gr}, "bf16", ("o", "ST") + GRADS)


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("io,gates", [("f32", "f32"), ("bf16", "f32"), ("bf16", "bf16"),
                                      ("f32", "bf16")])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (32, 128)])
def test_decode_small_step_by_step(io, gates, dk, dv):
    N, H, steps = 3, 2, 12
    S_gpu = (workloads.decode_state(N, H, dk, dv, 7, 0.3)).cuda()
    S_ref = S_gpu.double().cpu().numpy()
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    gt = torch.bfloat16 if gates == "bf16" else torch.float32
    tol = TOL_F32 if io == "f32" else TOL_BF16_OUT
    for s in range(steps):
        x = workloads.decode_step_inputs(N, H, dk, dv, 7, s, erase_scale=2.0 if s % 2 else 1.0)
        xr = io_round(x, io, gates)
        d = {n: (t.to(dt) if n in ("q", "k", "v") else t.to(gt)).cuda() for n, t in x.items()}
        o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S_gpu)
        r = {n: t.double().numpy()[:, None] for n, t in xr.items()}
        o_ref, S_ref = oracle.forward(r["q"], r["k"], r["v"], r["g"], r["b"], r["w"], S_ref)
        assert rel(o.float().cpu().numpy(), o_ref[:, 0]) < tol, s
        assert rel(S_gpu.cpu().numpy(), S_ref) < tol, s


@pytest.mark.parametrize("H,Hv,dk,dv", [(2, 4, 64, 32), (1, 2, 128, 128)])
def test_decode_grouped_value_heads(H, Hv, dk, dv):
    """The decode step with H_v value heads over H key heads, against the
    oracle's grouped form, step by step from the same state."""
    from oracle import grouped
    N, steps = 3, 6
    S_gpu = workloads.decode_state(N, Hv, dk, dv, 11, 0.3).cuda()
    S_ref = S_gpu.double().cpu().numpy()
    for s_ in range(steps):
        xk = workloads.decode_step_inputs(N, H, dk, dv, 12, s_)
        xv = workloads.decode_step_inputs(N, Hv, dk, dv, 13, s_)
        x = {n: (xk[n] if n in ("q", "k", "g", "b") else xv[n]) for n in ("q", "k", "v", "g", "b", "w")}
        d = {n: t.cuda() for n, t in x.items()}
        o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S_gpu)
        r = {n: t.double().numpy()[:, None] for n, t in x.items()}
        o_ref, S_ref = grouped.forward(r["q"], r["k"], r["v"], r["g"], r["b"], r["w"], S_ref)
        assert rel(o.cpu().numpy(), o_ref[:, 0]) < TOL_F32, s_
        assert rel(S_gpu.cpu().numpy(), S_ref) < TOL_F32, s_


def test_decode_equals_chunked_forward():
    """T decode steps reproduce the chunked forward's outputs and final state."""
    B, T, H, dk, dv = 2, 40, 2, 128, 128
    x = workloads.draw(B, T, H, dk, dv, 93, s0_std=0.1, with_dO=False)
    d = to_device(x, "f32")
    o, ST, _ = gdn.forward(*(d[n] for n in NAMES), chunk=16)
    S = d["S0"].clone()
    outs = []
    for t in range(T):
        outs.append(gdn.decode_step(*(d[n][:, t].contiguous() for n in NAMES[:-1]), S))
    torch.cuda.synchronize()
    assert rel(torch.stack(outs, 1).cpu().numpy(), o.cpu().numpy()) < TOL_F32
    assert rel(S.cpu().numpy(), ST.cpu().numpy()) < TOL_F32


def test_workload4_decode_sampled_every_step():
    """256 sequences x 16 heads, 1024 consecutive steps, bf16 q/k/v, float32
    state carried in HBM; sampled (sequence, head) pairs checked after every
    step against the oracle stepped from the same state, never re-synchronised."""
    wl = workloads.WORKLOADS[4]
    N, H, dk, dv = wl.B, wl.H, wl.dk, wl.dv
    pairs = [(0, 0), (255, 15), (100, 7), (17, 3)]
    S = workloads.decode_state(N, H, dk, dv, wl.seed, wl.s0_std).cuda()
    S_ref = np.stack([S[n, h].double().cpu().numpy() for n, h in pairs])[None]
    worst_o = worst_S = 0.0
    for s in range(wl.decode_steps):
        x = workloads.decode_step_inputs(N, H, dk, dv, wl.seed, s)
        d = {n: (t.to(torch.bfloat16) if n in ("q", "k", "v") else t).cuda() for n, t in x.items()}
        o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S)
        xr = io_round(x, "bf16")
        r = {n: np.stack([t[nn, hh].double().numpy() for nn, hh in pairs])[None, None]
             for n, t in xr.items()}
        o_ref, S_ref = oracle.forward(r["q"], r["k"], r["v"], r["g"], r["b"], r["w"], S_ref)
        o_s = np.stack([o[nn, hh].float().cpu().numpy() for nn, hh in pairs])
        worst_o = max(worst_o, rel(o_s, o_ref[0, 0]))
        if s % 64 == 63 or s == wl.decode_steps - 1:
            S_s = np.stack([S[nn, hh].cpu().numpy() for nn, hh in pairs])
            worst_S = max(worst_S, rel(S_s, S_ref[0]))
    assert worst_o < TOL_BF16_OUT and worst_S < TOL_BF16_OUT, (worst_o, worst_S)


# ------------------------------------------------------ bounded waits
def test_bounded_wait_reports_timeout_and_context_stays_usable():
    """A wait that nothing completes gives up, records GDN2_ERR_TIMEOUT in the
    status word (read once, then cleared), and later calls still run and
    still agree with the oracle."""
    assert gdn.gdn2_get_device_status() == 0
    gdn.gdn2_selftest_timeout(2_000_000)
    assert gdn.gdn2_get_device_status() == 5          # GDN2_ERR_TIMEOUT
    assert gdn.gdn2_get_device_status() == 0          # cleared by the read
    x = workloads.draw(1, 70, 2, 64, 64, 31, s0_std=0.1, with_dO=False)
    d = to_device(x, "f32")
    o, ST, _ = gdn.forward(*(d[n] for n in ("q", "k", "v", "g", "b", "w", "S0")), chunk=64)
    torch.cuda.synchronize()
    assert gdn.gdn2_get_device_status() == 0
    r = to_np64(x)
    o_ref, S_ref = oracle.forward(r["q"], r["k"], r["v"], r["g"], r["b"], r["w"], r["S0"])
    assert rel(o.cpu().numpy(), o_ref) < TOL_F32 and rel(ST.cpu().numpy(), S_ref) < TOL_F32


# ------------------------------------------------------ CUDA graph capture
def test_decode_steps_capture_in_a_cuda_graph():
    """Launches through the C ABI on a capturing stream are captured, not run:
    the state is untouched after capture, and one replay of 16 captured decode
    steps leaves it bit for bit where 16 eager steps do."""
    N, H, dk, dv = 32, 4, 128, 128
    S0 = workloads.decode_state(N, H, dk, dv, 11, 0.3).cuda()
    x = workloads.decode_step_inputs(N, H, dk, dv, 11, 0)
    d = {n: (t.to(torch.bfloat16) if n in ("q", "k", "v") else t).cuda() for n, t in x.items()}
    o = torch.empty(N, H, dv, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()

    def run(S, n):
        for _ in range(n):
            gdn.gdn2_decode_step(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], S, o, N, H, dk, dv,
                                 gdn.GDN2_IO_BF16, s)

    Sw = S0.clone()
    with torch.cuda.stream(s):
        run(Sw, 1)
    torch.cuda.synchronize()
    Sg = S0.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(Sg, 16)
    torch.cuda.synchronize()
    assert torch.equal(Sg, S0)
    with torch.cuda.stream(s):
        g.replay()
    Se = S0.clone()
    with torch.cuda.stream(s):
        run(Se, 16)
    torch.cuda.synchronize()
    assert torch.equal(Sg, Se) and not torch.equal(Se, S0)
    assert gdn.gdn2_get_device_status() == 0


# ------------------------------------------------------ steep decay, any g <= 0
def _steep(kind, seed):
    x = workloads.draw(1, 256, 2, 128, 128, seed, s0_std=0.2, with_dST=True)
    gen = torch.Generator().manual_seed(seed + 1)
    if kind == "logsigmoid_x4":   # per channel, about -2.8 on average, tails below -20
        x["g"] = torch.nn.functional.logsigmoid(torch.randn(x["g"].shape, generator=gen)) * 4
    elif kind == "const_-2":
        x["g"] = torch.full_like(x["g"], -2.0)
    elif kind == "mixed_-30":     # a third of the channels forget almost at once
        g = torch.nn.functional.logsigmoid(torch.randn(x["g"].shape, generator=gen)) / 16
        g[..., ::3] = -30.0
        x["g"] = g
    elif kind == "steep_then_mild":  # chunks 0, 1 steep, chunks 2, 3 mild: both tile paths in one call
        g = torch.nn.functional.logsigmoid(torch.randn(x["g"].shape, generator=gen)) / 16
        g[:, :128] = torch.nn.functional.logsigmoid(torch.randn(x["g"][:, :128].shape, generator=gen)) * 4
        x["g"] = g
    elif kind == "edge_-0.13":      # |G - G_31| reaches about 4.2: just past the single-frame bound
        x["g"] = torch.full_like(x["g"], -0.13)
    return x


@pytest.mark.parametrize("kind", ["logsigmoid_x4", "const_-2", "mixed_-30", "steep_then_mild", "edge_-0.13"])
def test_tensor_core_path_steep_decay(kind):
    """Any g <= 0 on the tensor-core path: the chunk-start frame keeps every
    state-side factor <= 1, and the in-chunk pair factors come from block
    frames, so steep decays match the oracle at the bf16 tolerances with a
    clean device status (gpu_fwd_bwd checks it)."""
    x = _steep(kind, 900 + len(kind))
    gpu = gpu_fwd_bwd(x, "bf16", 64)
    ref = oracle_fwd_bwd(x, "bf16")
    compare(gpu, ref, "bf16", ("o", "ST") + GRADS)


def test_tensor_core_path_reports_fp16_overflow():
    """The tensor-core operands are fp16: values beyond its range (here w v
    about 1e6) make the kernels record GDN2_ERR_RANGE instead of silently
    returning overflowed results; the word clears once read, and an in-range
    call afterwards reports nothing."""
    x = workloads.draw(1, 128, 2, 128, 128, 41, with_dO=False)
    x["v"] = x["v"] * 1e6
    d = to_device(x, "bf16")
    gdn.forward(*(d[n] for n in NAMES), chunk=64, check=False)
    torch.cuda.synchronize()
    assert gdn.gdn2_get_device_status() == 6          # GDN2_ERR_RANGE
    assert gdn.gdn2_get_device_status() == 0
    with pytest.raises(gdn.Gdn2Error):
        gdn.forward(*(d[n] for n in NAMES), chunk=64)  # check=True raises
    x2 = workloads.draw(1, 128, 2, 128, 128, 42, with_dO=False)
    d2 = to_device(x2, "bf16")
    gdn.forward(*(d2[n] for n in NAMES), chunk=64)
    torch.cuda.synchronize()
    assert gdn.gdn2_get_device_status() == 0
