"""gdn2_fwd_noalloc: the forward for callers that cannot allocate device memory
(a plugin that is handed only input and output pointers by a framework whose
allocator owns the GPU, or a latency-critical path that cannot afford
cudaMalloc's implicit synchronisation).  Its scratch is a fixed device array
inside the library, shared by every call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import pytest
import torch

import gated_delta_rule_128_b200 as gdn
from gated_delta_rule_128_b200 import build, workloads
from _util import TOL_BF16_OUT, TOL_F32, rel, to_device

NAMES = ("q", "k", "v", "g", "b", "w", "S0")
FAKE = 1 << 20   # aligned, never dereferenced: the size check fails first


def test_noalloc_rejects_problems_beyond_its_scratch():
    build.build()
    L = gdn.lib()
    limit = 64 << 20
    # d = 128, chunk 64: 292 chunk tiles fit, 293 do not
    f32 = gdn.GDN2_IO_F32   # the limit is the float32 path's workspace, whatever the io type
    assert gdn.gdn2_workspace_bytes(1, 292 * 64, 1, 128, 128, 64, f32, 0) <= limit
    assert gdn.gdn2_workspace_bytes(1, 293 * 64, 1, 128, 128, 64, f32, 0) > limit
    call = lambda T: L.gdn2_fwd_noalloc(*([FAKE] * 6), None, FAKE, None,  # noqa: E731
                                        1, T, 1, 128, 128, 64, 1, None)
    assert call(293 * 64) == 3            # GDN2_ERR_WORKSPACE, nothing enqueued
    assert L.gdn2_fwd_noalloc(*([FAKE] * 6), None, FAKE, None, 1, 64, 1, 48, 128, 64, 1,
                              None) == 2  # unsupported d_k
    assert L.gdn2_fwd_noalloc(None, *([FAKE] * 5), None, FAKE, None, 1, 64, 1, 128, 128, 64, 1,
                              None) == 1  # null q


def _one(io, B, T, H, dk, dv, chunk, seed):
    x = workloads.draw(B, T, H, dk, dv, seed, s0_std=0.1, with_dO=False)
    d = to_device(x, io)
    dt = d["q"].dtype
    iocode = gdn.GDN2_IO_BF16 if io == "bf16" else gdn.GDN2_IO_F32
    o_ref, ST_ref, _ = gdn.forward(*(d[n] for n in NAMES), chunk=chunk)
    o = torch.full((B, T, H, dv), float("nan"), dtype=dt, device="cuda")
    ST = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    gdn.gdn2_fwd_noalloc(*(d[n] for n in NAMES), o, ST, B, T, H, dk, dv, chunk, iocode)
    torch.cuda.synchronize()
    tol = TOL_F32 if io == "f32" else TOL_BF16_OUT
    assert rel(o.float().cpu().numpy(), o_ref.float().cpu().numpy()) <= tol
    assert rel(ST.cpu().numpy(), ST_ref.cpu().numpy()) <= tol


@pytest.mark.gpu
def test_noalloc_matches_gdn2_fwd_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # two different problems back to back: the shared scratch keeps the first
    # call's contents, which must not leak into the second
    _one("bf16", 2, 1000, 4, 128, 128, 64, 3101)
    _one("f32", 1, 77, 3, 64, 32, 16, 3102)
    _one("bf16", 2, 1000, 4, 128, 128, 64, 3103)
