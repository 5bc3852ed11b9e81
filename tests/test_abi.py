"""The C ABI library: it loads, exports every entry point include/gdn2.h
declares, sizes workspaces, and rejects bad arguments on the host before any
launch.  CPU only (no call here reaches the GPU)."""

import ctypes
import os
import re
import subprocess

import pytest

import gated_delta_rule_128_b200 as gdn
from gated_delta_rule_128_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn2.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return gdn.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn2_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdn2_fwd", "gdn2_bwd", "gdn2_decode_step", "gdn2_workspace_bytes",
              "gdn2_get_device_status", "gdn2_status_string", "gdn2_version"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gdn2_\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(L, n)


def test_library_links_no_torch(L):
    out = subprocess.run(["ldd", gdn.LIB_PATH], capture_output=True, text=True).stdout
    assert "torch" not in out and "c10" not in out


def test_status_strings_and_version(L):
    for s in range(7):
        assert len(L.gdn2_status_string(s)) > 0
    assert L.gdn2_status_string(99) == b"unknown status"
    assert L.gdn2_version() >= 100


def test_workspace_query(L):
    small = gdn.gdn2_workspace_bytes(1, 256, 2, 32, 32, 64, 0, 0)
    big = gdn.gdn2_workspace_bytes(1, 256, 2, 32, 32, 64, 0, 1)
    assert 0 < small < big
    assert gdn.gdn2_workspace_bytes(4, 4096, 16, 128, 128, 64, 1, 1) > 0
    # unsupported sizes report 0
    assert gdn.gdn2_workspace_bytes(1, 256, 2, 48, 32, 64, 0, 0) == 0
    assert gdn.gdn2_workspace_bytes(1, 256, 2, 32, 32, 128, 0, 0) == 0
    assert gdn.gdn2_workspace_bytes(0, 256, 2, 32, 32, 64, 0, 0) == 0
    assert gdn.gdn2_workspace_bytes(1, 256, 2, 32, 32, 64, 7, 0) == 0


FAKE = 1 << 20   # an aligned, never-dereferenced address: host checks fail first


def fwd(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, w=FAKE, S0=None, o=FAKE, ST=None, ws=FAKE,
             ws_bytes=1 << 40, B=1, T=16, H=1, dk=32, dv=32, chunk=16, io=0)
    a.update(kw)
    return L.gdn2_fwd(a["q"], a["k"], a["v"], a["g"], a["b"], a["w"], a["S0"], a["o"], a["ST"],
                      a["ws"], a["ws_bytes"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                      a["chunk"], a["io"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(w=None), 1),
    (dict(q=FAKE + 4), 1), (dict(S0=FAKE + 8), 1),
    (dict(B=0), 1), (dict(T=0), 1), (dict(H=-1), 1), (dict(io=3), 1),
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(chunk=128), 2), (dict(chunk=8), 2),
    (dict(ws=None), 3), (dict(ws_bytes=100), 3), (dict(ws=FAKE + 2), 3),
])
def test_fwd_rejects_bad_arguments(L, kw, status):
    assert fwd(L, **kw) == status


def test_bwd_rejects_bad_arguments(L):
    args = [FAKE] * 6 + [None, FAKE, None] + [FAKE] * 6 + [None, FAKE]
    call = lambda ws_bytes, dims: L.gdn2_bwd(*args, ws_bytes, 1, *dims, 0, None)  # noqa: E731
    assert call(10, (1, 16, 1, 32, 32, 16)) == 3
    assert call(1 << 40, (1, 16, 1, 32, 32, 24)) == 2
    bad = list(args)
    bad[9] = None  # dq
    assert L.gdn2_bwd(*bad, 1 << 40, 1, 1, 16, 1, 32, 32, 16, 0, None) == 1


def test_decode_rejects_bad_arguments(L):
    f = lambda *p, N=1, H=1, dk=32, dv=32, io=0: L.gdn2_decode_step(*p, N, H, dk, dv, io, None)  # noqa
    ok = [FAKE] * 8
    assert f(*([None] + ok[1:])) == 1
    assert f(*ok, N=0) == 1
    assert f(*ok, dk=16) == 2
    assert f(*ok, io=5) == 1
    bad = list(ok)
    bad[6] = FAKE + 4   # S misaligned
    assert f(*bad) == 1


def test_ex_entry_points_check_the_gate_type_and_value_heads(L):
    """bf16 gates need the tensor-core path: any other size or io type is
    rejected as unsupported, an unknown gate type as invalid, and float32
    gates with H_v = H behave as the calls without the suffix.  H_v must be a
    multiple of H whose group width G d_v is a supported d_v."""
    def fwd_ex(gate_io, dk=32, dv=32, chunk=16, io=0, ws_bytes=1 << 40, H=1, Hv=1):
        return L.gdn2_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, ws_bytes,
                             1, 16, H, Hv, dk, dv, chunk, io, gate_io, None)
    assert fwd_ex(1) == 2                              # f32 io, d = 32
    assert fwd_ex(1, dk=128, dv=128, chunk=64) == 2    # still f32 io
    assert fwd_ex(1, dk=128, dv=128, chunk=32, io=1) == 2
    assert fwd_ex(5) == 1
    assert fwd_ex(0, ws_bytes=10) == 3 == fwd(L, ws_bytes=10)
    assert fwd_ex(1, dk=128, dv=128, chunk=64, io=1, ws_bytes=10) == 3   # passes the gate check
    assert fwd_ex(0, H=2, Hv=3) == 1                   # not a multiple
    assert fwd_ex(0, H=2, Hv=1) == 1                   # fewer value heads
    assert fwd_ex(0, H=1, Hv=8, dv=32) == 2            # G d_v = 256
    assert fwd_ex(0, H=1, Hv=4, dv=32, ws_bytes=10) == 3   # G d_v = 128: passes
    assert fwd_ex(1, dk=128, dv=64, chunk=64, io=1, H=1, Hv=2, ws_bytes=10) == 3  # tensor cores
    # gate logits: tensor-core path only; B_X2 needs LOGITS; unknown flags are invalid
    assert fwd_ex(0x100) == 2
    assert fwd_ex(0x100 | 0x200, dk=128, dv=128, chunk=64, io=1, ws_bytes=10) == 3
    assert fwd_ex(0x200, dk=128, dv=128, chunk=64, io=1) == 1
    assert fwd_ex(0x400, dk=128, dv=128, chunk=64, io=1) == 1
    args = [FAKE] * 6 + [None, FAKE, None] + [FAKE] * 6 + [None, FAKE]
    assert L.gdn2_bwd_ex(*args, 1 << 40, 1, 1, 16, 1, 1, 32, 32, 16, 0, 1, None) == 2
    assert L.gdn2_bwd_ex(*args, 1 << 40, 1, 1, 16, 1, 1, 32, 32, 16, 0, 9, None) == 1
    assert L.gdn2_decode_step_ex(*([FAKE] * 8), 1, 1, 1, 32, 32, 0, 7, None) == 1
    assert L.gdn2_decode_step_ex(*([FAKE] * 8), 1, 1, 1, 16, 32, 0, 1, None) == 2
    assert L.gdn2_decode_step_ex(*([FAKE] * 8), 1, 2, 3, 32, 32, 0, 0, None) == 1


def test_workspace_sizes_of_the_ex_and_packed_calls(L):
    """H_v = H sizes as the plain call; grouped heads add two state buffers;
    packed sequences size for ceil(T / 64) + N chunks and need the tensor-core
    path."""
    plain = gdn.gdn2_workspace_bytes(2, 300, 4, 128, 128, 64, 1, 1)
    assert gdn.gdn2_workspace_bytes_ex(2, 300, 4, 4, 128, 128, 64, 1, 0, 1) == plain
    assert gdn.gdn2_workspace_bytes_ex(2, 300, 4, 0, 128, 128, 64, 1, 1, 1) == plain
    grouped = gdn.gdn2_workspace_bytes_ex(2, 300, 4, 8, 128, 64, 64, 1, 0, 1)
    assert grouped >= plain + 2 * 2 * 4 * 128 * 128 * 4
    one = gdn.gdn2_workspace_bytes_varlen(1, 600, 4, 4, 128, 128, 64, 1, 0, 1)
    many = gdn.gdn2_workspace_bytes_varlen(50, 600, 4, 4, 128, 128, 64, 1, 0, 1)
    assert 0 < one < many
    assert gdn.gdn2_workspace_bytes_varlen(1, 600, 4, 4, 64, 64, 64, 1, 0, 1) == 0   # no tensor cores
    assert gdn.gdn2_workspace_bytes_varlen(0, 600, 4, 4, 128, 128, 64, 1, 0, 1) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(gdn, "_lib", None)
    monkeypatch.setattr(gdn, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        gdn.lib()
