"""Host-side logic of bench.py: the algorithmic byte model behind every roofline
fraction it prints, and the rule that a recorded DRAM traffic figure applies only
to the kernel sources it was captured on.  No GPU."""

import json

import pytest

import bench

D = 128  # channels per head (d_k = d_v)


def _bytes(tensors, gs):
    # bf16 activations and their gradients; gates and their gradients in gs bytes
    gates = {"g", "b", "w", "dg", "db", "dw"}
    return sum(D * (gs if t in gates else 2) for t in tensors)


@pytest.mark.parametrize("gs, fwd_total, bwd_total", [(4, 2560, 4864), (2, 1792, 3328)])
def test_byte_model_counts_each_tensor_once(gs, fwd_total, bwd_total):
    # forward: reads q, k, v, g, b, w and writes o; backward: reads q, k, v, g,
    # b, w and dO, writes dq, dk, dv, dg, db, dw (the state and S0 are per (b, h),
    # not per token, and are left out)
    fwd_t = ["q", "k", "v", "g", "b", "w", "o"]
    bwd_t = ["q", "k", "v", "g", "b", "w", "dO", "dq", "dk", "dv", "dg", "db", "dw"]
    fwd, bwd, kern = bench.byte_model(gs)
    assert fwd == _bytes(fwd_t, gs) == fwd_total
    assert bwd == _bytes(bwd_t, gs) == bwd_total
    # every tensor is attributed to exactly one kernel of its pass
    assert kern["tc_prep"] == _bytes(["q", "k", "g", "b"], gs)
    assert kern["tc_fwd"] == _bytes(["v", "w", "o"], gs)
    assert kern["tc_bwd_grad"] == _bytes(["dq", "dk", "db", "dg"], gs)
    assert kern["tc_prep"] + kern["tc_fwd"] == fwd
    assert kern["tc_bwd_state"] + kern["tc_bwd_grad"] == bwd


def test_headline_bytes_are_the_float32_gate_model():
    assert (bench.FWD_BYTES, bench.BWD_BYTES) == (2560, 4864)
    # workload 2: B 4, T 4096, H 16 token-heads
    assert (bench.FWD_BYTES + bench.BWD_BYTES) * 4 * 4096 * 16 == 1_946_157_056


def test_traffic_record_applies_only_to_unchanged_sources(tmp_path, monkeypatch):
    rec = {"tc_fwd": {"dram_bytes_per_launch": 123, "src_sha256": "abc"}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("tc_fwd", "abc") == 123
    assert bench.traffic_from_profiles("tc_fwd", "def") is None
    assert bench.traffic_from_profiles("tc_prep", "abc") is None


def test_source_hash_covers_the_kernel_and_the_shared_headers():
    for k in bench.TC_KERNEL_SOURCES:
        h = bench.sources_hash(k)
        assert len(h) == 64 and h == bench.sources_hash(k)
    # different kernels hash different files
    assert len({bench.sources_hash(k) for k in bench.TC_KERNEL_SOURCES}) == len(bench.TC_KERNEL_SOURCES)
