"""Pins of the fp64 oracle against what the pages and the mathematics fix.

CPU only.  Sources ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
Attention"): the update (LIT-802 review, Key takeaways 1, Sec. 3.1
Eqs. 8-10), the KDA and Gated DeltaNet ties (App. A.5), chunkwise = token-wise
and fp64 gradient agreement (Key takeaways 2, Secs. 3.3-3.4, App. D.6), the
delta rule's overwrite behaviour (digg thread 7/), and the [0, 2] erase range
(Table 5 note).
"""

import glob
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import chunkwise, fd
from gated_delta_rule_128_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NAMES = ("q", "k", "v", "g", "b", "w", "S0")
GRADS = ("dq", "dk", "dv", "dg", "db", "dw", "dS0")


def rel(a, ref):
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(a - ref)) / (den if den > 0 else 1.0))


def inputs64(B, T, H, dk, dv, seed, s0_std=0.5, tie=None, erase_scale=1.0, dST=True):
    d = workloads.draw(B, T, H, dk, dv, seed, s0_std=s0_std, tie=tie,
                       erase_scale=erase_scale, with_dST=dST)
    return {n: x.double().numpy() for n, x in d.items()}


# ------------------------------------------------------------ golden cases

def _parse(path):
    vals = {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        name, *rest = line.split()
        vals[name] = rest
    return vals


def test_hand_worked_example():
    v = _parse(os.path.join(GOLDEN, "hand_2x2.txt"))
    f = lambda n: np.array([float(x) for x in v[n]])  # noqa: E731
    shape_tok = (1, 1, 1, 2)
    g = np.log(f("alpha")).reshape(shape_tok)
    o, ST = oracle.forward(f("q").reshape(shape_tok), f("k").reshape(shape_tok),
                           f("v").reshape(shape_tok), g, f("b").reshape(shape_tok),
                           f("w").reshape(shape_tok), f("S0").reshape(1, 1, 2, 2))
    np.testing.assert_allclose(ST.reshape(-1), f("S1"), rtol=0, atol=1e-15)
    np.testing.assert_allclose(o.reshape(-1), f("o"), rtol=0, atol=1e-15)


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "literal_*.txt"))))
def test_literal_matrix_form_golden(path):
    v = _parse(path)
    T, dk, dv = (int(x) for x in v["dims"])
    fr = lambda n: np.array([float(Fraction(x)) for x in v[n]])  # noqa: E731
    tok = {n: np.stack([fr(f"{n}{t}") for t in range(T)]) for n in ("q", "k", "v", "alpha", "b", "w")}
    sh = lambda x: x.reshape(1, T, 1, -1)  # noqa: E731
    o, ST = oracle.forward(sh(tok["q"]), sh(tok["k"]), sh(tok["v"]), sh(np.log(tok["alpha"])),
                           sh(tok["b"]), sh(tok["w"]), fr("S0").reshape(1, 1, dk, dv))
    o_ref = np.stack([fr(f"o{t}") for t in range(T)])
    assert rel(o[0, :, 0], o_ref) < 1e-13
    assert rel(ST.reshape(-1), fr("ST")) < 1e-13


# ---------------------------------------------------------- tie identities

@pytest.mark.parametrize("dk,dv", [(16, 8), (32, 32)])
def test_kda_tie_forward(dk, dv):
    x = inputs64(2, 96, 2, dk, dv, 11, tie="kda")
    o, ST = oracle.forward(*(x[n] for n in NAMES))
    o2, ST2 = oracle.kda_forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    assert rel(o, o2) < 1e-13 and rel(ST, ST2) < 1e-13


@pytest.mark.parametrize("dk,dv", [(16, 8), (32, 32)])
def test_gdn_tie_forward(dk, dv):
    x = inputs64(2, 96, 2, dk, dv, 12, tie="gdn")
    o, ST = oracle.forward(*(x[n] for n in NAMES))
    o2, ST2 = oracle.gdn_forward(x["q"], x["k"], x["v"], x["alpha_log"], x["beta"], x["S0"])
    assert rel(o, o2) < 1e-13 and rel(ST, ST2) < 1e-13


def test_untied_gates_differ_from_kda():
    # Sanity: with independent b and w the result is not KDA's.
    x = inputs64(1, 32, 1, 8, 8, 13)
    o, _ = oracle.forward(*(x[n] for n in NAMES))
    beta = x["b"].mean(-1)
    o2, _ = oracle.kda_forward(x["q"], x["k"], x["v"], x["g"], beta, x["S0"])
    assert rel(o, o2) > 1e-3


def test_kda_tie_gradients():
    """With b = w = beta 1, the Gated Delta Rule-2 reverse mode gives KDA's
    gradients: equal dq, dk, dv, dg, dS0, and dbeta = sum_c db_c + sum_c dw_c."""
    x = inputs64(1, 7, 1, 4, 3, 14, tie="kda")
    gr = oracle.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], ckpt=3)
    kda = lambda q, k, v, g, beta, S0: oracle.kda_forward(q, k, v, g, beta, S0, nthreads=1)  # noqa
    fdg = fd.gradients(x, x["dO"], x["dST"], fn=kda, names=("q", "k", "v", "g", "beta", "S0"))
    for n in ("dq", "dk", "dv", "dg", "dS0"):
        assert rel(gr[n], fdg[n]) < 1e-7, n
    dbeta = gr["db"].sum(-1) + gr["dw"].sum(-1)
    assert rel(dbeta, fdg["dbeta"]) < 1e-7


def test_gdn_tie_gradients():
    """With also g = a 1, the scalar decay gradient is the channel sum of dg."""
    x = inputs64(1, 7, 1, 4, 3, 15, tie="gdn")
    gr = oracle.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], ckpt=4)
    gdn = lambda q, k, v, a, beta, S0: oracle.gdn_forward(q, k, v, a, beta, S0, nthreads=1)  # noqa
    fdg = fd.gradients(x, x["dO"], x["dST"], fn=gdn,
                       names=("q", "k", "v", "alpha_log", "beta", "S0"))
    for n in ("dq", "dk", "dv", "dS0"):
        assert rel(gr[n], fdg[n]) < 1e-7, n
    assert rel(gr["dg"].sum(-1), fdg["dalpha_log"]) < 1e-7
    assert rel(gr["db"].sum(-1) + gr["dw"].sum(-1), fdg["dbeta"]) < 1e-7


# ----------------------------------------------------- gradients vs calculus

@pytest.mark.parametrize("erase_scale", [1.0, 2.0])
def test_token_backward_matches_finite_differences(erase_scale):
    x = inputs64(1, 12, 1, 4, 5, 16, erase_scale=erase_scale)
    gr = oracle.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], ckpt=5)
    fdg = fd.gradients(x, x["dO"], x["dST"])
    for n in GRADS:
        assert rel(gr[n], fdg[n]) < 1e-7, n


def test_token_backward_independent_of_checkpoint_spacing():
    x = inputs64(2, 37, 2, 8, 6, 17)
    ref = oracle.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], ckpt=1)
    for ck in (4, 16, 64):
        gr = oracle.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], ckpt=ck)
        for n in GRADS:
            assert rel(gr[n], ref[n]) < 1e-14, (ck, n)


# -------------------------------------------------- chunkwise == token-wise

@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 256])
def test_chunkwise_forward_equals_tokenwise(chunk, T):
    x = inputs64(1, T, 2, 8, 8, 20 + T)
    o, ST = oracle.forward(*(x[n] for n in NAMES))
    o2, ST2 = chunkwise.forward(*(x[n] for n in NAMES), chunk=chunk)
    assert rel(o2, o) < 1e-12 and rel(ST2, ST) < 1e-12


def test_chunkwise_forward_negative_eigenvalue_range():
    # erase gate in [0, 2]: the eigenvalue 1 - sum_c b_c k_c^2 reaches [-1, 1]
    x = inputs64(1, 130, 2, 16, 8, 21, erase_scale=2.0)
    o, ST = oracle.forward(*(x[n] for n in NAMES))
    o2, ST2 = chunkwise.forward(*(x[n] for n in NAMES), chunk=64)
    assert rel(o2, o) < 1e-12 and rel(ST2, ST) < 1e-12


@pytest.mark.parametrize("chunk,T", [(16, 40), (32, 64), (64, 65)])
def test_chunkwise_backward_equals_tokenwise(chunk, T):
    x = inputs64(1, T, 2, 8, 6, 22 + T)
    ref = oracle.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], ckpt=chunk)
    gr = chunkwise.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], chunk=chunk)
    for n in GRADS:
        assert rel(gr[n], ref[n]) < 1e-11, n


def test_chunkwise_backward_matches_finite_differences():
    x = inputs64(1, 11, 1, 3, 4, 23, erase_scale=2.0)
    gr = chunkwise.backward(*(x[n] for n in NAMES), x["dO"], x["dST"], chunk=4)
    fdg = fd.gradients(x, x["dO"], x["dST"])
    for n in GRADS:
        assert rel(gr[n], fdg[n]) < 1e-7, n


# ------------------------------------------------------------- closed forms

def test_no_erase_is_decayed_linear_attention():
    """b = 0: S_t = D_t S_{t-1} + k_t (w.v)_t^T, so
    o_t = sum_{j<=t} (q_t . e^{G_t - G_j}) . k_j  u_j  +  (q_t . e^{G_t})^T S0,
    with G the running (global) cumsum of g: an O(T^2) direct sum."""
    x = inputs64(1, 50, 1, 6, 5, 24)
    x["b"] = np.zeros_like(x["b"])
    q, k, g = x["q"][0, :, 0], x["k"][0, :, 0], x["g"][0, :, 0]
    u = (x["w"] * x["v"])[0, :, 0]
    S0 = x["S0"][0, 0]
    G = np.cumsum(g, axis=0)
    ref = np.zeros_like(u)
    for t in range(len(q)):
        ref[t] = (q[t] * np.exp(G[t])) @ S0
        for j in range(t + 1):
            ref[t] += np.sum(q[t] * np.exp(G[t] - G[j]) * k[j]) * u[j]
    o, _ = oracle.forward(*(x[n] for n in NAMES))
    o2, _ = chunkwise.forward(*(x[n] for n in NAMES), chunk=16)
    assert rel(o[0, :, 0], ref) < 1e-13
    assert rel(o2[0, :, 0], ref) < 1e-12


def test_no_erase_no_decay_is_causal_linear_attention():
    x = inputs64(1, 40, 1, 6, 5, 25, s0_std=0.0)
    x["b"] = np.zeros_like(x["b"])
    x["g"] = np.zeros_like(x["g"])
    q, k = x["q"][0, :, 0], x["k"][0, :, 0]
    u = (x["w"] * x["v"])[0, :, 0]
    ref = np.tril(q @ k.T) @ u
    o, _ = oracle.forward(*(x[n] for n in NAMES))
    assert rel(o[0, :, 0], ref) < 1e-13


def test_delta_rule_overwrite_and_fresh_key():
    """g = 0, b = w = 1, orthonormal keys: a repeated key overwrites its value,
    a fresh key acts as a plain add (digg thread 7/)."""
    dk = dv = 4
    e = np.eye(dk)
    vals = np.array([[1.0, 2, 3, 4], [-5.0, 6, 7, -8], [0.5, 0.25, -1, 9]])
    keys = [e[0], e[0], e[1]]
    queries = [e[0], e[0], e[0]]
    tok = lambda a: np.stack(a).reshape(1, 3, 1, -1)  # noqa: E731
    ones = np.ones((1, 3, 1, dk))
    o, ST = oracle.forward(tok(queries), tok(keys), vals.reshape(1, 3, 1, dv),
                           np.zeros((1, 3, 1, dk)), ones, np.ones((1, 3, 1, dv)), None)
    np.testing.assert_array_equal(o[0, 0, 0], vals[0])
    np.testing.assert_array_equal(o[0, 1, 0], vals[1])   # overwritten, not added
    np.testing.assert_array_equal(o[0, 2, 0], vals[1])   # untouched by the fresh key
    np.testing.assert_array_equal(ST[0, 0] .T @ e[1], vals[2])  # fresh key: plain add
    np.testing.assert_array_equal(ST[0, 0].T @ e[0], vals[1])


def test_erase_eigenvalue_with_widened_gate():
    """The erase operator I - k (b.k)^T maps k to (1 - sum_c b_c k_c^2) k; with
    b in [0, 2] and |k| = 1 that eigenvalue lies in [-1, 1] (Table 5 note)."""
    rng = np.random.default_rng(5)
    dk = dv = 6
    k = rng.normal(size=dk)
    k /= np.linalg.norm(k)
    b = 2.0 * np.ones(dk)
    S0 = np.outer(k, rng.normal(size=dv))
    lam = 1.0 - np.sum(b * k * k)
    assert abs(lam + 1.0) < 1e-14
    sh = lambda a: a.reshape(1, 1, 1, -1)  # noqa: E731
    _, ST = oracle.forward(sh(k), sh(k), sh(np.zeros(dv)), sh(np.zeros(dk)), sh(b),
                           sh(np.ones(dv)), S0.reshape(1, 1, dk, dv))
    np.testing.assert_allclose(ST[0, 0], lam * S0, atol=1e-14)


# ---------------------------------------------------------------- invariants

def test_linearity_in_state_and_value():
    x = inputs64(1, 33, 2, 8, 6, 26)
    y = inputs64(1, 33, 2, 8, 6, 27)
    a = 0.7
    mix = dict(x)
    mix["v"] = x["v"] + a * y["v"]
    mix["S0"] = x["S0"] + a * y["S0"]
    yy = dict(x)
    yy["v"], yy["S0"] = y["v"], y["S0"]
    o1, S1 = oracle.forward(*(x[n] for n in NAMES))
    o2, S2 = oracle.forward(*(yy[n] for n in NAMES))
    o3, S3 = oracle.forward(*(mix[n] for n in NAMES))
    assert rel(o3, o1 + a * o2) < 1e-13 and rel(S3, S1 + a * S2) < 1e-13


def test_resume_from_final_state():
    x = inputs64(2, 70, 2, 8, 8, 28)
    o, ST = oracle.forward(*(x[n] for n in NAMES))
    T1 = 29
    first = {n: x[n][:, :T1] for n in NAMES if n != "S0"}
    second = {n: x[n][:, T1:] for n in NAMES if n != "S0"}
    oa, Sa = oracle.forward(*(first[n] for n in NAMES[:-1]), x["S0"])
    ob, Sb = oracle.forward(*(second[n] for n in NAMES[:-1]), Sa)
    assert rel(np.concatenate([oa, ob], axis=1), o) < 1e-14 and rel(Sb, ST) < 1e-14


def test_value_permutation_permutes_outputs():
    x = inputs64(1, 40, 2, 8, 8, 29)
    perm = np.random.default_rng(0).permutation(8)
    y = dict(x)
    y["v"], y["w"] = x["v"][..., perm], x["w"][..., perm]
    y["S0"] = x["S0"][..., perm]
    o, ST = oracle.forward(*(x[n] for n in NAMES))
    o2, ST2 = oracle.forward(*(y[n] for n in NAMES))
    assert rel(o2, o[..., perm]) < 1e-14 and rel(ST2, ST[..., perm]) < 1e-14


def test_decode_is_one_token_of_the_recurrence():
    x = inputs64(3, 5, 2, 8, 8, 30)
    o, ST = oracle.forward(*(x[n] for n in NAMES))
    S = x["S0"]
    for t in range(5):
        tok = [x[n][:, t:t + 1] for n in NAMES[:-1]]
        ot, S = oracle.forward(*tok, S)
        assert rel(ot[:, 0], o[:, t]) < 1e-14
    assert rel(S, ST) < 1e-14


# ------------------------------------- the pins catch plausible mistakes

def test_pins_reject_planted_mistakes(monkeypatch):
    """Plant a mistake in the chunkwise oracle (a wrong mask on A, a sign
    flip in the inverse) and check that the chunkwise == token-wise pin fails."""
    x = inputs64(1, 48, 1, 8, 8, 31)
    o, _ = oracle.forward(*(x[n] for n in NAMES))
    real = chunkwise._chunk_factors

    def non_strict_mask(*a):
        f = real(*a)
        f["A"] = np.tril(f["Kc"] @ f["Kh"].T)
        f["T"] = np.linalg.inv(np.eye(len(f["A"])) + f["A"])
        f["W"], f["Up"] = f["T"] @ f["Kc"], f["T"] @ f["U"]
        return f

    def wrong_sign(*a):
        f = real(*a)
        f["T"] = np.linalg.inv(np.eye(len(f["A"])) - f["A"])
        f["W"], f["Up"] = f["T"] @ f["Kc"], f["T"] @ f["U"]
        return f

    for bad in (non_strict_mask, wrong_sign):
        monkeypatch.setattr(chunkwise, "_chunk_factors", bad)
        o2, _ = chunkwise.forward(*(x[n] for n in NAMES), chunk=16)
        assert rel(o2, o) > 1e-3, bad.__name__
    monkeypatch.setattr(chunkwise, "_chunk_factors", real)
    o2, _ = chunkwise.forward(*(x[n] for n in NAMES), chunk=16)
    assert rel(o2, o) < 1e-12


def test_forward_substitution_inverse():
    rng = np.random.default_rng(1)
    A = np.tril(rng.normal(size=(20, 20)), -1) * 0.3
    T = chunkwise._forward_substitution_inverse(A)
    np.testing.assert_allclose(T @ (np.eye(20) + A), np.eye(20), atol=1e-12)
    assert math.isclose(np.linalg.det(T), 1.0, rel_tol=1e-12)


# ------------------------------------------------------ packed sequences

def _packed(x, lens):
    """Equal-length batch rows -> one packed row (for lens all equal to T)."""
    return {n: (t.reshape(1, -1, *t.shape[2:]) if t.dim() == 4 and n not in ("S0", "dST") else t)
            for n, t in x.items()}


def test_varlen_oracle_equals_the_batch_for_equal_lengths():
    """B rows of T tokens packed back to back with cu_seqlens = 0, T, 2T, ...
    give the batch oracle's results: each sequence starts from its own S0."""
    from oracle import varlen
    B, T, H, dk, dv = 3, 37, 2, 8, 6
    x = workloads.draw(B, T, H, dk, dv, 611, s0_std=0.3, with_dST=True)
    r = {n: t.double().numpy() for n, t in x.items()}
    o, ST = oracle.forward(*(r[n] for n in ("q", "k", "v", "g", "b", "w", "S0")))
    gr = oracle.backward(*(r[n] for n in ("q", "k", "v", "g", "b", "w", "S0")), r["dO"], r["dST"])
    p = {n: t.double().numpy() for n, t in _packed(x, None).items()}
    cu = [0, T, 2 * T, 3 * T]
    o2, ST2 = varlen.forward(*(p[n] for n in ("q", "k", "v", "g", "b", "w")), cu, p["S0"])
    gr2 = varlen.backward(*(p[n] for n in ("q", "k", "v", "g", "b", "w")), cu, p["S0"], p["dO"], p["dST"])
    assert np.array_equal(o2, o.reshape(1, B * T, H, dv)) and np.array_equal(ST2, ST)
    for n in ("dq", "dk", "dv", "dg", "db", "dw"):
        assert np.array_equal(gr2[n], gr[n].reshape(1, B * T, H, -1)), n
    assert np.array_equal(gr2["dS0"], gr["dS0"])


def test_varlen_oracle_sequences_are_independent():
    """Changing one sequence's inputs leaves every other sequence's outputs
    and gradients bit for bit; an empty sequence passes S0 through to S_T and
    dS_T through to dS0."""
    from oracle import varlen
    lens = [5, 1, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, dk, dv = int(cu[-1]), 2, 4, 3
    x = workloads.draw(1, T, H, dk, dv, 612, with_dST=True)
    S0 = workloads.draw(len(lens), 1, H, dk, dv, 613, s0_std=0.5)["S0"]
    dST = workloads.draw(len(lens), 1, H, dk, dv, 614, s0_std=0.5)["S0"]
    r = {n: t.double().numpy() for n, t in x.items()}
    names = ("q", "k", "v", "g", "b", "w")
    o, ST = varlen.forward(*(r[n] for n in names), cu, S0.double().numpy())
    gr = varlen.backward(*(r[n] for n in names), cu, S0.double().numpy(), r["dO"], dST.double().numpy())
    assert np.array_equal(ST[2], S0[2].double().numpy()) and np.array_equal(gr["dS0"][2], dST[2].double().numpy())
    r2 = dict(r)
    r2["v"] = r["v"].copy()
    r2["v"][:, 5] += 1.0            # the length-1 sequence
    o2, ST2 = varlen.forward(*(r2[n] for n in names), cu, S0.double().numpy())
    keep = np.r_[0:5, 6:T]
    assert np.array_equal(o2[:, keep], o[:, keep]) and not np.array_equal(o2[:, 5], o[:, 5])
    assert np.array_equal(ST2[[0, 2, 3]], ST[[0, 2, 3]]) and not np.array_equal(ST2[1], ST[1])


# ------------------------------------------------------ grouped value heads

def test_grouped_oracle_gradients_match_finite_differences():
    """H = 1 key head, H_v = 2 value heads: the grouped forward's gradients
    (the key side summed over the group) against central differences of the
    grouped forward itself."""
    from oracle import grouped
    B, T, H, Hv, dk, dv = 1, 7, 1, 2, 3, 2
    x = workloads.draw(B, T, H, dk, dv, 621)
    xv = workloads.draw(B, T, Hv, dk, dv, 622, s0_std=0.4, with_dST=True)
    r = {n: t.double().numpy() for n, t in x.items()}
    for n in ("v", "w", "S0", "dO", "dST"):
        r[n] = xv[n].double().numpy()
    names = ("q", "k", "v", "g", "b", "w", "S0")
    gr = grouped.backward(*(r[n] for n in names), r["dO"], r["dST"])
    num = fd.gradients({n: r[n] for n in names}, r["dO"], r["dST"], fn=grouped.forward)
    for n in names:
        assert np.max(np.abs(gr["d" + n] - num["d" + n])) < 1e-7, n


def test_grouped_oracle_is_the_plain_recurrence_per_value_head():
    """Each value head of a grouped call equals a plain call on its key head:
    value heads 2 and 3 of H = 2, H_v = 4 read key head 1."""
    from oracle import grouped
    B, T, H, Hv, dk, dv = 2, 9, 2, 4, 4, 3
    x = workloads.draw(B, T, H, dk, dv, 623)
    xv = workloads.draw(B, T, Hv, dk, dv, 624, s0_std=0.3)
    r = {n: t.double().numpy() for n, t in x.items()}
    for n in ("v", "w", "S0"):
        r[n] = xv[n].double().numpy()
    o, ST = grouped.forward(*(r[n] for n in ("q", "k", "v", "g", "b", "w", "S0")))
    o3, ST3 = oracle.forward(r["q"][:, :, 1:2], r["k"][:, :, 1:2], r["v"][:, :, 3:4], r["g"][:, :, 1:2],
                             r["b"][:, :, 1:2], r["w"][:, :, 3:4], r["S0"][:, 3:4])
    assert np.array_equal(o[:, :, 3:4], o3) and np.array_equal(ST[:, 3:4], ST3)


# ------------------------------------------------------ fused gate prologue

@pytest.mark.parametrize("b_scale", [1.0, 2.0])
def test_gate_logits_oracle_matches_finite_differences(b_scale):
    """Logits in: the chain-rule gradients of x_g, x_b, x_w against central
    differences of the logit forward; the activations themselves against
    their definitions at a few points."""
    from oracle import gates
    B, T, H, dk, dv = 1, 6, 1, 3, 2
    x = workloads.draw(B, T, H, dk, dv, 631, s0_std=0.3, with_dST=True)
    r = {n: t.double().numpy() for n, t in x.items()}
    gen = np.random.default_rng(632)
    xs = {"g": gen.normal(1.0, 1.5, r["g"].shape), "b": gen.normal(0, 1.5, r["b"].shape),
          "w": gen.normal(0, 1.5, r["w"].shape)}
    fn = lambda q, k, v, xg, xb, xw, S0: gates.forward(q, k, v, xg, xb, xw, S0, b_scale=b_scale)  # noqa: E731
    inputs = {"q": r["q"], "k": r["k"], "v": r["v"], "g": xs["g"], "b": xs["b"], "w": xs["w"], "S0": r["S0"]}
    gr = gates.backward(r["q"], r["k"], r["v"], xs["g"], xs["b"], xs["w"], r["S0"], r["dO"], r["dST"],
                        b_scale=b_scale)
    num = fd.gradients(inputs, r["dO"], r["dST"], fn=fn)
    for n in ("dg", "db", "dw", "dq", "dk", "dv", "dS0"):
        assert np.max(np.abs(gr[n] - num[n])) < 1e-7, n
    g, b, w = gates.activate(np.array([0.0, -40.0, 40.0]), np.array([0.0]), np.array([0.0]), b_scale)
    assert abs(g[0] + math.log(2.0)) < 1e-15 and abs(g[1] + 40.0) < 1e-12 and abs(g[2]) < 1e-17
    assert b[0] == 0.5 * b_scale and w[0] == 0.5
