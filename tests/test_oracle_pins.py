"""Pins for the float64 oracle: each check ties it to something other than itself.

* the worked example printed on the page "Efficient Transformers: Linear Attention and
  Flash Attention", section "Worked example: the reassociation trick, by hand"
  (tests/golden/worked_example.txt);
* the quadratic brute force (phi(Q) phi(K)^T masked, row-normalised, times V): the
  left-hand side of the associativity law stated in that page's section "Linear
  attention: reordering the matmuls, not shrinking them";
* the recurrence of the section "The recurrent view: attention as an RNN": a decode
  replayed token by token equals the causal forward;
* special values of phi(x) = elu(x) + 1 and the invariants that follow from phi > 0
  (the page's answer A4: the weights form a convex combination);
* the closed forms and tables printed on the pages "Linear Attention > Memory
  Efficiency" and "Linear Attention > Computational Complexity Analysis".

The last test builds the oracle with each planted mistake and checks that these pins
catch every one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import PHI_ELU1, PHI_IDENTITY

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------ fixtures
def _parse_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rhs = (s.strip() for s in line.split("=", 1))
            rows = [[Fraction(tok) for tok in row.split()] for row in rhs.split(";")]
            vals[key] = rows
    return vals


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _rand(seed, shape):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------------------ the pin suite
# Each check returns None when it holds, or a message.  The suite runs against any
# Oracle instance so that the mutation test can run it on planted variants.
def check_phi(orc):
    cases = [(0.0, 1.0), (1.0, 2.0), (2.5, 3.5), (-1.0, math.exp(-1.0)),
             (-3.0, math.exp(-3.0)), (1e-300, 1.0), (-1e-300, 1.0)]
    for x, want in cases:
        got = orc.phi(x)
        if abs(got - want) > 1e-15 * max(1.0, abs(want)):
            return f"phi({x}) = {got}, want {want}"
    if not orc.phi(-700.0) > 0.0:
        return "phi must stay positive"
    return None


def check_worked_example(orc):
    g = _parse_golden("worked_example.txt")
    Q = np.array(g["Q"], dtype=np.float64)
    K = np.array(g["K"], dtype=np.float64)
    V = np.array(g["V"], dtype=np.float64)
    want_out = np.array([[float(x) for x in r] for r in g["out"]])
    out = orc.forward(Q, K, V, causal=False, phi_kind=PHI_IDENTITY)
    if np.max(np.abs(out - want_out)) > 1e-15:
        return f"worked example outputs {out.tolist()} != {want_out.tolist()}"
    S, z = orc.state(K, V, phi_kind=PHI_IDENTITY)
    if not np.array_equal(S, np.array(g["KtV"], dtype=np.float64)):
        return f"worked example K^T V {S.tolist()}"
    if not np.array_equal(z, np.array(g["k_sum"][0], dtype=np.float64)):
        return f"worked example k_sum {z.tolist()}"
    return None


def check_brute_force(orc):
    for seed, (n, d) in enumerate([(1, 2), (2, 2), (3, 4), (17, 4), (33, 8), (64, 8), (5, 3)]):
        q, k, v = _rand([seed, 0], (n, d)), _rand([seed, 1], (n, d)), _rand([seed, 2], (n, d))
        for causal in (False, True):
            ref = oracle.brute_force(q, k, v, causal)
            got = orc.forward(q, k, v, causal)
            err = np.max(np.abs(got - ref)) / max(1e-300, np.max(np.abs(ref)))
            if not np.isfinite(err) or err > 1e-12:
                return f"brute force n={n} d={d} causal={causal}: rel err {err}"
    return None


def check_decode_replay(orc):
    n, d = 40, 8
    q, k, v = _rand([7, 0], (2, n, d)), _rand([7, 1], (2, n, d)), _rand([7, 2], (2, n, d))
    ref = orc.forward(q, k, v, causal=True)
    S = np.zeros((2, d, d))
    z = np.zeros((2, d))
    for t in range(n):
        S, z, out = orc.decode_step(S, z, q[:, t], k[:, t], v[:, t])
        err = np.max(np.abs(out - ref[:, t])) / np.max(np.abs(ref[:, t]))
        if not np.isfinite(err) or err > 1e-12:
            return f"decode replay step {t}: rel err {err}"
    S_ref, z_ref = orc.state(k, v)
    if np.max(np.abs(S - S_ref)) > 1e-12 * np.max(np.abs(S_ref)) or \
            np.max(np.abs(z - z_ref)) > 1e-12 * np.max(np.abs(z_ref)):
        return "decode replay final state differs from state()"
    return None


def check_rows(orc):
    n, d = 50, 4
    q, k, v = _rand([9, 0], (3, n, d)), _rand([9, 1], (3, n, d)), _rand([9, 2], (3, n, d))
    rows = [0, 7, 7, 31, 49]
    for causal in (False, True):
        full = orc.forward(q, k, v, causal)
        part = orc.forward_rows(q, k, v, rows, causal)
        if not np.array_equal(part, full[:, rows]):
            return f"forward_rows causal={causal} differs from forward"
    return None


PIN_SUITE = [check_phi, check_worked_example, check_brute_force, check_decode_replay, check_rows]


def run_suite(orc):
    failures = []
    for check in PIN_SUITE:
        with np.errstate(all="ignore"):
            msg = check(orc)
        if msg:
            failures.append(f"{check.__name__}: {msg}")
    return failures


# ------------------------------------------------------------------------ tests
def test_phi_special_values(orc):
    assert check_phi(orc) is None


def test_worked_example_from_page(orc):
    assert check_worked_example(orc) is None


def test_brute_force_reproduces_worked_example():
    """The quadratic form itself reproduces the page's standard-path weights and outputs."""
    g = _parse_golden("worked_example.txt")
    Q = np.array(g["Q"], dtype=np.float64)
    K = np.array(g["K"], dtype=np.float64)
    V = np.array(g["V"], dtype=np.float64)
    scores = Q @ K.T
    assert np.array_equal(scores, np.array(g["scores"], dtype=np.float64))
    weights = np.array([[float(x) for x in r] for r in g["weights"]])
    assert np.allclose(scores / scores.sum(1, keepdims=True), weights, rtol=0, atol=1e-15)
    out = oracle.brute_force(Q, K, V, causal=False, phi_kind=PHI_IDENTITY)
    want = np.array([[float(x) for x in r] for r in g["out"]])
    assert np.max(np.abs(out - want)) <= 1e-15


def test_brute_force_agreement(orc):
    assert check_brute_force(orc) is None


def test_decode_replay_equals_causal_forward(orc):
    assert check_decode_replay(orc) is None


def test_forward_rows_matches_forward(orc):
    assert check_rows(orc) is None


@pytest.mark.parametrize("causal", [False, True])
def test_invariants(orc, causal):
    rng = np.random.default_rng(11)
    n, d = 37, 6
    q = rng.standard_normal((n, d))
    k = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    out = orc.forward(q, k, v, causal)
    # 1. constant value rows give that constant (the weights sum to one)
    c = rng.standard_normal(d)
    out_c = orc.forward(q, k, np.tile(c, (n, 1)), causal)
    assert np.max(np.abs(out_c - c)) < 1e-12
    # 2. identical keys give the plain (prefix) mean of the values, whatever Q is
    k_eq = np.tile(rng.standard_normal(d), (n, 1))
    out_eq = orc.forward(q, k_eq, v, causal)
    if causal:
        want = np.cumsum(v, 0) / np.arange(1, n + 1)[:, None]
    else:
        want = np.tile(v.mean(0), (n, 1))
    assert np.max(np.abs(out_eq - want)) < 1e-12
    # 3. a single token returns its own value
    assert np.max(np.abs(orc.forward(q[:1], k[:1], v[:1], causal) - v[:1])) < 1e-12
    # 6. linear in V
    v2 = rng.standard_normal((n, d))
    lin = orc.forward(q, k, 2.0 * v - 3.0 * v2, causal)
    assert np.max(np.abs(lin - (2.0 * out - 3.0 * orc.forward(q, k, v2, causal)))) < 1e-11
    # 8. every output lies within the range of the values it averages
    for i in range(n):
        vis = v[: i + 1] if causal else v
        assert np.all(out[i] >= vis.min(0) - 1e-12) and np.all(out[i] <= vis.max(0) + 1e-12)


def test_causal_last_row_is_noncausal_and_permutation(orc):
    rng = np.random.default_rng(12)
    n, d = 29, 5
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    nc = orc.forward(q, k, v, False)
    ca = orc.forward(q, k, v, True)
    # 4. the last causal row sees every token
    assert np.max(np.abs(ca[-1] - nc[-1])) < 1e-12
    # 5. non-causal output does not depend on the order of the (key, value) pairs
    perm = rng.permutation(n)
    assert np.max(np.abs(orc.forward(q, k[perm], v[perm], False) - nc)) < 1e-12


def test_state_bytes_closed_form_and_table():
    """D*d*4 + D*4 bytes: 16,640 at d = D = 64 for every n, and the printed table."""
    assert oracle.memory_linear_attention(128, 64) == 16640
    assert oracle.memory_linear_attention(65536, 128) == 66048
    for seq, std_mb, lin_kb, red in _table("memory_table.txt"):
        n = int(seq)
        std = oracle.memory_standard_attention(n, 64)
        lin = oracle.memory_linear_attention(n, 64)
        assert lin == 16640
        assert f"{std / 1e6:.1f}" == std_mb
        assert f"{lin / 1024:.1f}" == lin_kb
        assert f"{std / lin:.0f}" == red


def _fmt_flops(x):
    return f"{x / 1e9:.2f}G" if x >= 1e9 else f"{x / 1e6:.1f}M"


def test_flops_closed_form_and_table():
    """2nd + 2nDd + 2nDd + 2nD + n reproduces every printed row."""
    assert oracle.flops_linear_attention(128, 64) == 2130048
    assert oracle.flops_linear_attention(16384, 64) == 272646144
    for seq, std_s, lin_s, speed in _table("flops_table.txt"):
        n = int(seq)
        std = oracle.flops_standard_attention(n, 64)
        lin = oracle.flops_linear_attention(n, 64)
        assert _fmt_flops(std) == std_s
        assert _fmt_flops(lin) == lin_s
        assert f"{std / lin:.1f}" == speed


def test_default_oracle_passes_suite(orc):
    assert orc.plant == 0
    assert run_suite(orc) == []


@pytest.mark.parametrize("plant", [1, 2, 3, 4, 5])
def test_pins_catch_planted_mistakes(plant):
    """Plant one mistake at a time in the oracle (CPU only) and check a pin fails:
    1 exclusive causal diagonal, 2 transposed state, 3 dropped normaliser,
    4 phi without its +1, 5 decode reading the state before the update."""
    bad = oracle.load_planted(plant)
    assert bad.plant == plant
    assert run_suite(bad), f"planted mistake {plant} went unnoticed"
