"""Pins of the oracle's FAVOR+ features (Performer's positive random features, named on the
page "Efficient Transformers: Linear Attention and Flash Attention" as random features that
approximate the softmax kernel exp(q . k)).

They are pinned by that property itself, not by re-evaluating their formula:
  - unbiasedness: over many random rows w ~ N(0, I), phi(q) . phi(k) -> exp(q . k), within the
    Monte Carlo error;
  - attention with these features (the kernelised formula, identity feature map) approaches
    exact softmax attention (exp(q . k) weights, written out in numpy) as m grows;
  - W = 0 gives the closed form exp(-|x|^2 / 2) / sqrt(m) in every feature;
  - a planted mistake (the -|x|^2/2 term dropped) is caught.
"""
import numpy as np
import pytest

import oracle


def _unbiased_check(orc, seed):
    rng = np.random.default_rng(seed)
    d, m = 4, 400_000
    q, k = rng.standard_normal(d) * 0.5, rng.standard_normal(d) * 0.5
    W = rng.standard_normal((m, d))
    fq, fk = orc.favor_features(q, W), orc.favor_features(k, W)
    terms = fq * fk * m                     # m samples of exp(w.q - |q|^2/2) exp(w.k - |k|^2/2)
    est, se = terms.mean(), terms.std() / np.sqrt(m)
    return abs(est - np.exp(q @ k)) / se


def test_features_estimate_the_softmax_kernel():
    assert _unbiased_check(oracle.default(), 0) < 5.0


def test_attention_with_features_approaches_softmax_attention():
    rng = np.random.default_rng(1)
    n, d = 24, 4
    q, k, v = (rng.standard_normal((n, d)) * 0.4 for _ in range(3))
    for causal in (False, True):
        w = np.exp(q @ k.T)
        if causal:
            w = np.tril(w)
        exact = (w / w.sum(1, keepdims=True)) @ v
        errs = []
        for m in (1_000, 100_000):
            W = rng.standard_normal((m, d))
            fq, fk = oracle.favor_features(q, W), oracle.favor_features(k, W)
            # the kernelised formula on these features (m > d, so the quadratic form)
            approx = oracle.brute_force(fq, fk, v, causal, phi_kind=oracle.PHI_IDENTITY)
            errs.append(np.max(np.abs(approx - exact)))
        assert errs[1] < 0.02 and errs[1] < errs[0]


def test_zero_projection_closed_form():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 8))
    f = oracle.favor_features(x, np.zeros((16, 8)))
    want = np.exp(-0.5 * (x * x).sum(1)) / 4.0
    assert np.allclose(f, want[:, None], rtol=1e-15, atol=0)


def test_planted_favor_mistake_is_caught():
    orc = oracle.load_planted(8)
    assert orc.plant == 8
    assert _unbiased_check(orc, 0) > 50.0


# ------------------------------------------------------------------ features of their own size
# The pass on m features with d-dimensional values (S is m x d; page "Linear Attention > Memory
# Efficiency" writes the state as D x d with D the feature dimension) is pinned by the
# quadratic form written out in numpy, which never forms S, for m < d and m > d, both modes.
@pytest.mark.parametrize("m,d", [(3, 5), (8, 2), (16, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_forward_on_m_features_matches_brute_force(m, d, causal):
    rng = np.random.default_rng(10 * m + d)
    n = 37
    fq, fk = (np.abs(rng.standard_normal((2, n, m))) + 0.05 for _ in range(2))
    v = rng.standard_normal((2, n, d))
    got = oracle.forward(fq, fk, v, causal, phi_kind=oracle.PHI_IDENTITY)
    assert got.shape == v.shape
    for h in range(2):  # the brute force takes one head
        ref = oracle.brute_force(fq[h], fk[h], v[h], causal, phi_kind=oracle.PHI_IDENTITY)
        assert np.max(np.abs(got[h] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_forward_on_m_features_reduces_to_the_square_pass():
    """With m = d padded by zero features, the result equals the m = d pass (zero features add
    nothing to S, z or the denominators)."""
    rng = np.random.default_rng(11)
    n, d = 29, 4
    fq, fk = (np.abs(rng.standard_normal((n, d))) + 0.1 for _ in range(2))
    v = rng.standard_normal((n, d))
    pad = lambda x: np.concatenate([x, np.zeros((n, 3))], axis=1)  # noqa: E731
    for causal in (False, True):
        sq = oracle.forward(fq, fk, v, causal, phi_kind=oracle.PHI_IDENTITY)
        wide = oracle.forward(pad(fq), pad(fk), v, causal, phi_kind=oracle.PHI_IDENTITY)
        assert np.max(np.abs(sq - wide)) <= 1e-13


def test_planted_transposed_state_is_caught_with_m_features():
    orc = oracle.load_planted(2)  # S indexed as [value][feature]
    rng = np.random.default_rng(12)
    fq, fk = (np.abs(rng.standard_normal((20, 6))) + 0.1 for _ in range(2))
    v = rng.standard_normal((20, 3))
    got = orc.forward(fq, fk, v, True, phi_kind=oracle.PHI_IDENTITY)
    ref = oracle.brute_force(fq, fk, v, True, phi_kind=oracle.PHI_IDENTITY)
    assert np.max(np.abs(got - ref)) > 1e-3
