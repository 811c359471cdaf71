"""Pins of the float64 backward oracle (gradients of sum(g * out) with respect to q, k, v).

The pages give no backward formulas, so the oracle differentiates the forward pass they
define.  It is pinned against things that do not share its code:
  - central finite differences of the forward oracle (itself pinned in test_oracle_pins);
  - torch.autograd through an independent float64 brute force (phi(Q) phi(K)^T, masked,
    row-normalised, times V);
  - identities of the method: sum_j dL/dv_j = sum_i g_i (each output row is a convex
    combination of the values), and a constant V makes the output independent of q and k;
  - planted mistakes (the normaliser's term dropped; the chain rule through phi dropped)
    that these pins must catch.
"""
import numpy as np
import pytest

import oracle


def _fd_grads(q, k, v, g, causal, forward, h=1e-6):
    grads = []
    for which in range(3):
        base = [q, k, v]
        X = base[which]
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            ap, am = list(base), list(base)
            ap[which], am[which] = Xp, Xm
            num[idx] = ((g * forward(*ap, causal)).sum() - (g * forward(*am, causal)).sum()) / (2 * h)
        grads.append(num)
    return grads


def _rel(a, b):
    # relative to the gradient's size, with a floor of 1: some gradients vanish exactly
    # (one token: the output is v whatever q and k are)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1.0))


def _fd_check(orc, seed):
    rng = np.random.default_rng(seed)
    worst = 0.0
    for causal in (True, False):
        for n, d in ((1, 2), (5, 3), (9, 2)):
            q, k, v, g = (rng.standard_normal((2, n, d)) for _ in range(4))
            got = orc.backward(q, k, v, g, causal)
            ref = _fd_grads(q, k, v, g, causal, oracle.forward)
            worst = max(worst, max(_rel(a, b) for a, b in zip(got, ref)))
    return worst


def test_backward_matches_finite_differences():
    assert _fd_check(oracle.default(), 0) <= 1e-7


def test_backward_matches_autograd_brute_force():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    for causal in (True, False):
        q, k, v, g = (rng.standard_normal((3, 48, 8)) for _ in range(4))
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))

        def phi(x):
            return torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))

        W = phi(tq) @ phi(tk).transpose(-1, -2)
        if causal:
            W = torch.tril(W)
        out = (W / W.sum(-1, keepdim=True)) @ tv
        (out * torch.tensor(g)).sum().backward()
        got = oracle.backward(q, k, v, g, causal)
        for a, b in zip(got, (tq.grad, tk.grad, tv.grad)):
            assert _rel(a, b.numpy()) <= 1e-12


@pytest.mark.parametrize("causal", [True, False])
def test_value_gradients_sum_to_output_gradients(causal):
    rng = np.random.default_rng(2)
    q, k, v, g = (rng.standard_normal((2, 200, 16)) / 4 for _ in range(4))
    _, _, dv = oracle.backward(q, k, v, g, causal)
    assert np.allclose(dv.sum(axis=1), g.sum(axis=1), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_constant_values_give_no_query_or_key_gradient(causal):
    rng = np.random.default_rng(3)
    q, k, g = (rng.standard_normal((2, 100, 8)) for _ in range(3))
    v = np.broadcast_to(rng.standard_normal(8), q.shape).copy()
    dq, dk, dv = oracle.backward(q, k, v, g, causal)
    assert np.max(np.abs(dq)) <= 1e-12 and np.max(np.abs(dk)) <= 1e-12
    assert np.max(np.abs(dv)) > 1e-3


@pytest.mark.parametrize("plant", [6, 7])
def test_planted_backward_mistakes_are_caught(plant):
    orc = oracle.load_planted(plant)
    assert orc.plant == plant
    assert _fd_check(orc, 0) > 1e-3
