"""Parity of the CUDA decode step (through the C ABI) with the float64 oracle, and the
recurrent-view identity on the device: decode replayed token by token equals the causal
forward (page "Efficient Transformers: Linear Attention and Flash Attention", section
"The recurrent view: attention as an RNN")."""
import numpy as np
import pytest

import oracle
from linear_attention_linattn_b200 import inputs
from tests.helpers import STATE_TOL_BF16, TOL, max_row_rel_err, to_dev, to_host

torch = pytest.importorskip("torch")
la = pytest.importorskip("linear_attention_linattn_b200")

pytestmark = pytest.mark.gpu


def _state_err(S, S_ref):
    d = S.shape[-1]
    a = S.reshape(-1, d * d)
    b = S_ref.reshape(-1, d * d)
    return float(np.max(np.linalg.norm(a - b, axis=1) / np.linalg.norm(b, axis=1)))


@pytest.mark.parametrize("d", [64, 128])
def test_decode_steps_match_oracle(d):
    Bseq, H, P, T = 3, 2, 300, 24
    (pq, pk, pv), (sq, sk, sv) = inputs.decode_batch(21, Bseq, H, d, P, T, True)
    pk, pv = inputs.round_bf16(pk), inputs.round_bf16(pv)
    sq, sk, sv = (inputs.round_bf16(x) for x in (sq, sk, sv))
    S_ref, z_ref = oracle.state(pk, pv)
    S = torch.from_numpy(S_ref.astype(np.float32)).cuda()
    z = torch.from_numpy(z_ref.astype(np.float32)).cuda()
    S_ref = S.double().cpu().numpy()
    z_ref = z.double().cpu().numpy()
    for t in range(T):
        out = la.decode_step(S, z, to_dev(sq[t], "bf16"), to_dev(sk[t], "bf16"),
                             to_dev(sv[t], "bf16"))
        S_ref, z_ref, ref = oracle.decode_step(S_ref, z_ref, sq[t], sk[t], sv[t])
        assert max_row_rel_err(to_host(out), ref) <= TOL["bf16"], t
    assert la.device_error() == la.LINATTN_OK
    assert _state_err(to_host(S), S_ref) <= 1e-5
    assert np.max(np.abs(to_host(z) - z_ref) / z_ref) <= 1e-5


@pytest.mark.parametrize("d", [64, 128])
def test_decode_replay_equals_causal_forward(d):
    B, H, n = 2, 2, 150
    q, k, v = inputs.forward_qkv(31, B, H, n, d, scaled=True)
    q, k, v = (inputs.round_bf16(x) for x in (q, k, v))
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    fwd = to_host(la.forward(qd, kd, vd, True))
    S = torch.zeros((B, H, d, d), dtype=torch.float32, device="cuda")
    z = torch.zeros((B, H, d), dtype=torch.float32, device="cuda")
    outs = []
    for t in range(n):
        outs.append(to_host(la.decode_step(S, z, qd[:, :, t].contiguous(),
                                           kd[:, :, t].contiguous(), vd[:, :, t].contiguous())))
    rep = np.stack(outs, axis=2)
    ref = oracle.forward(q, k, v, True)
    assert max_row_rel_err(rep, ref) <= TOL["bf16"]
    assert max_row_rel_err(rep, fwd) <= 2 * TOL["bf16"]
    # the state left by the replay is the forward_state of the same tokens (the bf16
    # forward_state rounds phi(k) to bf16 for the tensor cores: STATE_TOL_BF16)
    S2, z2 = la.forward_state(kd, vd)
    assert _state_err(to_host(S), to_host(S2)) <= STATE_TOL_BF16


def test_workload_decode_256x32x128():
    """256 sequences x 32 heads, d = 128, prefill 2048 tokens then 512 steps, as benchmarked;
    the oracle follows 24 sampled (sequence, head) pairs through every step."""
    from linear_attention_linattn_b200 import workloads
    w = inputs.WORKLOADS["decode_256x32x128"]
    Bseq, H, d, P, T = w.B, w.H, w.d, w.n, w.steps
    pairs = [(0, 0), (5, 31), (100, 7), (255, 31), (128, 16), (17, 3)]
    pairs += [(int(s), int(h)) for s, h in zip(np.random.default_rng(3).integers(0, Bseq, 18),
                                               np.random.default_rng(4).integers(0, H, 18))]
    pairs = sorted(set(pairs))
    S, z, qs, ks, vs = workloads.decode_inputs("decode_256x32x128")
    idx_s = [s for s, _ in pairs]
    idx_h = [h for _, h in pairs]
    outs = torch.empty((T, len(pairs), d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((Bseq, H, d), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        la.decode_step(S, z, qs[t], ks[t], vs[t], out=out)
        outs[t] = out[idx_s, idx_h]
    assert la.device_error() == la.LINATTN_OK
    (_, pk, pv), (sq, sk, sv) = inputs.decode_batch(w.seed, Bseq, H, d, P, T, w.scaled,
                                                    pairs=pairs)
    S_ref, z_ref = oracle.state(inputs.round_bf16(pk), inputs.round_bf16(pv))
    sq, sk, sv = (inputs.round_bf16(x) for x in (sq, sk, sv))
    ref = np.empty((T, len(pairs), d))
    for t in range(T):
        S_ref, z_ref, ref[t] = oracle.decode_step(S_ref, z_ref, sq[t], sk[t], sv[t])
    assert max_row_rel_err(to_host(outs), ref) <= TOL["bf16"]
    # the starting state came from the bf16 tensor-core prefill
    assert _state_err(to_host(S[idx_s, idx_h]), S_ref) <= STATE_TOL_BF16
