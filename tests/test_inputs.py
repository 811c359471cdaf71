"""The seeded generator is deterministic, per head, and independent of how it is sliced."""
import numpy as np

from linear_attention_linattn_b200 import inputs


def test_forward_inputs_deterministic_and_sliceable():
    q, k, v = inputs.forward_qkv(2, 2, 3, 40, 8, True)
    q2, k2, v2 = inputs.forward_qkv(2, 2, 3, 40, 8, True)
    assert np.array_equal(q, q2) and np.array_equal(k, k2) and np.array_equal(v, v2)
    qs, ks, vs = inputs.forward_qkv(2, 2, 3, 40, 8, True, heads=[(1, 2), (0, 1)])
    assert np.array_equal(qs[0], q[1, 2]) and np.array_equal(vs[1], v[0, 1])
    assert not np.array_equal(q[0, 0], k[0, 0])
    # scaling by 1/sqrt(d) is the only difference between the two recipes
    qu, _, _ = inputs.forward_qkv(2, 2, 3, 40, 8, False)
    assert np.allclose(q, qu * np.float32(1 / np.sqrt(8)), rtol=0, atol=0)


def test_decode_inputs_layout():
    (pq, pk, pv), (sq, sk, sv) = inputs.decode_batch(4, 3, 2, 8, 16, 5, True)
    (a, b, c), (x, y, w) = inputs.decode_qkv(4, 2, 1, 8, 16, 5, True)
    assert np.array_equal(pk[2, 1], b) and np.array_equal(sv[:, 2, 1], w)
    (pq2, _, _), (sq2, _, _) = inputs.decode_batch(4, 3, 2, 8, 16, 5, True, pairs=[(2, 1)])
    assert np.array_equal(pq2[0], a) and np.array_equal(sq2[:, 0], x)


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 3.0e38], dtype=np.float32)
    r = inputs.round_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2**-6 and r[3] == -2.5
    assert inputs.bf16_bits(np.array([1.0], dtype=np.float32))[0] == 0x3F80
