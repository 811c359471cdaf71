"""FAVOR+ on the GPU against the oracle: the positive random features, the forward pass on
given features, and the two together.

Bars: features 1e-5 per row (float32 I/O; they are intermediates, so tighter than the
outputs' bar) and 2e-2 (bfloat16 I/O, one rounding to 8 bits); outputs at the forward's bars,
1e-4 (float32) and 2e-2 (bfloat16).  W [m, d] has i.i.d. N(0, 1) entries (the caller's random
draw, seeded here); m = d and, for bf16 I/O, m != d (the tensor-core kernels keep the feature
and value dimensions apart).
"""
import numpy as np
import pytest

import oracle
from linear_attention_linattn_b200 import inputs
from tests.helpers import TOL, as_io, max_row_rel_err, to_dev, to_host

torch = pytest.importorskip("torch")
la = pytest.importorskip("linear_attention_linattn_b200")

pytestmark = pytest.mark.gpu

FEATURE_TOL = {"f32": 1e-5, "bf16": 2e-2}


def _W(m, d, seed):
    return np.random.default_rng(seed).standard_normal((m, d)).astype(np.float32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d,m", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_favor_features_match_oracle(dtype, d, m):
    x = as_io(inputs.forward_qkv(51, 1, 3, 333, d, scaled=True)[0], dtype)  # 999 rows, ragged
    W = _W(m, d, 1)
    got = to_host(la.favor_features(to_dev(x, dtype), torch.from_numpy(W).cuda()))
    assert la.device_error() == la.LINATTN_OK
    ref = oracle.favor_features(x, W)
    assert max_row_rel_err(got, ref) <= FEATURE_TOL[dtype]


@pytest.mark.parametrize("dtype,d,m", [("f32", 64, 64), ("f32", 128, 128), ("bf16", 64, 64),
                                       ("bf16", 128, 128), ("bf16", 64, 128), ("bf16", 128, 64)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,n", [(1, 2, 65), (2, 1, 200), (1, 1, 1000), (2, 3, 2500)])
def test_forward_on_given_features(dtype, causal, d, m, B, H, n):
    """The pass with no feature map of its own, on oracle features (m of them) rounded to the
    I/O type, with d-dimensional values."""
    q, k, v = inputs.forward_qkv(52 + n, B, H, n, d, scaled=True)
    W = _W(m, d, 2)
    fq, fk = (as_io(oracle.favor_features(x, W).astype(np.float32), dtype) for x in (q, k))
    v = as_io(v, dtype)
    got = to_host(la.forward_features(to_dev(fq, dtype), to_dev(fk, dtype), to_dev(v, dtype),
                                      causal))
    assert la.device_error() == la.LINATTN_OK
    ref = oracle.forward(fq, fk, v, causal, phi_kind=oracle.PHI_IDENTITY)
    assert max_row_rel_err(got, ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,m", [("f32", 64), ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_favor_attention_end_to_end(dtype, m, causal):
    B, H, n, d = 1, 2, 700, 64
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(53, B, H, n, d, scaled=True))
    W = _W(m, d, 3)
    got = to_host(la.forward_favor(to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype),
                                   torch.from_numpy(W).cuda(), causal))
    assert la.device_error() == la.LINATTN_OK
    ref = oracle.forward(oracle.favor_features(q, W), oracle.favor_features(k, W), v, causal,
                         phi_kind=oracle.PHI_IDENTITY)
    assert max_row_rel_err(got, ref) <= TOL[dtype]


def test_fp32_features_of_another_size_are_unsupported():
    """The fp32 (CUDA-core) pass keeps m = d; m != d needs bf16 I/O."""
    lib = la.load_library()
    fq = torch.ones((1, 1, 64, 128), device="cuda")
    v = torch.ones((1, 1, 64, 64), device="cuda")
    out = torch.empty_like(v)
    st = lib.linattn_forward_features(fq.data_ptr(), fq.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      1, 1, 64, 128, 64, 1, la.LINATTN_F32, None)
    assert st == la.LINATTN_ERR_UNSUPPORTED
