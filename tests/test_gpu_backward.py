"""Parity of the CUDA backward pass (through the C ABI) with the float64 oracle's gradients.

Metric: per row, ||got_i - ref_i|| / max(||ref_i||, mean_i ||ref_i||), maximised over the rows
of dq, dk and dv.  The floor at the mean row norm is needed because some gradient rows
vanish exactly (causal: the first token's dq is zero, its output being v_0 whatever q_0 is),
where a plain per-row ratio would divide rounding by zero.

Bars: 1e-3 for float32 I/O, 2e-2 for bfloat16 I/O.  No bar is stated for gradients; this one
follows from their arithmetic.  dphi(q_i) = (S_i g_i - z_i (g_i . out_i)) / den_i (and dphi(k_j)
likewise) is a difference of two sums of up to n terms each, of the same size as the result,
so float32 rounding (2^-24 per operation, grown by the square root of the ~D * n/64 terms
the chunked sums accumulate) lands near 1e-4 at d = 128 and n = 1000 (measured 1.4e-4 for
dq); 1e-3 keeps a margin of several times that while still catching any wrong term, which
moves the gradients by O(1).  bfloat16 I/O rounds each gradient once to 8 bits (2^-9).
"""
import numpy as np
import pytest

import oracle
from linear_attention_linattn_b200 import inputs
from tests.helpers import as_io, to_dev, to_host

TOL = {"f32": 1e-3, "bf16": 2e-2}

torch = pytest.importorskip("torch")
la = pytest.importorskip("linear_attention_linattn_b200")

pytestmark = pytest.mark.gpu


def grad_err(got, ref) -> float:
    d = ref.shape[-1]
    g = np.asarray(got, np.float64).reshape(-1, d)
    r = np.asarray(ref, np.float64).reshape(-1, d)
    rn = np.linalg.norm(r, axis=1)
    floor = max(rn.mean(), 1e-30)
    return float(np.max(np.linalg.norm(g - r, axis=1) / np.maximum(rn, floor)))


def _check(B, H, n, d, causal, dtype, seed):
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(seed, B, H, n, d, scaled=True))
    g = as_io(inputs.forward_qkv(seed + 1000, B, H, n, d, scaled=True)[0], dtype)
    dq, dk, dv = la.backward(*(to_dev(x, dtype) for x in (q, k, v, g)), causal)
    assert la.device_error() == la.LINATTN_OK
    ref = oracle.backward(q, k, v, g, causal)
    errs = [grad_err(to_host(a), b) for a, b in zip((dq, dk, dv), ref)]
    assert max(errs) <= TOL[dtype], errs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,n", [(1, 2, 2), (2, 1, 63), (1, 2, 65), (1, 3, 200), (1, 1, 1000)])
def test_backward_small_shapes(dtype, causal, d, B, H, n):
    _check(B, H, n, d, causal, dtype, 300 + n)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("causal", [True, False])
def test_backward_longer_sequence(dtype, causal):
    _check(1, 2, 4096, 64, causal, dtype, 7)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("segment_len", [64, 128, 320, 1024])
def test_backward_bf16_segment_edges(causal, d, segment_len):
    """The bf16 backward walks segments (work items) chunk by chunk, forwards for dq and
    backwards for dk and dv, carrying [S | z] and [R | r] across chunks in TMEM and across
    segments through the scans: moving the segment edges, ragged n included, changes nothing
    beyond rounding."""
    B, H, n = 2, 3, 1000
    dtype = "bf16"
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(41, B, H, n, d, scaled=True))
    g = as_io(inputs.forward_qkv(42, B, H, n, d, scaled=True)[0], dtype)
    dq, dk, dv = la.backward(*(to_dev(x, dtype) for x in (q, k, v, g)), causal,
                             segment_len=segment_len)
    assert la.device_error() == la.LINATTN_OK
    ref = oracle.backward(q, k, v, g, causal)
    errs = [grad_err(to_host(a), b) for a, b in zip((dq, dk, dv), ref)]
    assert max(errs) <= TOL[dtype], errs


@pytest.mark.parametrize("causal", [True, False])
def test_backward_bf16_many_items_per_cta(causal):
    """More segments than CTA slots (each CTA walks several items, its loads running one chunk
    ahead across item boundaries), at the shape of the batched benchmark's heads (d = 64)."""
    B, H, n, d = 2, 16, 2048, 64
    dtype = "bf16"
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(43, B, H, n, d, scaled=True))
    g = as_io(inputs.forward_qkv(44, B, H, n, d, scaled=True)[0], dtype)
    dq, dk, dv = la.backward(*(to_dev(x, dtype) for x in (q, k, v, g)), causal, segment_len=64)
    assert la.device_error() == la.LINATTN_OK
    ref = oracle.backward(q, k, v, g, causal)
    errs = [grad_err(to_host(a), b) for a, b in zip((dq, dk, dv), ref)]
    assert max(errs) <= TOL[dtype], errs


def test_backward_bf16_unaligned_outputs():
    """Buffers only 16-byte aligned (the interface's promise): the gradient rows are written
    with 16-byte stores there."""
    B, H, n, d = 1, 2, 300, 64
    dtype = "bf16"
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(45, B, H, n, d, scaled=True))
    g = as_io(inputs.forward_qkv(46, B, H, n, d, scaled=True)[0], dtype)
    qd, kd, vd, gd = (to_dev(x, dtype) for x in (q, k, v, g))
    numel = B * H * n * d
    bufs = [torch.full((numel + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
            for _ in range(3)]
    outs = [b_[8:].view(B, H, n, d) for b_ in bufs]
    assert all(o.data_ptr() % 32 == 16 for o in outs)
    lib = la.load_library()
    st = lib.linattn_backward(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), gd.data_ptr(),
                              outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), B, H,
                              n, d, 1, la.LINATTN_BF16, torch.cuda.current_stream().cuda_stream)
    assert st == la.LINATTN_OK
    assert la.device_error() == la.LINATTN_OK
    ref = oracle.backward(q, k, v, g, True)
    errs = [grad_err(to_host(a), b) for a, b in zip(outs, ref)]
    assert max(errs) <= TOL[dtype], errs
    assert all(torch.isnan(b_[:8].float()).all() for b_ in bufs)


def test_value_gradients_sum_to_output_gradients_on_gpu():
    """sum_j dL/dv_j = sum_i dL/dout_i: each output row is a convex combination of values."""
    B, H, n, d = 2, 2, 700, 64
    q, k, v = (to_dev(x, "f32") for x in inputs.forward_qkv(9, B, H, n, d, scaled=True))
    g = to_dev(inputs.forward_qkv(10, B, H, n, d, scaled=True)[0], "f32")
    for causal in (True, False):
        _, _, dv = la.backward(q, k, v, g, causal)
        assert torch.allclose(dv.double().sum(2), g.double().sum(2), rtol=1e-4, atol=1e-4)
