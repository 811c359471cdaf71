"""Parity of the CUDA forward pass (through the C ABI) with the float64 oracle.

Small cases span several chunks and segments with ragged tails; the five measured
workloads run at full size in the launch configuration the benchmark times, compared
on sampled heads and rows that the oracle computes one by one.
"""
import numpy as np
import pytest

import oracle
from linear_attention_linattn_b200 import inputs
from tests.helpers import STATE_TOL_BF16, TOL, as_io, max_row_rel_err, to_dev, to_host

torch = pytest.importorskip("torch")
la = pytest.importorskip("linear_attention_linattn_b200")

pytestmark = pytest.mark.gpu


def _run(q, k, v, causal, dtype, segment_len=0):
    qd, kd, vd = to_dev(q, dtype), to_dev(k, dtype), to_dev(v, dtype)
    out = la.forward(qd, kd, vd, causal, segment_len=segment_len)
    assert la.device_error() == la.LINATTN_OK
    return to_host(out)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,n", [(1, 1, 1), (1, 2, 2), (2, 1, 63), (1, 3, 65), (2, 2, 200),
                                   (1, 1, 1000), (1, 2, 4097)])
def test_small_shapes(dtype, causal, d, B, H, n):
    q, k, v = inputs.forward_qkv(100 + n, B, H, n, d, scaled=True)
    q, k, v = as_io(q, dtype), as_io(k, dtype), as_io(v, dtype)
    got = _run(q, k, v, causal, dtype)
    ref = oracle.forward(q, k, v, causal)
    assert max_row_rel_err(got, ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("seg", [0, 128, 256, 512, 1024])
def test_segment_length_invariance(dtype, seg):
    B, H, n, d = 1, 2, 3000, 128
    q, k, v = inputs.forward_qkv(7, B, H, n, d, scaled=True)
    q, k, v = as_io(q, dtype), as_io(k, dtype), as_io(v, dtype)
    got = _run(q, k, v, True, dtype, segment_len=seg)
    ref = oracle.forward(q, k, v, True)
    assert max_row_rel_err(got, ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_invariants_on_device(dtype, d):
    rng = np.random.default_rng(5)
    B, H, n = 1, 2, 777
    q, k, v = (as_io(rng.standard_normal((B, H, n, d)).astype(np.float32) / np.sqrt(d), dtype)
               for _ in range(3))
    # constant values come back unchanged (the weights are a convex combination)
    c = as_io(rng.standard_normal(d).astype(np.float32), dtype)
    vc = np.broadcast_to(c, (B, H, n, d)).copy()
    for causal in (False, True):
        got = _run(q, k, vc, causal, dtype)
        assert max_row_rel_err(got, np.broadcast_to(c, got.shape)) <= TOL[dtype]
    # a single token returns its own value
    got1 = _run(q[:, :, :1], k[:, :, :1], v[:, :, :1], True, dtype)
    assert max_row_rel_err(got1, v[:, :, :1]) <= TOL[dtype]
    # the last causal row sees every key: it equals the non-causal row
    nc = _run(q, k, v, False, dtype)
    ca = _run(q, k, v, True, dtype)
    assert max_row_rel_err(ca[:, :, -1], nc[:, :, -1]) <= 2 * TOL[dtype]


def test_output_canary_untouched():
    """Nothing is written outside out: guard regions on both sides keep their pattern."""
    B, H, n, d = 1, 2, 130, 64
    q, k, v = inputs.forward_qkv(3, B, H, n, d, scaled=True)
    for dtype in ("f32", "bf16"):
        qd, kd, vd = to_dev(as_io(q, dtype), dtype), to_dev(as_io(k, dtype), dtype), \
            to_dev(as_io(v, dtype), dtype)
        pad = 4096
        buf = torch.full((2 * pad + qd.numel(),), 12345.0, dtype=qd.dtype, device="cuda")
        out = buf[pad:pad + qd.numel()].view(qd.shape)
        for causal in (False, True):
            la.forward(qd, kd, vd, causal, out=out)
            torch.cuda.synchronize()
            assert bool((buf[:pad] == 12345.0).all()) and bool((buf[-pad:] == 12345.0).all())


@pytest.mark.parametrize("causal", [False, True])
def test_outputs_only_16_byte_aligned(causal):
    """The interface promises 16-byte aligned buffers, not 32: an output that starts 16 bytes
    past a 32-byte boundary is written with 16-byte stores, and matches."""
    B, H, n, d = 2, 3, 700, 64
    q, k, v = (as_io(x, "bf16") for x in inputs.forward_qkv(21, B, H, n, d, scaled=True))
    qd, kd, vd = (to_dev(x, "bf16") for x in (q, k, v))
    buf = torch.full((qd.numel() + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[8:].view(qd.shape)
    assert out.data_ptr() % 32 == 16
    la.forward(qd, kd, vd, causal, out=out)
    assert la.device_error() == la.LINATTN_OK
    assert max_row_rel_err(to_host(out), oracle.forward(q, k, v, causal)) <= TOL["bf16"]
    assert bool(torch.isnan(buf[:8].float()).all())


def test_forward_state_matches_oracle():
    for dtype in ("f32", "bf16"):
        for d in (64, 128):
            B, H, n = 2, 2, 1500
            _, k, v = inputs.forward_qkv(11, B, H, n, d, scaled=True)
            k, v = as_io(k, dtype), as_io(v, dtype)
            S, z = la.forward_state(to_dev(k, dtype), to_dev(v, dtype))
            assert la.device_error() == la.LINATTN_OK
            S_ref, z_ref = oracle.state(k, v)
            S, z = to_host(S), to_host(z)
            tol = 1e-5 if dtype == "f32" else STATE_TOL_BF16
            for b in range(B):
                for h in range(H):
                    e = np.linalg.norm(S[b, h] - S_ref[b, h]) / np.linalg.norm(S_ref[b, h])
                    assert e <= tol, (dtype, d, e)
                    assert np.max(np.abs(z[b, h] - z_ref[b, h]) / z_ref[b, h]) <= tol


# ------------------------------------------------------------------ the measured workloads
def test_workload_noncausal_1x1x512x64_f32():
    w = inputs.WORKLOADS["noncausal_1x1x512x64_f32"]
    q, k, v = inputs.forward_qkv(w.seed, w.B, w.H, w.n, w.d, w.scaled)
    got = _run(q, k, v, False, "f32")
    assert max_row_rel_err(got, oracle.forward(q, k, v, False)) <= TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_workload_causal_1x1x4096x64(dtype):
    w = inputs.WORKLOADS["causal_1x1x4096x64"]
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(w.seed, w.B, w.H, w.n, w.d, w.scaled))
    got = _run(q, k, v, True, dtype)
    assert max_row_rel_err(got, oracle.forward(q, k, v, True)) <= TOL[dtype]


def _sample_rows(n, extra, seed, edge_step=0):
    """Chunk edges, powers of two, the last rows and random rows; with edge_step, both sides of
    every multiple of it (every segment edge the library can pick: its segments are multiples
    of 128 tokens, chosen from multiples of 256)."""
    rng = np.random.default_rng(seed)
    rows = {0, 1, 2, 63, 64, 65, 127, 128, 129, 255, 256, n // 2, n - 2, n - 1}
    rows |= {r for m in (512, 1024, 2048, 4096) for r in (m - 1, m) if r < n}
    if edge_step:
        rows |= {r for m in range(edge_step, n, edge_step) for r in (m - 1, m)}
    rows |= set(rng.integers(0, n, size=extra).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < n), dtype=np.int64)


@pytest.mark.parametrize("causal", [False, True])
def test_workload_batched_8x16x8192x64_bf16(causal):
    """Full size, as the benchmark runs it: every row of head (3, 7); on two more heads the
    rows on both sides of every multiple of 128 tokens (every chunk and segment edge)."""
    w = inputs.WORKLOADS["batched_8x16x8192x64_bf16"]
    q, k, v = inputs.forward_qkv(w.seed, w.B, w.H, w.n, w.d, w.scaled)
    q, k, v = (inputs.round_bf16(x) for x in (q, k, v))
    got = _run(q, k, v, causal, "bf16")
    assert np.all(np.isfinite(got))
    b, h = 3, 7
    whole = oracle.forward(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], causal)
    assert max_row_rel_err(got[b:b + 1, h:h + 1], whole) <= TOL["bf16"]
    heads = [(0, 0), (7, 15)]
    rows = _sample_rows(w.n, 64, 1, edge_step=128)
    qs = np.stack([q[b, h] for b, h in heads])
    ks = np.stack([k[b, h] for b, h in heads])
    vs = np.stack([v[b, h] for b, h in heads])
    ref = oracle.forward_rows(qs, ks, vs, rows, causal)
    gs = np.stack([got[b, h][rows] for b, h in heads])
    assert max_row_rel_err(gs, ref) <= TOL["bf16"]


def test_workload_longctx_1x32x131072x128_bf16():
    """Full size, as the benchmark runs it: every row of head 17; on heads 0 and 31 the rows on
    both sides of every multiple of 256 tokens (every segment edge) plus random rows."""
    w = inputs.WORKLOADS["longctx_1x32x131072x128_bf16"]
    q, k, v = inputs.forward_qkv(w.seed, w.B, w.H, w.n, w.d, w.scaled)
    q, k, v = (inputs.round_bf16(x) for x in (q, k, v))
    got = _run(q, k, v, True, "bf16")
    assert np.all(np.isfinite(got))
    h = 17
    whole = oracle.forward(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], True)
    assert max_row_rel_err(got[:, h:h + 1], whole) <= TOL["bf16"]
    heads = [0, 31]
    rows = _sample_rows(w.n, 48, 2, edge_step=256)
    ref = oracle.forward_rows(q[0, heads], k[0, heads], v[0, heads], rows, True)
    gs = np.stack([got[0, h][rows] for h in heads])
    assert max_row_rel_err(gs, ref) <= TOL["bf16"]


# ------------------------------------------------------------------ persistent work items
# The tensor-core kernels walk a list of (head, segment) items per CTA (one per SM); these
# cases put several items of different lengths on each CTA, and ragged final segments.
def _sampled_parity(q, k, v, causal, segment_len, heads_to_check, seed):
    got = _run(q, k, v, causal, "bf16", segment_len=segment_len)
    assert np.all(np.isfinite(got))
    B, H, n, d = q.shape
    rows = _sample_rows(n, 24, seed)
    qs = np.stack([q[b, h] for b, h in heads_to_check])
    ks = np.stack([k[b, h] for b, h in heads_to_check])
    vs = np.stack([v[b, h] for b, h in heads_to_check])
    ref = oracle.forward_rows(qs, ks, vs, rows, causal)
    gs = np.stack([got[b, h][rows] for b, h in heads_to_check])
    assert max_row_rel_err(gs, ref) <= TOL["bf16"]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_persistent_many_heads_ragged_items(causal, d):
    """400 heads of 200 tokens: more items than SMs, each ending in a partial chunk."""
    B, H, n = 4, 100, 200
    q, k, v = (inputs.round_bf16(x) for x in inputs.forward_qkv(21, B, H, n, d, scaled=True))
    _sampled_parity(q, k, v, causal, 0, [(0, 0), (1, 37), (2, 63), (3, 99)], 3)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("seg", [256, 2304])
def test_persistent_segments_of_unequal_length(causal, seg):
    """160 heads split into segments whose last one is shorter (n = 4500): the items of one
    CTA differ in length.  seg = 256 runs the causal items on persistent CTAs (4 chunks
    each), seg = 2304 runs them one CTA per item (36 chunks)."""
    B, H, n, d = 2, 80, 4500, 64
    q, k, v = (inputs.round_bf16(x) for x in inputs.forward_qkv(22, B, H, n, d, scaled=True))
    _sampled_parity(q, k, v, causal, seg, [(0, 0), (0, 79), (1, 5), (1, 79)], 4)


@pytest.mark.parametrize("causal", [False, True])
def test_fewer_items_than_sms(causal):
    """3 heads x 2 segments: a grid of 6 CTAs, one item each."""
    B, H, n, d = 1, 3, 700, 128
    q, k, v = (inputs.round_bf16(x) for x in inputs.forward_qkv(23, B, H, n, d, scaled=True))
    got = _run(q, k, v, causal, "bf16", segment_len=384)
    assert max_row_rel_err(got, oracle.forward(q, k, v, causal)) <= TOL["bf16"]


# Host buffers in, host buffers out: the library copies head groups in, runs them and copies
# them back on its own streams.  24 heads make 8 groups of 3 on 3 streams (each stream's
# buffers reused), 5 heads make 5 groups of 1.
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,n,d,pinned", [(2, 12, 777, 128, True), (1, 5, 1000, 64, False),
                                             (1, 1, 5, 64, True)])
def test_forward_host_buffers(dtype, causal, B, H, n, d, pinned):
    q, k, v = inputs.forward_qkv(31 + n, B, H, n, d, scaled=True)
    q, k, v = as_io(q, dtype), as_io(k, dtype), as_io(v, dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    qh, kh, vh = (torch.from_numpy(x.astype(np.float32)).to(tdt).contiguous() for x in (q, k, v))
    if pinned:
        qh, kh, vh = qh.pin_memory(), kh.pin_memory(), vh.pin_memory()
    out = la.forward_host(qh, kh, vh, causal)
    assert la.device_error() == la.LINATTN_OK
    assert not out.is_cuda and out.is_pinned() == pinned
    got = out.float().numpy()
    ref = oracle.forward(q, k, v, causal)
    assert max_row_rel_err(got, ref) <= TOL[dtype]
    # the same result as the device entry point (up to the segment lengths its head count picks)
    dev = _run(q, k, v, causal, dtype)
    assert max_row_rel_err(got, dev) <= TOL[dtype]


def test_forward_host_rejects_device_tensors():
    q = torch.zeros((1, 1, 64, 64), device="cuda")
    with pytest.raises(ValueError):
        la.forward_host(q, q, q, True)


def test_forward_host_calls_on_two_streams():
    """Two calls enqueued back to back on different streams share the library's group streams;
    each result is its own."""
    outs, refs = [], []
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for seed, st in ((41, s1), (42, s2)):
        q, k, v = inputs.forward_qkv(seed, 1, 6, 700, 64, scaled=True)
        q, k, v = as_io(q, "bf16"), as_io(k, "bf16"), as_io(v, "bf16")
        qh, kh, vh = (torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).pin_memory()
                      for x in (q, k, v))
        out = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
        st_ = la.load_library().linattn_forward_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(),
                                                     out.data_ptr(), 1, 6, 700, 64, 1,
                                                     la.LINATTN_BF16, st.cuda_stream)
        assert st_ == la.LINATTN_OK
        outs.append((out, qh, kh, vh))
        refs.append(oracle.forward(q, k, v, True))
    s1.synchronize()
    s2.synchronize()
    assert la.device_error() == la.LINATTN_OK
    for (out, *_), ref in zip(outs, refs):
        assert max_row_rel_err(out.float().numpy(), ref) <= TOL["bf16"]

