"""linattn for B200: linear attention (phi = elu + 1) as hand-written sm_100a CUDA kernels.

The compute path is the C-ABI library ``liblinattn.so`` built from ``csrc/`` (declared in
``include/linattn.h``).  This module only marshals arguments: it passes device pointers,
sizes and the current CUDA stream of PyTorch tensors to the C entry points of the same
names.  There is no fallback: if the library is missing or fails to load, every call
raises.

Raw C entry points (pointers as ints):
    linattn_forward, linattn_forward_ex, linattn_forward_state, linattn_decode_step,
    linattn_state_bytes, linattn_status_string, linattn_device_error, linattn_version,
    linattn_launch_count, linattn_forward_noalloc, linattn_profile_events,
    linattn_forward_init, linattn_sum_states, linattn_backward, linattn_favor_features,
    linattn_forward_features, linattn_selftest_wait_timeout,
    linattn_selftest_noalloc_wait_timeout

Tensor helpers: ``forward``, ``forward_init``, ``forward_state``, ``sum_states``,
``backward``, ``favor_features``, ``forward_features``, ``forward_favor``, ``decode_step``,
``device_error``; ``seqshard`` splits one sequence over ranks.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblinattn.so")

LINATTN_OK = 0
LINATTN_ERR_INVALID_ARG = 1
LINATTN_ERR_UNSUPPORTED = 2
LINATTN_ERR_CUDA = 3
LINATTN_ERR_TIMEOUT = 4
LINATTN_F32 = 0
LINATTN_BF16 = 1

# Every symbol include/linattn.h declares, with its ctypes signature.
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
SIGNATURES = {
    "linattn_forward": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.c_int,
                                       ctypes.c_int, _vp]),
    "linattn_forward_ex": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                          ctypes.c_int, ctypes.c_int, _i64, _vp]),
    "linattn_forward_host": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                            ctypes.c_int, ctypes.c_int, _vp]),
    "linattn_forward_state": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                             ctypes.c_int, _vp]),
    "linattn_decode_step": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "linattn_state_bytes": (ctypes.c_size_t, [_i64]),
    "linattn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "linattn_device_error": (ctypes.c_int, [_vp]),
    "linattn_version": (ctypes.c_int, []),
    "linattn_launch_count": (ctypes.c_uint64, []),
    "linattn_forward_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                               ctypes.c_int, ctypes.c_int, _vp]),
    "linattn_profile_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]),
    "linattn_forward_init": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                            _i64, ctypes.c_int, ctypes.c_int, _vp]),
    "linattn_sum_states": (ctypes.c_int, [_vp, _i64, _i64, _i64, _i64, _i64, _vp, _vp, _vp]),
    "linattn_backward": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                        _i64, ctypes.c_int, ctypes.c_int, _vp]),
    "linattn_backward_ex": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                           _i64, _i64, ctypes.c_int, ctypes.c_int, _i64, _vp]),
    "linattn_block_aggregates_bytes": (ctypes.c_size_t, [_i64, _i64, _i64, _i64, ctypes.c_int]),
    "linattn_forward_state_keep": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                                  _i64, ctypes.c_int, _vp]),
    "linattn_forward_init_from": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                                 _i64, _i64, ctypes.c_int, ctypes.c_int, _vp]),
    "linattn_favor_features": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int,
                                              _vp]),
    "linattn_selftest_wait_timeout": (ctypes.c_int, [_vp]),
    "linattn_selftest_noalloc_wait_timeout": (ctypes.c_int, [_vp]),
    "linattn_forward_features": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                                _i64, ctypes.c_int, ctypes.c_int, _vp]),
}

_lib = None


class LinattnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Loads liblinattn.so (raises if it is missing: build it with
    ``python -m linear_attention_linattn_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"liblinattn.so not found at {p}; build it with "
                           "`python -m linear_attention_linattn_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().linattn_status_string(int(status)).decode()


def __getattr__(name):  # raw C entry points: linear_attention_linattn_b200.linattn_forward(...)
    if name in SIGNATURES:
        return getattr(load_library(), name)
    raise AttributeError(name)


# ------------------------------------------------------------------ tensor helpers
def _stream_ptr(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return LINATTN_F32
    if t.dtype == torch.bfloat16:
        return LINATTN_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _check(status: int, what: str):
    if status != LINATTN_OK:
        raise LinattnError(status, what)


def _dev(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def forward(q, k, v, causal: bool, out=None, segment_len: int = 0, stream=None):
    """q, k, v: [B, H, n, d] CUDA tensors (float32 or bfloat16).  Returns out (same shape)."""
    import torch
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, nm)
    if not (q.shape == k.shape == v.shape and q.dim() == 4 and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share one [B, H, n, d] shape and dtype")
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out")
    B, H, n, d = q.shape
    lib = load_library()
    st = lib.linattn_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                B, H, n, d, int(bool(causal)), _dtype_code(q), int(segment_len),
                                _stream_ptr(stream))
    _check(st, "linattn_forward")
    return out


def forward_host(q, k, v, causal: bool, out=None, stream=None):
    """forward on host tensors: q, k, v [B, H, n, d] contiguous CPU tensors (float32 or
    bfloat16; pinned ones let the library overlap the copies with the work).  The library
    copies head groups in, runs them and copies the outputs back on its own streams; this
    waits for `stream` (default: the current CUDA stream) before returning out, a CPU tensor
    (pinned when q is)."""
    import torch
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous CPU tensor")
    if not (q.shape == k.shape == v.shape and q.dim() == 4 and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share one [B, H, n, d] shape and dtype")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=q.is_pinned())
    if out.is_cuda or not out.is_contiguous() or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must be a contiguous CPU tensor of q's shape and dtype")
    B, H, n, d = q.shape
    s = stream if stream is not None else torch.cuda.current_stream()
    st = load_library().linattn_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                             out.data_ptr(), B, H, n, d, int(bool(causal)),
                                             _dtype_code(q), int(s.cuda_stream))
    _check(st, "linattn_forward_host")
    s.synchronize()
    return out


def forward_init(q, k, v, S0, z0, causal: bool, out=None, aggregates=None, stream=None):
    """forward continued from a state: S0 [B, H, d, d] and z0 [B, H, d] (float32) hold what
    the tokens before this block (causal) or the rest of the sequence (non-causal)
    contribute.  aggregates: the buffer forward_state(k, v, keep=True) returned for the same
    k, v (its sums are reused instead of recomputed, and the buffer is overwritten)."""
    import torch
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (S0, "S0"), (z0, "z0")):
        _dev(t, nm)
    if not (q.shape == k.shape == v.shape and q.dim() == 4 and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share one [B, H, n, d] shape and dtype")
    B, H, n, d = q.shape
    if S0.dtype != torch.float32 or z0.dtype != torch.float32 or \
            tuple(S0.shape) != (B, H, d, d) or tuple(z0.shape) != (B, H, d):
        raise ValueError("S0 must be float32 [B, H, d, d] and z0 float32 [B, H, d]")
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out")
    lib = load_library()
    if aggregates is not None:
        _dev(aggregates, "aggregates")
        if aggregates.numel() * aggregates.element_size() < lib.linattn_block_aggregates_bytes(
                B, H, n, d, _dtype_code(q)):
            raise ValueError("aggregates is smaller than this block's aggregates")
        st = lib.linattn_forward_init_from(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           out.data_ptr(), S0.data_ptr(), z0.data_ptr(),
                                           aggregates.data_ptr(), B, H, n, d, int(bool(causal)),
                                           _dtype_code(q), _stream_ptr(stream))
        _check(st, "linattn_forward_init_from")
        return out
    st = lib.linattn_forward_init(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  S0.data_ptr(), z0.data_ptr(), B, H, n, d, int(bool(causal)),
                                  _dtype_code(q), _stream_ptr(stream))
    _check(st, "linattn_forward_init")
    return out


def sum_states(states, count: int, skip: int = -1, S=None, z=None, stream=None):
    """states: float32 [G, B, H, d*d + d] (S row-major then z, per head).  Returns the sum of
    states[i] over i < count, i != skip, as S [B, H, d, d] and z [B, H, d]."""
    import torch
    _dev(states, "states")
    G, B, H, per = states.shape
    d = int(round((-1 + (1 + 4 * per) ** 0.5) / 2))
    if d * d + d != per or states.dtype != torch.float32 or not 0 <= count <= G:
        raise ValueError("states must be float32 [G, B, H, d*d + d] and 0 <= count <= G")
    if S is None:
        S = torch.empty((B, H, d, d), dtype=torch.float32, device=states.device)
    if z is None:
        z = torch.empty((B, H, d), dtype=torch.float32, device=states.device)
    lib = load_library()
    st = lib.linattn_sum_states(states.data_ptr(), int(count), int(skip), B, H, d, S.data_ptr(),
                                z.data_ptr(), _stream_ptr(stream))
    _check(st, "linattn_sum_states")
    return S, z


def favor_features(x, W, out=None, stream=None):
    """FAVOR+ positive random features exp(W x - |x|^2/2) / sqrt(m) of x [..., d] (float32 or
    bfloat16 CUDA tensor); W: float32 [m, d] CUDA tensor of m random rows.  Returns [..., m]."""
    import torch
    _dev(x, "x")
    _dev(W, "W")
    d = x.shape[-1]
    if W.dtype != torch.float32 or W.dim() != 2 or W.shape[1] != d:
        raise ValueError("W must be a float32 [m, d] tensor")
    m = W.shape[0]
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (m,), dtype=x.dtype, device=x.device)
    _dev(out, "out")
    lib = load_library()
    st = lib.linattn_favor_features(x.data_ptr(), W.contiguous().data_ptr(), out.data_ptr(),
                                    x.numel() // d, d, m, _dtype_code(x), _stream_ptr(stream))
    _check(st, "linattn_favor_features")
    return out


def forward_features(phi_q, phi_k, v, causal: bool, out=None, stream=None):
    """forward with caller-computed non-negative features phi_q, phi_k [B, H, n, m] and
    values v [B, H, n, d]; returns [B, H, n, d]."""
    import torch
    for t, nm in ((phi_q, "phi_q"), (phi_k, "phi_k"), (v, "v")):
        _dev(t, nm)
    if not (phi_q.shape == phi_k.shape and v.dim() == 4 and phi_q.shape[:3] == v.shape[:3] and
            phi_q.dtype == phi_k.dtype == v.dtype):
        raise ValueError("phi_q, phi_k must share one [B, H, n, m] shape, v be [B, H, n, d], "
                         "all of one dtype")
    if out is None:
        out = torch.empty_like(v)
    _dev(out, "out")
    B, H, n, d = v.shape
    m = phi_q.shape[-1]
    lib = load_library()
    st = lib.linattn_forward_features(phi_q.data_ptr(), phi_k.data_ptr(), v.data_ptr(),
                                      out.data_ptr(), B, H, n, m, d, int(bool(causal)),
                                      _dtype_code(v), _stream_ptr(stream))
    _check(st, "linattn_forward_features")
    return out


def forward_favor(q, k, v, W, causal: bool, stream=None):
    """FAVOR+ linear attention: the forward pass on favor_features(q, W), favor_features(k, W)
    (m = W.shape[0] random features)."""
    return forward_features(favor_features(q, W, stream=stream), favor_features(k, W, stream=stream),
                            v, causal, stream=stream)


def backward(q, k, v, dout, causal: bool, segment_len: int = 0, stream=None):
    """Gradients (dq, dk, dv) of a loss given dout = dL/dout for out = forward(q, k, v, causal);
    all [B, H, n, d] CUDA tensors of one dtype (float32 or bfloat16).  segment_len (bf16, a
    multiple of 64; 0 = default) sets the tokens of one work item."""
    import torch
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _dev(t, nm)
    if not (q.shape == k.shape == v.shape == dout.shape and q.dim() == 4 and
            q.dtype == k.dtype == v.dtype == dout.dtype):
        raise ValueError("q, k, v, dout must share one [B, H, n, d] shape and dtype")
    B, H, n, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    lib = load_library()
    st = lib.linattn_backward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                 dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, n, d,
                                 int(bool(causal)), _dtype_code(q), int(segment_len),
                                 _stream_ptr(stream))
    _check(st, "linattn_backward")
    return dq, dk, dv


def forward_state(k, v, S=None, z=None, keep: bool = False, stream=None):
    """Final causal state of k, v [B, H, n, d]: S [B, H, d, d] and z [B, H, d] (float32).
    keep=True also returns the block's aggregates (a float32 device buffer) for
    forward_init(..., aggregates=...), which then skips summing k, v again."""
    import torch
    _dev(k, "k")
    _dev(v, "v")
    B, H, n, d = k.shape
    if S is None:
        S = torch.empty((B, H, d, d), dtype=torch.float32, device=k.device)
    if z is None:
        z = torch.empty((B, H, d), dtype=torch.float32, device=k.device)
    lib = load_library()
    if keep:
        nbytes = lib.linattn_block_aggregates_bytes(B, H, n, d, _dtype_code(k))
        if nbytes == 0:
            raise ValueError("unsupported shape or dtype for the block's aggregates")
        agg = torch.empty((nbytes + 3) // 4, dtype=torch.float32, device=k.device)
        st = lib.linattn_forward_state_keep(k.data_ptr(), v.data_ptr(), S.data_ptr(),
                                            z.data_ptr(), agg.data_ptr(), B, H, n, d,
                                            _dtype_code(k), _stream_ptr(stream))
        _check(st, "linattn_forward_state_keep")
        return S, z, agg
    st = lib.linattn_forward_state(k.data_ptr(), v.data_ptr(), S.data_ptr(), z.data_ptr(),
                                   B, H, n, d, _dtype_code(k), _stream_ptr(stream))
    _check(st, "linattn_forward_state")
    return S, z


def decode_step(S, z, q, k, v, out=None, stream=None):
    """One step in place on S [Bseq, H, d, d], z [Bseq, H, d] (float32) with bf16 q, k, v
    [Bseq, H, d].  Returns out [Bseq, H, d] (bfloat16)."""
    import torch
    for t, nm in ((S, "S"), (z, "z"), (q, "q"), (k, "k"), (v, "v")):
        _dev(t, nm)
    if S.dtype != torch.float32 or z.dtype != torch.float32:
        raise TypeError("the decode state is float32")
    if not (q.dtype == k.dtype == v.dtype == torch.bfloat16):
        raise TypeError("decode q, k, v are bfloat16")
    Bseq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    lib = load_library()
    st = lib.linattn_decode_step(S.data_ptr(), z.data_ptr(), q.data_ptr(), k.data_ptr(),
                                 v.data_ptr(), out.data_ptr(), Bseq, H, d, _stream_ptr(stream))
    _check(st, "linattn_decode_step")
    return out


def device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the kernels' error status."""
    return load_library().linattn_device_error(_stream_ptr(stream))
