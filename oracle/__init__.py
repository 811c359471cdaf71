"""Float64 CPU oracle for linear attention (phi = elu + 1).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
The CUDA library never imports, links or calls it, and it imports nothing from the
library: the only code both sides share is the seeded input generator
``linear_attention_linattn_b200.inputs``, which holds none of the method's arithmetic.

Contents
--------
* ``backward``: gradients of sum(g * out) with respect to q, k, v, by the chain rule
  through the forward's definition as weights w_ij = phi(q_i).phi(k_j) (the pages give
  no backward formulas; this is plain differentiation of the forward they define).
* ``favor_features``: Performer's positive random features exp(W x - |x|^2/2)/sqrt(m), whose
  dot products approximate exp(q . k) (named on the same page); with them ``forward(...,
  phi_kind=PHI_IDENTITY)`` is FAVOR+ linear attention.
* ``forward`` / ``forward_rows`` / ``state`` / ``decode_step``: ctypes wrappers around
  ``oracle.c`` (plain float64 loops, OpenMP over heads).  The method follows the page
  "Efficient Transformers: Linear Attention and Flash Attention", section "Linear
  attention: reordering the matmuls, not shrinking them" (the kernelised formula) and
  its section "The recurrent view: attention as an RNN" (causal state, inclusive of
  the current token).
* ``brute_force``: the quadratic form written out in numpy: form W = phi(Q) phi(K)^T,
  mask it causally (j <= i), divide each row by its sum, multiply by V.  It is the
  left-hand side of the associativity law that the same page states, so agreeing with
  it pins the linear-order oracle independently.
* Closed forms from the pages: ``memory_linear_attention`` / ``memory_standard_attention``
  (page "Linear Attention > Memory Efficiency") and ``flops_linear_attention`` /
  ``flops_standard_attention`` (page "Linear Attention > Computational Complexity
  Analysis").

Parity pins for every function are in ``tests/test_oracle_pins.py``; none is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

PHI_ELU1 = 0
PHI_IDENTITY = 1

_i64 = ctypes.c_int64
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)


def build(plant: int = 0, out_path: str | None = None) -> str:
    """Compile oracle.c with gcc (-O2, OpenMP).  ``plant`` != 0 builds a variant with a
    deliberate mistake (only the mutation test uses that)."""
    path = out_path or _LIB_PATH
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
           f"-DORACLE_PLANT={int(plant)}", _SRC, "-o", path, "-lm"]
    subprocess.run(cmd, check=True)
    return path


def _needs_build() -> bool:
    return (not os.path.exists(_LIB_PATH)
            or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))


class Oracle:
    """One loaded copy of the oracle library (the default build, or a planted one)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.oracle_phi.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.oracle_phi.restype = ctypes.c_double
        lib.oracle_forward_f64.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                           ctypes.c_int, ctypes.c_int]
        lib.oracle_forward_f64.restype = None
        lib.oracle_forward_dkv_f64.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                               ctypes.c_int, ctypes.c_int]
        lib.oracle_forward_dkv_f64.restype = None
        lib.oracle_forward_rows_f64.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64,
                                                ctypes.c_int, _ip, _i64, ctypes.c_int]
        lib.oracle_forward_rows_f64.restype = None
        lib.oracle_state_f64.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, ctypes.c_int]
        lib.oracle_state_f64.restype = None
        lib.oracle_decode_step_f64.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64,
                                               ctypes.c_int]
        lib.oracle_decode_step_f64.restype = None
        lib.oracle_backward_f64.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _i64, _i64,
                                            _i64, _i64, ctypes.c_int, ctypes.c_int]
        lib.oracle_backward_f64.restype = None
        lib.oracle_favor_features_f64.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64]
        lib.oracle_favor_features_f64.restype = None
        lib.oracle_plant.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = None
        lib.oracle_get_threads.restype = ctypes.c_int
        self.lib = lib
        self.plant = lib.oracle_plant()

    @staticmethod
    def _f64(a) -> np.ndarray:
        return np.ascontiguousarray(np.asarray(a, dtype=np.float64))

    @staticmethod
    def _ptr(a: np.ndarray):
        return a.ctypes.data_as(_dp)

    def phi(self, x: float, phi_kind: int = PHI_ELU1) -> float:
        return self.lib.oracle_phi(float(x), int(phi_kind))

    def forward(self, q, k, v, causal: bool, phi_kind: int = PHI_ELU1) -> np.ndarray:
        """q, k, v: [..., n, d] (any number of leading head axes).  Returns float64 out.
        q and k may have their own last dimension m (features, e.g. FAVOR+ with
        phi_kind=PHI_IDENTITY): then S is m x d and out has v's shape."""
        q, k, v = self._f64(q), self._f64(k), self._f64(v)
        if q.shape[-1] != v.shape[-1]:
            assert q.shape == k.shape and q.shape[:-1] == v.shape[:-1] and q.ndim >= 2
            n, m, d = q.shape[-2], q.shape[-1], v.shape[-1]
            heads = int(np.prod(q.shape[:-2], dtype=np.int64)) if q.ndim > 2 else 1
            out = np.empty_like(v)
            self.lib.oracle_forward_dkv_f64(self._ptr(q), self._ptr(k), self._ptr(v),
                                            self._ptr(out), heads, n, m, d, int(bool(causal)),
                                            int(phi_kind))
            return out
        assert q.shape == k.shape == v.shape and q.ndim >= 2
        n, d = q.shape[-2:]
        heads = int(np.prod(q.shape[:-2], dtype=np.int64)) if q.ndim > 2 else 1
        out = np.empty_like(q)
        self.lib.oracle_forward_f64(self._ptr(q), self._ptr(k), self._ptr(v), self._ptr(out),
                                    1, heads, n, d, int(bool(causal)), int(phi_kind))
        return out

    def forward_rows(self, q, k, v, rows, causal: bool, phi_kind: int = PHI_ELU1) -> np.ndarray:
        """Only the listed rows (sorted ascending) of each head: returns [heads, len(rows), d]."""
        q, k, v = self._f64(q), self._f64(k), self._f64(v)
        n, d = q.shape[-2:]
        heads = int(np.prod(q.shape[:-2], dtype=np.int64)) if q.ndim > 2 else 1
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        assert np.all(np.diff(rows) >= 0) and rows.min() >= 0 and rows.max() < n
        out = np.empty((heads, rows.size, d), dtype=np.float64)
        self.lib.oracle_forward_rows_f64(self._ptr(q), self._ptr(k), self._ptr(v),
                                         self._ptr(out), heads, n, d, int(bool(causal)),
                                         rows.ctypes.data_as(_ip), rows.size, int(phi_kind))
        return out

    def backward(self, q, k, v, g, causal: bool, phi_kind: int = PHI_ELU1):
        """Gradients of sum(g * forward(q, k, v)) with respect to q, k, v: q, k, v, g are
        [..., n, d]; returns (dq, dk, dv) as float64 arrays of that shape."""
        q, k, v, g = self._f64(q), self._f64(k), self._f64(v), self._f64(g)
        assert q.shape == k.shape == v.shape == g.shape and q.ndim >= 2
        n, d = q.shape[-2:]
        heads = int(np.prod(q.shape[:-2], dtype=np.int64)) if q.ndim > 2 else 1
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        self.lib.oracle_backward_f64(self._ptr(q), self._ptr(k), self._ptr(v), self._ptr(g),
                                     self._ptr(dq), self._ptr(dk), self._ptr(dv), 1, heads, n,
                                     d, int(bool(causal)), int(phi_kind))
        return dq, dk, dv

    def favor_features(self, x, W):
        """x: [..., d]; W: [m, d].  Returns exp(W x - |x|^2 / 2) / sqrt(m): [..., m]."""
        x, W = self._f64(x), self._f64(W)
        d = x.shape[-1]
        m = W.shape[0]
        assert W.shape == (m, d)
        rows = int(np.prod(x.shape[:-1], dtype=np.int64)) if x.ndim > 1 else 1
        out = np.empty(x.shape[:-1] + (m,), dtype=np.float64)
        self.lib.oracle_favor_features_f64(self._ptr(x), self._ptr(W), self._ptr(out), rows, d, m)
        return out

    def state(self, k, v, phi_kind: int = PHI_ELU1):
        """Final causal state per head: S [..., d, d] (row = feature, col = value), z [..., d]."""
        k, v = self._f64(k), self._f64(v)
        n, d = k.shape[-2:]
        lead = k.shape[:-2]
        heads = int(np.prod(lead, dtype=np.int64)) if lead else 1
        S = np.empty(lead + (d, d), dtype=np.float64)
        z = np.empty(lead + (d,), dtype=np.float64)
        self.lib.oracle_state_f64(self._ptr(k), self._ptr(v), self._ptr(S), self._ptr(z),
                                  heads, n, d, int(phi_kind))
        return S, z

    def decode_step(self, S, z, q, k, v, phi_kind: int = PHI_ELU1):
        """One recurrent step.  S [..., d, d], z [..., d], q/k/v [..., d].
        Returns (S', z', out) as new float64 arrays; the inputs are not modified."""
        S = np.array(S, dtype=np.float64, copy=True, order="C")
        z = np.array(z, dtype=np.float64, copy=True, order="C")
        q, k, v = self._f64(q), self._f64(k), self._f64(v)
        d = q.shape[-1]
        heads = int(np.prod(q.shape[:-1], dtype=np.int64)) if q.ndim > 1 else 1
        out = np.empty_like(q)
        self.lib.oracle_decode_step_f64(self._ptr(S), self._ptr(z), self._ptr(q), self._ptr(k),
                                        self._ptr(v), self._ptr(out), 1, heads, d,
                                        int(phi_kind))
        return S, z, out


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    """The oracle built from oracle.c without planted mistakes (built on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        if _needs_build():
            build()
        _DEFAULT = Oracle(_LIB_PATH)
    return _DEFAULT


def load_planted(plant: int) -> Oracle:
    """Build and load a variant of the oracle with planted mistake ``plant`` (1..8)."""
    tmp = tempfile.mkdtemp(prefix="oracle_plant_")
    path = build(plant=plant, out_path=os.path.join(tmp, f"liboracle_plant{plant}.so"))
    return Oracle(path)


def forward(q, k, v, causal: bool, phi_kind: int = PHI_ELU1) -> np.ndarray:
    return default().forward(q, k, v, causal, phi_kind)


def forward_rows(q, k, v, rows, causal: bool, phi_kind: int = PHI_ELU1) -> np.ndarray:
    return default().forward_rows(q, k, v, rows, causal, phi_kind)


def state(k, v, phi_kind: int = PHI_ELU1):
    return default().state(k, v, phi_kind)


def backward(q, k, v, g, causal: bool, phi_kind: int = PHI_ELU1):
    return default().backward(q, k, v, g, causal, phi_kind)


def favor_features(x, W):
    return default().favor_features(x, W)


def decode_step(S, z, q, k, v, phi_kind: int = PHI_ELU1):
    return default().decode_step(S, z, q, k, v, phi_kind)


def phi(x: float, phi_kind: int = PHI_ELU1) -> float:
    return default().phi(x, phi_kind)


def set_threads(threads: int) -> None:
    """Threads of the oracle's OpenMP loops (for timing; results do not depend on it)."""
    default().lib.oracle_set_threads(int(threads))


def get_threads() -> int:
    return int(default().lib.oracle_get_threads())


# --------------------------------------------------------------------------------------
# Brute force: the quadratic (n x n) form, the left side of the associativity law.
# --------------------------------------------------------------------------------------
def _phi_np(x: np.ndarray, phi_kind: int) -> np.ndarray:
    if phi_kind == PHI_IDENTITY:
        return x
    # elu(x) + 1 with alpha = 1: x + 1 above zero, exp(x) at or below zero
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def brute_force(q, k, v, causal: bool, phi_kind: int = PHI_ELU1) -> np.ndarray:
    """out = rownorm(mask(phi(Q) phi(K)^T)) V for one head, q/k/v [n, d], float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    W = _phi_np(q, phi_kind) @ _phi_np(k, phi_kind).T  # n x n similarity matrix
    if causal:
        W = np.tril(W)  # keep j <= i, the diagonal included
    W = W / W.sum(axis=1, keepdims=True)
    return W @ v


# --------------------------------------------------------------------------------------
# Closed forms printed on the pages.
# --------------------------------------------------------------------------------------
def memory_standard_attention(n: int, d: int, dtype_bytes: int = 4) -> int:
    """Bytes of the n x n attention weights (page "Linear Attention > Memory Efficiency")."""
    return n * n * dtype_bytes


def memory_linear_attention(n: int, d: int, D: int | None = None, dtype_bytes: int = 4) -> int:
    """Bytes of the D x d aggregate plus the D-vector key sum; independent of n
    (page "Linear Attention > Memory Efficiency")."""
    D = d if D is None else D
    return D * d * dtype_bytes + D * dtype_bytes


def flops_standard_attention(n: int, d: int) -> int:
    """QK^T (2n^2 d) + softmax (5n^2) + weights times V (2n^2 d)
    (page "Linear Attention > Computational Complexity Analysis")."""
    return 2 * n * n * d + 5 * n * n + 2 * n * n * d


def flops_linear_attention(n: int, d: int, D: int | None = None) -> int:
    """Feature map (2nd) + phi(K)^T V (2nDd) + phi(Q) times the aggregate (2nDd)
    + normalisation (2nD + n) (page "Linear Attention > Computational Complexity
    Analysis")."""
    D = d if D is None else D
    return 2 * n * d + 2 * n * D * d + 2 * n * D * d + 2 * n * D + n
