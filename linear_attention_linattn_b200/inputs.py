"""Seeded synthetic inputs, shared by the CUDA path's tests/benchmark and the oracle.

This module holds none of the method's arithmetic: it only draws numbers and rounds
them to the I/O precision.  Both sides receive the same arrays from here.

Recipe (the pages name no generator; this is the one used everywhere):
  * per head (b, h): ``rng = numpy.random.default_rng([seed, b, h])``;
  * one draw ``rng.standard_normal((3, n, d), dtype=float32)`` gives q, k, v in that order;
  * multiplied by float32(1/sqrt(d)) when the workload says "N(0,1)/sqrt(d)";
  * for bf16 I/O, rounded to bf16 (round to nearest even); the oracle is then given the
    rounded values, so input quantisation is not counted as error.
  * decode workloads: per (sequence s, head h), ``default_rng([seed, s, h])`` draws the
    prefill block (3, P, d) and then the step block (3, T, d), q/k/v in that order.

The five workloads of this library's measurement plan are listed in ``WORKLOADS``.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "forward" or "decode"
    B: int               # batch (forward) or sequences (decode)
    H: int
    n: int               # tokens per head (forward) or prefill length (decode)
    d: int
    causal: tuple        # modes run on this workload
    dtypes: tuple        # I/O dtypes ("f32", "bf16")
    seed: int
    scaled: bool         # inputs multiplied by 1/sqrt(d)
    steps: int = 0       # decode steps

    @property
    def tokens(self) -> int:
        return self.B * self.n


WORKLOADS = {
    # non-causal, 1 x 1 x 512 x 64, fp32, N(0,1) unscaled, seed 0
    "noncausal_1x1x512x64_f32": Workload("noncausal_1x1x512x64_f32", "forward", 1, 1, 512, 64,
                                         (False,), ("f32",), 0, False),
    # causal, 1 x 1 x 4096 x 64, fp32 and bf16 I/O, N(0,1)/sqrt(d), seed 1
    "causal_1x1x4096x64": Workload("causal_1x1x4096x64", "forward", 1, 1, 4096, 64,
                                   (True,), ("f32", "bf16"), 1, True),
    # 8 x 16 x 8192 x 64, bf16, non-causal and causal, N(0,1)/sqrt(d), seed 2
    "batched_8x16x8192x64_bf16": Workload("batched_8x16x8192x64_bf16", "forward", 8, 16, 8192,
                                          64, (False, True), ("bf16",), 2, True),
    # long-context causal 1 x 32 x 131072 x 128, bf16, N(0,1)/sqrt(d), seed 3
    "longctx_1x32x131072x128_bf16": Workload("longctx_1x32x131072x128_bf16", "forward", 1, 32,
                                             131072, 128, (True,), ("bf16",), 3, True),
    # decode: 256 sequences x 32 heads, d = 128, prefill 2048 tokens, 512 steps, seed 4
    "decode_256x32x128": Workload("decode_256x32x128", "decode", 256, 32, 2048, 128,
                                  (True,), ("bf16",), 4, True, steps=512),
}


def head_qkv(seed: int, b: int, h: int, n: int, d: int, scaled: bool):
    """q, k, v for one head as float32 arrays [n, d]."""
    rng = np.random.default_rng([seed, b, h])
    x = rng.standard_normal((3, n, d), dtype=np.float32)
    if scaled:
        x *= np.float32(1.0 / math.sqrt(d))
    return x[0], x[1], x[2]


def forward_qkv(seed: int, B: int, H: int, n: int, d: int, scaled: bool,
                heads=None, threads: int = 8):
    """q, k, v as float32 [B, H, n, d].  ``heads`` (a list of (b, h)) restricts the draw to
    those heads and returns [len(heads), n, d] arrays instead."""
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    q = np.empty((len(pairs), n, d), dtype=np.float32)
    k = np.empty_like(q)
    v = np.empty_like(q)

    def fill(i):
        b, h = pairs[i]
        q[i], k[i], v[i] = head_qkv(seed, b, h, n, d, scaled)

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range(len(pairs))))
    if heads is None:
        return q.reshape(B, H, n, d), k.reshape(B, H, n, d), v.reshape(B, H, n, d)
    return q, k, v


def decode_qkv(seed: int, s: int, h: int, d: int, prefill: int, steps: int, scaled: bool):
    """For one (sequence, head): prefill q, k, v [prefill, d] and step q, k, v [steps, d]."""
    rng = np.random.default_rng([seed, s, h])
    pre = rng.standard_normal((3, prefill, d), dtype=np.float32)
    stp = rng.standard_normal((3, steps, d), dtype=np.float32)
    if scaled:
        pre *= np.float32(1.0 / math.sqrt(d))
        stp *= np.float32(1.0 / math.sqrt(d))
    return (pre[0], pre[1], pre[2]), (stp[0], stp[1], stp[2])


def decode_batch(seed: int, Bseq: int, H: int, d: int, prefill: int, steps: int, scaled: bool,
                 threads: int = 8, pairs=None):
    """Arrays for a decode workload: prefill q/k/v [Bseq, H, prefill, d] and step
    q/k/v [steps, Bseq, H, d] (step-major, as each step call consumes one slice).
    ``pairs`` restricts to a list of (s, h) and returns [len, ...] leading axes."""
    sel = [(s, h) for s in range(Bseq) for h in range(H)] if pairs is None else list(pairs)
    pq = np.empty((len(sel), prefill, d), dtype=np.float32)
    pk = np.empty_like(pq)
    pv = np.empty_like(pq)
    sq = np.empty((steps, len(sel), d), dtype=np.float32)
    sk = np.empty_like(sq)
    sv = np.empty_like(sq)

    def fill(i):
        s, h = sel[i]
        (a, b_, c), (x, y, w) = decode_qkv(seed, s, h, d, prefill, steps, scaled)
        pq[i], pk[i], pv[i] = a, b_, c
        sq[:, i], sk[:, i], sv[:, i] = x, y, w

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range(len(sel))))
    if pairs is None:
        return ((pq.reshape(Bseq, H, prefill, d), pk.reshape(Bseq, H, prefill, d),
                 pv.reshape(Bseq, H, prefill, d)),
                (sq.reshape(steps, Bseq, H, d), sk.reshape(steps, Bseq, H, d),
                 sv.reshape(steps, Bseq, H, d)))
    return (pq, pk, pv), (sq, sk, sv)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bf16 (ties to even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(x.shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of float32 values, round to nearest even."""
    r = round_bf16(x)
    return (r.view(np.uint32) >> 16).astype(np.uint16)
