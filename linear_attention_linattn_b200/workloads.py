"""Device-resident inputs for the measured workloads (used by the benchmark and tests).

Inputs come from the seeded generator in ``inputs.py``.  The decode workload's starting
state is the final state of a causal prefill over its 2048 prefill tokens, computed on
the device with ``linattn_forward_state`` in batches of sequences, so the host never
holds the whole prefill at once.
"""
from __future__ import annotations

import numpy as np

from . import inputs


def forward_inputs(name: str, dtype: str, device="cuda"):
    """q, k, v on the device for a forward workload; dtype "f32" or "bf16"."""
    import torch
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.forward_qkv(w.seed, w.B, w.H, w.n, w.d, w.scaled)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return tuple(torch.from_numpy(x).to(tdt).to(device) for x in (q, k, v))


def decode_inputs(name: str = "decode_256x32x128", device="cuda", seq_batch: int = 16,
                  steps: int | None = None):
    """(S, z, q_steps, k_steps, v_steps): S [Bseq,H,d,d] and z [Bseq,H,d] float32 from the
    prefill; per-step q/k/v [T,Bseq,H,d] bfloat16."""
    import torch

    import linear_attention_linattn_b200 as la
    w = inputs.WORKLOADS[name]
    Bseq, H, d, P = w.B, w.H, w.d, w.n
    T = w.steps if steps is None else steps
    S = torch.empty((Bseq, H, d, d), dtype=torch.float32, device=device)
    z = torch.empty((Bseq, H, d), dtype=torch.float32, device=device)
    qs = torch.empty((T, Bseq, H, d), dtype=torch.bfloat16, device=device)
    ks = torch.empty_like(qs)
    vs = torch.empty_like(qs)
    for s0 in range(0, Bseq, seq_batch):
        s1 = min(Bseq, s0 + seq_batch)
        pairs = [(s, h) for s in range(s0, s1) for h in range(H)]
        (_, pk, pv), (sq, sk, sv) = inputs.decode_batch(w.seed, Bseq, H, d, P, w.steps, w.scaled,
                                                        pairs=pairs)
        nb = s1 - s0
        kd = torch.from_numpy(pk.reshape(nb, H, P, d)).to(torch.bfloat16).to(device)
        vd = torch.from_numpy(pv.reshape(nb, H, P, d)).to(torch.bfloat16).to(device)
        la.forward_state(kd, vd, S[s0:s1], z[s0:s1])
        for dst, src in ((qs, sq), (ks, sk), (vs, sv)):
            dst[:, s0:s1] = torch.from_numpy(
                np.ascontiguousarray(src[:T]).reshape(T, nb, H, d)).to(torch.bfloat16).to(device)
        del kd, vd
    torch.cuda.synchronize()
    return S, z, qs, ks, vs
