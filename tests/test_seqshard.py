"""Sequence sharding (one sequence split over ranks, one exchange of block states).

CPU: two gloo ranks run the exchange logic of seqshard.forward_sequence_sharded with float64
numpy stand-ins for the three device steps (block state, state sum, forward from a state);
each rank's block must equal the matching rows of the oracle's forward over the whole
sequence.  GPU: the library's own steps, with the ranks emulated one after another on one
device (no kernel waits for another), against the oracle.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from linear_attention_linattn_b200 import inputs, seqshard
from tests.helpers import TOL, as_io, max_row_rel_err


def _phi(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


class NumpyOps:
    """float64 stand-ins for the device steps (test scaffolding on CPU tensors)."""

    @staticmethod
    def state(k, v):
        fk = _phi(k.double().numpy())
        vv = v.double().numpy()
        S = np.einsum("bhnr,bhnc->bhrc", fk, vv)
        return torch.from_numpy(S), torch.from_numpy(fk.sum(axis=2)), None

    @staticmethod
    def sum(states, count, skip):
        st = states.double().numpy()
        B, H, per = st.shape[1:]
        d = int(round((-1 + (1 + 4 * per) ** 0.5) / 2))
        acc = np.zeros((B, H, per))
        for i in range(count):
            if i != skip:
                acc += st[i]
        return (torch.from_numpy(acc[..., :d * d].reshape(B, H, d, d)),
                torch.from_numpy(acc[..., d * d:].copy()))

    @staticmethod
    def forward_init(q, k, v, S0, z0, causal, carry=None):
        fq, fk = _phi(q.double().numpy()), _phi(k.double().numpy())
        vv = v.double().numpy()
        S0, z0 = S0.double().numpy(), z0.double().numpy()
        if causal:
            S = S0[:, :, None] + np.cumsum(np.einsum("bhnr,bhnc->bhnrc", fk, vv), axis=2)
            z = z0[:, :, None] + np.cumsum(fk, axis=2)
            num = np.einsum("bhnr,bhnrc->bhnc", fq, S)
            den = np.einsum("bhnr,bhnr->bhn", fq, z)
        else:
            S = S0 + np.einsum("bhnr,bhnc->bhrc", fk, vv)
            z = z0 + fk.sum(axis=2)
            num = np.einsum("bhnr,bhrc->bhnc", fq, S)
            den = np.einsum("bhnr,bhr->bhn", fq, z)
        return torch.from_numpy(num / den[..., None])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, n, d = 1, 2, 96, 8
        q, k, v = inputs.forward_qkv(41, B, H, n, d, scaled=True)
        blk = n // world
        sl = slice(rank * blk, (rank + 1) * blk)
        mine = [torch.from_numpy(np.ascontiguousarray(x[:, :, sl])) for x in (q, k, v)]
        got = seqshard.forward_sequence_sharded(*mine, causal, ops=NumpyOps())
        out[rank] = got.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("causal", [True, False])
def test_two_gloo_ranks_match_whole_sequence(causal):
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, causal, out), nprocs=world,
                           start_method="spawn")
        res = dict(out)
    B, H, n, d = 1, 2, 96, 8
    q, k, v = inputs.forward_qkv(41, B, H, n, d, scaled=True)
    ref = oracle.forward(q, k, v, causal)
    got = np.concatenate([res[r] for r in range(world)], axis=2)
    assert max_row_rel_err(got, ref) <= 1e-12


def test_start_state_selects_earlier_or_other_ranks():
    """Which blocks a rank's start state sums: causal, the ranks before it; non-causal, all
    the others."""
    G, B, H, d = 4, 1, 1, 2
    states = torch.zeros(G, B, H, d * d + d, dtype=torch.float64)
    for i in range(G):
        states[i] = 10.0 ** i
    for r in range(G):
        S, _ = seqshard.start_state(states, r, True, NumpyOps())
        assert float(S[0, 0, 0, 0]) == sum(10.0 ** i for i in range(r))
        S, _ = seqshard.start_state(states, r, False, NumpyOps())
        assert float(S[0, 0, 0, 0]) == sum(10.0 ** i for i in range(G) if i != r)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_blocks_on_one_gpu_match_oracle(dtype, causal, d):
    """Four blocks of 1100 tokens (ragged against the 64-token chunk), emulated as ranks one
    after another on one GPU with the library's kernels."""
    import linear_attention_linattn_b200 as la
    from tests.helpers import to_dev, to_host
    B, H, G, blk = 1, 3, 4, 1100
    n = G * blk
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(42, B, H, n, d, scaled=True))
    blocks = [[to_dev(np.ascontiguousarray(x[:, :, r * blk:(r + 1) * blk]), dtype)
               for x in (q, k, v)] for r in range(G)]
    packed = [seqshard.pack_state(*la.forward_state(bk, bv)) for _, bk, bv in blocks]
    gathered = torch.stack(packed)
    outs = []
    for r, (bq, bk, bv) in enumerate(blocks):
        S0, z0 = seqshard.start_state(gathered, r, causal)
        outs.append(to_host(la.forward_init(bq, bk, bv, S0, z0, causal)))
    assert la.device_error() == la.LINATTN_OK
    got = np.concatenate(outs, axis=2)
    assert max_row_rel_err(got, oracle.forward(q, k, v, causal)) <= TOL[dtype]


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_blocks_reusing_their_sums_match_oracle(dtype, causal, d):
    """The same four blocks through the calls that read k, v once per block: the state call
    keeps the block's sums (linattn_forward_state_keep) and the block's pass reuses them
    (linattn_forward_init_from), as forward_sequence_sharded does."""
    import linear_attention_linattn_b200 as la
    from tests.helpers import to_dev, to_host
    B, H, G, blk = 1, 3, 4, 1100
    n = G * blk
    q, k, v = (as_io(x, dtype) for x in inputs.forward_qkv(43, B, H, n, d, scaled=True))
    blocks = [[to_dev(np.ascontiguousarray(x[:, :, r * blk:(r + 1) * blk]), dtype)
               for x in (q, k, v)] for r in range(G)]
    kept = [la.forward_state(bk, bv, keep=True) for _, bk, bv in blocks]
    # the kept call's state is the plain call's
    for (_, bk, bv), (S, z, _) in zip(blocks, kept):
        S1, z1 = la.forward_state(bk, bv)
        assert torch.equal(S, S1) and torch.equal(z, z1)
    gathered = torch.stack([seqshard.pack_state(S, z) for S, z, _ in kept])
    outs = []
    for r, (bq, bk, bv) in enumerate(blocks):
        S0, z0 = seqshard.start_state(gathered, r, causal)
        outs.append(to_host(la.forward_init(bq, bk, bv, S0, z0, causal, aggregates=kept[r][2])))
    assert la.device_error() == la.LINATTN_OK
    got = np.concatenate(outs, axis=2)
    assert max_row_rel_err(got, oracle.forward(q, k, v, causal)) <= TOL[dtype]


@pytest.mark.gpu
def test_sharded_forward_reads_each_block_once():
    """forward_sequence_sharded without a process group (one block = the whole sequence)
    launches the aggregates once: the state call's, reused by the block's pass."""
    import linear_attention_linattn_b200 as la
    from tests.helpers import to_dev, to_host
    B, H, n, d = 1, 2, 3000, 64
    q, k, v = (as_io(x, "bf16") for x in inputs.forward_qkv(44, B, H, n, d, scaled=True))
    qd, kd, vd = (to_dev(x, "bf16") for x in (q, k, v))
    for causal in (True, False):
        got = to_host(seqshard.forward_sequence_sharded(qd, kd, vd, causal))
        assert max_row_rel_err(got, oracle.forward(q, k, v, causal)) <= TOL["bf16"]
    lib = la.load_library()
    l0 = lib.linattn_launch_count()
    seqshard.forward_sequence_sharded(qd, kd, vd, True)
    torch.cuda.synchronize()
    # state: aggregates + total; sum of states; pass: prefix + outputs (no second aggregate)
    assert lib.linattn_launch_count() - l0 == 5


@pytest.mark.gpu
def test_sum_states_on_gpu():
    """linattn_sum_states adds the gathered states in order, skipping one."""
    import linear_attention_linattn_b200 as la
    rng = np.random.default_rng(3)
    G, B, H, d = 5, 2, 3, 64
    st = rng.standard_normal((G, B, H, d * d + d)).astype(np.float32)
    states = torch.from_numpy(st).cuda()
    for count, skip in ((0, -1), (3, -1), (5, 2), (5, -1)):
        S, z = la.sum_states(states, count, skip)
        ref = sum((st[i].astype(np.float64) for i in range(count) if i != skip),
                  np.zeros((B, H, d * d + d)))
        assert np.allclose(S.cpu().numpy().reshape(B, H, -1), ref[..., :d * d], atol=1e-5)
        assert np.allclose(z.cpu().numpy(), ref[..., d * d:], atol=1e-5)
