"""One sequence split over ranks: each rank holds a contiguous block of every head's tokens.

The recurrent view of linear attention (page "Efficient Transformers: Linear Attention and
Flash Attention", section "The recurrent view: attention as an RNN") carries everything the
earlier tokens contribute in one fixed-size state (S, z).  So the blocks need one exchange:

  1. this rank's block state   (S_r, z_r) = linattn_forward_state_keep(k_r, v_r), which also
     keeps the block's sums of k_r, v_r for step 4
  2. one all-gather of every rank's packed state, B*H*(d*d + d)*4 bytes per rank
  3. the state the block starts from, with linattn_sum_states:
       causal:     the sum over ranks r' < r  (the tokens before this block)
       non-causal: the sum over ranks r' != r (the rest of the sequence)
  4. out_r = linattn_forward_init_from(q_r, k_r, v_r, S0, z0, kept sums)  (k_r, v_r are read
     once in all)

Rank r of G holds tokens [r*n/G, (r+1)*n/G) of a length-n sequence (ranks in group order).
Steps 1, 3 and 4 run in this library's kernels; step 2 is the process group's all-gather
(NCCL on GPUs).  The arithmetic of steps 1, 3 and 4 is supplied by ``ops`` so that the
exchange logic can be exercised on CPU ranks; the default is the CUDA library.
"""
from __future__ import annotations


class DeviceOps:
    """The library's kernels on the tensors' CUDA device."""

    @staticmethod
    def state(k, v):
        """(S, z, carry): the block state and what forward_init may reuse."""
        from . import forward_state
        return forward_state(k, v, keep=True)

    @staticmethod
    def sum(states, count: int, skip: int):
        from . import sum_states
        return sum_states(states, count, skip)

    @staticmethod
    def forward_init(q, k, v, S0, z0, causal: bool, carry=None):
        from . import forward_init
        return forward_init(q, k, v, S0, z0, causal, aggregates=carry)


def pack_state(S, z):
    """[B, H, d, d] and [B, H, d] -> [B, H, d*d + d] (S row-major, then z)."""
    import torch
    B, H, d, _ = S.shape
    return torch.cat((S.reshape(B, H, d * d), z), dim=2).contiguous()


def start_state(gathered, rank: int, causal: bool, ops=None):
    """The state rank `rank`'s block starts from, given every rank's packed block state
    gathered[r'] ([G, B, H, d*d + d])."""
    ops = ops or DeviceOps()
    G = gathered.shape[0]
    if causal:
        return ops.sum(gathered, rank, -1)
    return ops.sum(gathered, G, rank)


def forward_sequence_sharded(q, k, v, causal: bool, group=None, ops=None):
    """q, k, v: this rank's block [B, H, n_r, d] of one sequence per head.  Returns this
    block's outputs, equal to the matching rows of the forward pass over the whole
    sequence.  Every rank of `group` must call it (one all-gather); without an initialised
    process group the block is the whole sequence."""
    import torch
    import torch.distributed as dist
    ops = ops or DeviceOps()
    single = not dist.is_available() or not dist.is_initialized()
    G = 1 if single else dist.get_world_size(group)
    r = 0 if single else dist.get_rank(group)
    S, z, carry = ops.state(k, v)
    packed = pack_state(S, z)
    if G == 1:
        gathered = packed[None]
    else:
        parts = [torch.empty_like(packed) for _ in range(G)]
        dist.all_gather(parts, packed, group=group)
        gathered = torch.stack(parts)
    S0, z0 = start_state(gathered, r, causal, ops)
    return ops.forward_init(q, k, v, S0, z0, causal, carry)
