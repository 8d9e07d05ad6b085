"""Sequence-sharded chunkwise retention across ranks (one process per GPU).

The chunkwise recurrent form of "阅读笔记：RetNet" §2.4 carries the state from chunk to chunk,
R_i = gamma^B R_{i-1} + K_[i]^T (V_[i] (.) zeta).  That recurrence is an associative scan:
a stretch of L tokens whose own state (from a zero start) is W moves any state R to
gamma^L R + W.  So a sequence cut into consecutive shards, one shard per rank, needs one
exchange:

  1. every rank computes the state W_r its own shard leaves behind from a zero start
     (retnet_chunkwise_segment_state: K and V only, no outputs);
  2. the W_r are all-gathered (NCCL over NVLink on GPUs);
  3. rank r builds the state in front of its shard,
        R_in(r) = gamma^(L_0+...+L_{r-1}) S0 + sum_{j<r} gamma^(L_{j+1}+...+L_{r-1}) W_j,
     by repeated retnet_state_advance, and runs its chunkwise call from it with the shard's
     absolute start position.

Chunk boundaries match the unsharded call when every shard but the last is a whole number of
chunks; that is required.  The computation runs in the library's kernels; this module only
moves tensors and calls the collective.
"""
from dataclasses import dataclass
from typing import Callable, Optional


@dataclass
class ShardOps:
    """The three device operations a rank runs (the library's entry points by default)."""
    segment_state: Callable  # (k, v, state_out, gamma, theta, pos0, flags, chunk)
    state_advance: Callable  # (state, w, gamma, length)
    chunkwise: Callable      # (q, k, v, o, gamma, theta, pos0, flags, chunk, state_in, state_out)


def library_ops() -> ShardOps:
    import linear_attention_sequence_chunkwise_b200 as rn
    return ShardOps(
        segment_state=lambda k, v, w, g, th, p0, fl, ch: rn.retnet_chunkwise_segment_state(k, v, w, g, th, p0, fl, ch),
        state_advance=lambda s, w, g, n: rn.retnet_state_advance(s, w, g, n),
        chunkwise=lambda q, k, v, o, g, th, p0, fl, ch, si, so: rn.retnet_retention_chunkwise(
            q, k, v, o, g, th, p0, fl, ch, state_in=si, state_out=so))


def retention_chunkwise_sharded(q, k, v, o, gamma, theta, pos0, flags, chunk, state_in=None, state_out=None,
                                group=None, ops: Optional[ShardOps] = None):
    """Chunkwise retention of a sequence whose consecutive shards live on the ranks of `group`.

    Rank r holds q, k (batch, L_r, heads, d_k) and v, o (batch, L_r, heads, d_v) of its shard;
    ranks are in sequence order.  pos0 is the absolute position of the whole sequence's first
    token and state_in its initial state (batch, heads, d_k, d_v) fp32 (None = zeros) -- the
    same on every rank.  state_out, if given, receives the state after this rank's shard (on
    the last rank: after the whole sequence).  Returns the shard's absolute start position.
    """
    import torch
    import torch.distributed as dist
    ops = ops or library_ops()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    # shard lengths, in rank order
    lens_t = torch.empty(world, dtype=torch.int64, device=dev)
    dist.all_gather_into_tensor(lens_t, torch.tensor([L], dtype=torch.int64, device=dev), group=group)
    lens = [int(x) for x in lens_t.cpu()]
    if any(n % chunk for n in lens[:-1]):
        raise ValueError(f"every shard but the last must be a whole number of chunks of {chunk}: {lens}")
    start = int(pos0) + sum(lens[:rank])
    # 1. this shard's own state
    w = torch.empty(b, h, dk, dv, dtype=torch.float32, device=dev)
    ops.segment_state(k, v, w, gamma, theta, start, flags, chunk)
    # 2. every shard's state
    w_all = torch.empty(world * b, h, dk, dv, dtype=torch.float32, device=dev)  # rank-major
    dist.all_gather_into_tensor(w_all, w, group=group)
    # 3. the state in front of this shard, then the shard itself
    r_in = torch.zeros(b, h, dk, dv, dtype=torch.float32, device=dev)
    if state_in is not None:
        r_in.copy_(state_in)
    for j in range(rank):
        ops.state_advance(r_in, w_all[j * b:(j + 1) * b], gamma, lens[j])
    ops.chunkwise(q, k, v, o, gamma, theta, start, flags, chunk, r_in, state_out)
    return start
