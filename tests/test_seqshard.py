"""Sequence sharding over ranks (the exchange step of sequence-parallel chunkwise retention).

CPU, gloo, world size 2 and 3: every rank holds a consecutive shard; the per-rank operations
are stood in for by the fp64 oracle (tests may call it), so this checks the exchange itself
-- shard lengths and start positions, the all-gather of shard states, the combination order
-- against the oracle on the whole sequence.  The device operations are checked on a GPU in
tests/test_gpu_seqshard.py.
"""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FLAGS = 1 | 2 | 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops():
    import torch

    import oracle
    from linear_attention_sequence_chunkwise_b200.seqshard import ShardOps

    def segment_state(k, v, w, g, th, p0, fl, ch):
        _, S, _ = oracle.recurrent(k.numpy(), k.numpy(), v.numpy(), g, th, p0, fl)
        w.copy_(torch.from_numpy(S).float())

    def state_advance(s, w, g, n):
        f = torch.tensor(np.asarray(g, dtype=np.float64) ** n, dtype=torch.float32).view(1, -1, 1, 1)
        s.mul_(f).add_(w)

    def chunkwise(q, k, v, o, g, th, p0, fl, ch, si, so):
        out, S, _ = oracle.recurrent(q.numpy(), k.numpy(), v.numpy(), g, th, p0, fl, si.double().numpy())
        o.copy_(torch.from_numpy(out).float())
        if so is not None:
            so.copy_(torch.from_numpy(S).float())

    return ShardOps(segment_state, state_advance, chunkwise)


def _worker(rank, world, port, lens, queue):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import synth_inputs as si
    from linear_attention_sequence_chunkwise_b200.seqshard import retention_chunkwise_sharded
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    b, h, dk, dv, chunk, pos0 = 2, 2, 8, 6, 4, 37
    L = sum(lens)
    q, k, v = si.qkv(b, L, h, dk, dv, 50, "f32")
    s0 = si.decode_state(b, h, dk, dv, 51, std=0.5)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    lo = sum(lens[:rank])
    sl = slice(lo, lo + lens[rank])
    o = torch.empty(b, lens[rank], h, dv)
    so = torch.empty(b, h, dk, dv)
    start = retention_chunkwise_sharded(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), o, g,
                                        th, pos0, FLAGS, chunk, state_in=s0, state_out=so, ops=_oracle_ops())
    queue.put((rank, start, o.numpy(), so.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def _run(lens):
    import oracle
    import synth_inputs as si
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    world = len(lens)
    procs = [ctx.Process(target=_worker, args=(r, world, port, lens, queue)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((queue.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    b, h, dk, dv, pos0 = 2, 2, 8, 6, 37
    L = sum(lens)
    q, k, v = si.qkv(b, L, h, dk, dv, 50, "f32")
    s0 = si.decode_state(b, h, dk, dv, 51, std=0.5)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref, s_ref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS, s0)
    assert [r[1] for r in res] == [pos0 + sum(lens[:i]) for i in range(world)]
    out = np.concatenate([r[2] for r in res], axis=1)
    rms = np.sqrt((ref ** 2).mean())
    assert np.abs(out - ref).max() / rms <= 1e-5
    assert np.abs(res[-1][3] - s_ref).max() / np.sqrt((s_ref ** 2).mean()) <= 1e-5


def test_two_ranks_whole_chunks():
    _run([12, 9])


def test_three_ranks_ragged_last_shard():
    _run([8, 16, 7])
