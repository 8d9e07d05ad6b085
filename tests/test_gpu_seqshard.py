"""Device side of sequence sharding: the shard-state pass, the state-advance step, and the
chunkwise call from a combined state, run as three consecutive shards on one GPU (the ranks
of a sequence-parallel job, in order) against the fp64 oracle on the whole sequence.  The
orchestration module also runs end to end as a one-rank NCCL group.  The exchange between
several ranks is tested on CPU (tests/test_seqshard.py): this pool gives one GPU per job.
"""
import os
import socket

import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_BF16, dev, err, require_gpu

pytestmark = pytest.mark.gpu
FLAGS = rn.F_XPOS | rn.F_SCALE_SQRT_D | rn.F_NORM_D


@pytest.fixture(autouse=True)
def _gpu(cuda_lib):
    require_gpu()
    rn.retnet_debug_wait_timeouts(clear=True)
    rn.retnet_fp16_range_errors(clear=True)
    yield
    assert rn.retnet_fp16_range_errors(clear=True) == 0  # no tensor-core operand left the fp16 range
    assert rn.retnet_debug_wait_timeouts(clear=True) == 0


@pytest.mark.parametrize("dk,dv,B", [(128, 128, 64), (256, 64, 128), (64, 128, 256)])
def test_segment_state_matches_oracle(dk, dv, B):
    b, L, h, pos0 = 2, 3 * B + 17, 3, 999
    q, k, v = si.qkv(b, L, h, dk, dv, 130 + dk, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    _, s_ref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS)
    w = torch.empty(b, h, dk, dv, device="cuda")
    rn.retnet_chunkwise_segment_state(dev(k), dev(v), w, g, th, pos0, FLAGS, B)
    torch.cuda.synchronize()
    assert err(w, s_ref) <= TOL_BF16


def test_state_advance():
    b, h, dk, dv = 2, 5, 64, 96
    g = si.gamma_schedule(h)
    s0 = si.decode_state(b, h, dk, dv, 131, std=1.0)
    w = si.decode_state(b, h, dk, dv, 132, std=1.0)
    s = dev(s0)
    rn.retnet_state_advance(s, dev(w), g, 300)
    torch.cuda.synchronize()
    ref = (np.asarray(g, np.float64) ** 300)[None, :, None, None] * s0.double().numpy() + w.double().numpy()
    assert err(s, ref) <= 1e-6


@pytest.mark.parametrize("lens,dk,dv,B", [((640, 576, 300), 128, 128, 64), ((256, 512, 129), 256, 64, 128)])
def test_three_shards_match_whole_sequence(lens, dk, dv, B):
    b, h, pos0 = 1, 4, 55
    L = sum(lens)
    q, k, v = si.qkv(b, L, h, dk, dv, 133 + dk, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    s0 = si.decode_state(b, h, dk, dv, 134, std=0.3)
    ref, s_ref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS, s0)
    starts = [sum(lens[:j]) for j in range(len(lens))]
    shard = lambda x, j: dev(x[:, starts[j]:starts[j] + lens[j]])
    ws = []
    for j in range(len(lens)):  # every rank: its own shard state
        w = torch.empty(b, h, dk, dv, device="cuda")
        rn.retnet_chunkwise_segment_state(shard(k, j), shard(v, j), w, g, th, pos0 + starts[j], FLAGS, B)
        ws.append(w)
    outs, s_last = [], None
    for r in range(len(lens)):  # every rank: combine the earlier states, then its shard
        r_in = dev(s0)
        for j in range(r):
            rn.retnet_state_advance(r_in, ws[j], g, lens[j])
        o = torch.empty(b, lens[r], h, dv, device="cuda")
        s_last = torch.empty(b, h, dk, dv, device="cuda")
        rn.retnet_retention_chunkwise(shard(q, r), shard(k, r), shard(v, r), o, g, th, pos0 + starts[r], FLAGS, B,
                                      state_in=r_in, state_out=s_last)
        outs.append(o)
    torch.cuda.synchronize()
    assert err(torch.cat(outs, dim=1), ref) <= TOL_BF16
    assert err(s_last, s_ref) <= TOL_BF16


def test_module_one_rank_nccl():
    import torch.distributed as dist
    from linear_attention_sequence_chunkwise_b200.seqshard import retention_chunkwise_sharded
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        b, L, h, dk, dv, B, pos0 = 2, 333, 3, 128, 64, 64, 7
        q, k, v = si.qkv(b, L, h, dk, dv, 135, "bf16")
        g, th = si.gamma_schedule(h), si.theta_schedule(dk)
        ref, s_ref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS)
        o = torch.empty(b, L, h, dv, device="cuda")
        so = torch.empty(b, h, dk, dv, device="cuda")
        assert retention_chunkwise_sharded(dev(q), dev(k), dev(v), o, g, th, pos0, FLAGS, B, state_out=so) == pos0
        torch.cuda.synchronize()
        assert err(o, ref) <= TOL_BF16 and err(so, s_ref) <= TOL_BF16
    finally:
        dist.destroy_process_group()
