"""Multi-process host logic of bench.py on CPU (gloo, world size 2, 127.0.0.1).

The retention path shards by batch with no exchange step, so the only collectives the timed
step uses are a barrier and the MAX of the per-rank timings; the reference arm runs on rank 0
only; `--gpus N` starts N ranks.  These run here without a GPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w, r, lr = bench.dist_env()
    bench.barrier(w)
    mx = bench.max_over_ranks(1.5 + rank, w, torch.device("cpu"))
    # every rank generates its own batch: the seeds differ by rank
    cfg = dict(bench.MAIN, batch=1, seqlen=8)
    sets = bench.make_main_inputs(cfg, torch.device("cpu"), rank)
    q.put((rank, (w, r, lr), mx, float(sets[0][0].float().sum())))
    bench.barrier(w)
    dist.destroy_process_group()


def test_max_over_ranks_and_rank_local_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [(2, 0, 0), (2, 1, 1)]
    assert all(r[2] == 2.5 for r in res)     # max over ranks of 1.5 + rank
    assert res[0][3] != res[1][3]            # each rank draws its own batch


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def _clean_env():
    env = dict(os.environ)
    for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT", "LOCAL_WORLD_SIZE"):
        env.pop(key, None)
    return env


def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun relaunches itself with two processes; the stub leg
    (launch plumbing only, gloo on CPU) counts the ranks that joined and rank 0 reports them."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--stub", "--steps", "1",
                        "--warmup", "3"], env=_clean_env(), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2 and rec["ranks_seen"] == 2 and rec["value"] is None


def test_rank_count_mismatch_fails_loudly():
    """A launcher that starts fewer ranks than --gpus asks for is an error, not a 1-GPU number."""
    env = dict(_clean_env(), RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--stub"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "--gpus 2" in r.stderr
