"""Parity at the benchmark workloads' full sizes, on the benchmark's own seeds and launch
configuration, against the fp64 oracle on sampled (batch, head) pairs.

The whole call runs on the device at full size; the oracle recomputes the sampled pairs one by
one (its recurrent form, "阅读笔记：RetNet" §2.2, which §2.4's chunkwise form must reproduce).
Pairs include the extreme heads of the decay schedule (gamma_0 = 1 - 2^-5, the shortest memory,
and the last head, the longest), where the fp16 operand scaling and the state's growth are at
their limits.

  - long-sequence chunkwise forward: batch 2, L 8192, 16 heads, d_k 256, d_v 512, chunks of 128
    and 512 tokens (§2.4); every output of each sampled pair and its final state.
  - recurrent decode: batch 64, 16 heads, d_k 256, d_v 512, fp32 state from 0.01 N(0, 1), 1024
    successive steps with new bf16 q, k, v each step (§2.2); every step's output of each
    sampled pair and the final state.
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_BF16, TOL_F32, err, err_bf16_out, require_gpu

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


LONG = dict(b=2, L=8192, h=16, dk=256, dv=512, seed=3)
LONG_PAIRS = [(0, 0), (1, 15), (1, 7)]


@pytest.fixture(scope="module")
def long_case():
    c = LONG
    q, k, v = si.qkv(c["b"], c["L"], c["h"], c["dk"], c["dv"], c["seed"], "bf16")
    g, th = si.gamma_schedule(c["h"]), si.theta_schedule(c["dk"])
    refs = {}
    for (bb, hh) in LONG_PAIRS:
        sl = (slice(bb, bb + 1), slice(None), slice(hh, hh + 1))
        o, S, _ = oracle.recurrent(q[sl], k[sl], v[sl], g[hh:hh + 1], th, 0, FLAGS)
        refs[(bb, hh)] = (o[0, :, 0], S[0, 0])
    return q, k, v, g, th, refs


@pytest.mark.parametrize("B", [128, 512])
def test_long_sequence_full_size(long_case, B):
    """b2/L8192/h16/d_k256/d_v512 through the workspace call the benchmark times, on the
    tensor-core kernel; fp32 output (the parity view) and bf16 output (the benchmark's)."""
    q, k, v, g, th, refs = long_case
    c = LONG
    b, L, h, dk, dv = c["b"], c["L"], c["h"], c["dk"], c["dv"]
    assert rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, B, g) == 1
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty(b, L, h, dv, device="cuda")
    so = torch.empty(b, h, dk, dv, device="cuda")
    rn.retnet_retention_chunkwise_ws(qd, kd, vd, o, g, th, 0, FLAGS, B, state_out=so, workspace=ws)
    ob = torch.empty(b, L, h, dv, device="cuda", dtype=torch.bfloat16)
    rn.retnet_retention_chunkwise_ws(qd, kd, vd, ob, g, th, 0, FLAGS, B, workspace=ws)
    torch.cuda.synchronize()
    for (bb, hh), (ro, rS) in refs.items():
        e_o = err(o[bb, :, hh], ro)
        e_b = err_bf16_out(ob[bb, :, hh], ro)
        e_s = err(so[bb, hh], rS)
        print(f"B={B} pair ({bb},{hh}): out {e_o:.3e}, bf16 out {e_b:.3e}, state {e_s:.3e}")
        assert e_o <= TOL_BF16 and e_b <= TOL_BF16 and e_s <= TOL_BF16


DEC = dict(b=64, h=16, dk=256, dv=512, seed=4, steps=1024)
DEC_PAIRS = [(0, 0), (63, 15), (17, 9)]


def test_decode_1024_steps_full_size():
    """1024 decode steps of b64/h16/d_k256/d_v512 from the 0.01 N(0,1) state; the step kernel
    computes in fp32, so outputs and state are held to the fp32 bar."""
    c = DEC
    b, h, dk, dv, n = c["b"], c["h"], c["dk"], c["dv"], c["steps"]
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, c["seed"])
    S = S0.cuda()
    o = torch.empty(b, h, dv, device="cuda")
    outs = {p: np.zeros((n, dv)) for p in DEC_PAIRS}
    toks = {p: [np.zeros((n, dk)), np.zeros((n, dk)), np.zeros((n, dv))] for p in DEC_PAIRS}
    for t in range(n):
        q, k, v = si.decode_token(b, h, dk, dv, c["seed"], t)
        rn.retnet_retention_step(q.cuda(), k.cuda(), v.cuda(), o, S, g, th, t, FLAGS)
        oh = o.cpu()
        for (bb, hh) in DEC_PAIRS:
            outs[(bb, hh)][t] = oh[bb, hh].double().numpy()
            for j, x in enumerate((q, k, v)):
                toks[(bb, hh)][j][t] = x[bb, hh].double().numpy()
    Sh = S.cpu()
    for (bb, hh) in DEC_PAIRS:
        tq, tk, tv = (torch.from_numpy(x)[None, :, None] for x in toks[(bb, hh)])
        ro, rS, _ = oracle.recurrent(tq, tk, tv, g[hh:hh + 1], th, 0, FLAGS, S0[bb:bb + 1, hh:hh + 1])
        e_o = err(outs[(bb, hh)], ro[0, :, 0])
        e_s = err(Sh[bb, hh], rS[0, 0])
        print(f"decode pair ({bb},{hh}): outputs {e_o:.3e}, final state {e_s:.3e}")
        assert e_o <= TOL_F32 and e_s <= TOL_F32


MSR = dict(b=4, L=4096, h=8, dk=256, dv=256, B=256, seed=5)
MSR_ROWS = [0, 3]
EPS = 1e-5


@pytest.fixture(scope="module")
def msr_case():
    c = MSR
    q, k, v = si.qkv(c["b"], c["L"], c["h"], c["dk"], c["dv"], c["seed"], "bf16")
    gt = si.gate(c["b"], c["L"], c["h"], c["dv"], c["seed"], "bf16")
    g, th = si.gamma_schedule(c["h"]), si.theta_schedule(c["dk"])
    refs = {}
    for bb in MSR_ROWS:
        y, _, _ = oracle.recurrent(q[bb:bb + 1], k[bb:bb + 1], v[bb:bb + 1], g, th, 0, FLAGS)
        refs[bb] = oracle.msr_epilogue(y, gt[bb:bb + 1], c["h"], EPS)[0]
    return q, k, v, gt, g, th, refs


@pytest.mark.parametrize("form", ["fused", "two_kernel"])
def test_msr_full_size(msr_case, form):
    """b4/L4096/h8/d256/chunk 256 MSR block (retention, GroupNorm per head, swish gate),
    compared after the epilogue on whole batch rows (every head: GroupNorm is per head)."""
    q, k, v, gt, g, th, refs = msr_case
    c = MSR
    b, L, h, dk, dv, B = c["b"], c["L"], c["h"], c["dk"], c["dv"], c["B"]
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), gt.cuda()
    outs = {}
    for out_dtype in (torch.float32, torch.bfloat16):
        out = torch.empty(b, L, h, dv, device="cuda", dtype=out_dtype)
        if form == "fused":
            rn.retnet_msr_chunkwise(qd, kd, vd, gd.view(b, L, h, dv), out, g, th, 0, FLAGS, B, EPS, workspace=ws)
        else:
            y = torch.empty(b, L, h, dv, device="cuda", dtype=torch.float32)
            rn.retnet_retention_chunkwise_ws(qd, kd, vd, y, g, th, 0, FLAGS, B, workspace=ws)
            yb = y.view(b, L, h * dv)
            rn.retnet_msr_epilogue(yb, gd.float(), out.view(b, L, h * dv), h, EPS)
        outs[out_dtype] = out
    torch.cuda.synchronize()
    for bb, ref in refs.items():
        e = err(outs[torch.float32][bb].reshape(L, h * dv), ref.reshape(L, h * dv))
        e_b = err_bf16_out(outs[torch.bfloat16][bb].reshape(L, h * dv), ref.reshape(L, h * dv))
        print(f"MSR {form} row {bb}: out {e:.3e}, bf16 out {e_b:.3e}")
        assert e <= TOL_BF16 and e_b <= TOL_BF16
