"""Parity of the retention gradient (retnet_retention_backward) against the fp64 oracle's
gradient (pinned by finite differences in test_oracle_pins.py), on both paths.

Bar: max|err|/rms(oracle) <= 1e-4 for every output on the fp32 CUDA-core path (fp32
arithmetic; bf16 inputs are exact in both); <= 1e-2 on the tensor-core path (three runs of the
chunkwise kernel: fp16 operands, the rotated / scaled value rows rounded to fp16 once).
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_BF16, TOL_F32, dev, err, require_gpu

pytestmark = pytest.mark.gpu
FLAGS = rn.F_XPOS | rn.F_SCALE_SQRT_D | rn.F_NORM_D


@pytest.fixture(autouse=True)
def _gpu(cuda_lib):
    require_gpu()
    rn.retnet_debug_wait_timeouts(clear=True)
    rn.retnet_fp16_range_errors(clear=True)
    yield
    assert rn.retnet_fp16_range_errors(clear=True) == 0  # no tensor-core operand left the fp16 range
    assert rn.retnet_debug_wait_timeouts(clear=True) == 0  # no bounded wait in the runs gave up


@pytest.mark.parametrize("b,L,h,dk,dv,dtype,flags,pos0,with_state", [
    (2, 100, 3, 64, 32, "f32", FLAGS, 5, True),
    (2, 300, 3, 64, 128, "bf16", FLAGS, 17, True),   # tensor cores: ragged last chunk, state
    (1, 130, 2, 256, 64, "bf16", FLAGS, 0, False),
    (4, 640, 2, 128, 128, "bf16", FLAGS, 3, True),   # two-pass segments inside the runs
    (1, 200, 2, 128, 128, "bf16", FLAGS, 0, False),
    (1, 70, 2, 256, 256, "bf16", FLAGS, 1000, True),
    (2, 37, 2, 6, 5, "f32", FLAGS, 3, True),   # ragged widths: lanes past d_k, d_v idle
    (1, 1, 1, 64, 64, "f32", FLAGS, 0, True),  # one token
    (1, 90, 4, 32, 64, "bf16", 0, 0, True),    # no rotation, no row factors
])
def test_backward_matches_oracle(b, L, h, dk, dv, dtype, flags, pos0, with_state):
    q, k, v = si.qkv(b, L, h, dk, dv, 500 + dk + L, dtype)
    do = si.randn((b, L, h, dv), 501 + L, dtype)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 502, std=0.3) if with_state else None
    rq, rk, rv, rs = oracle.backward(q, k, v, do, g, th, pos0, flags, state_in=S0)
    dq = torch.empty(b, L, h, dk, device="cuda")
    dk_ = torch.empty_like(dq)
    dv_ = torch.empty(b, L, h, dv, device="cuda")
    ds = torch.empty(b, h, dk, dv, device="cuda")
    ws = torch.empty(rn.retnet_backward_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    path = rn.retnet_backward_kernel((b, L, h, dk), dv, rn.BF16 if dtype == "bf16" else rn.F32, flags, g, ws.numel())
    assert path == (1 if dtype == "bf16" and dk in (64, 128, 256) and dv in (64, 128, 256) else 0)
    rn.retnet_retention_backward(dev(q), dev(k), dev(v), dev(do), dq, dk_, dv_, g, th, pos0, flags,
                                 state_in=None if S0 is None else dev(S0), dstate=ds, workspace=ws)
    torch.cuda.synchronize()
    if S0 is None:  # dS0 does not depend on S0: the oracle gives it with a zero state
        _, _, _, rs = oracle.backward(q, k, v, do, g, th, pos0, flags, state_in=np.zeros((b, h, dk, dv)))
    errs = [err(dq, rq), err(dk_, rk), err(dv_, rv), err(ds, rs)]
    print(f"backward b={b} L={L} h={h} dk={dk} dv={dv} {dtype} path={path}: dq/dk/dv/dS0 errors " +
          " ".join(f"{e:.2e}" for e in errs))
    assert max(errs) <= (TOL_BF16 if path == 1 else TOL_F32)


def test_backward_rejects_norm_r_and_checks_workspace():
    b, L, h, dk, dv = 1, 16, 1, 64, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 9, "f32")
    g = si.gamma_schedule(h)
    out = [torch.empty(b, L, h, d, device="cuda") for d in (dk, dk, dv)]
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        rn.retnet_retention_backward(dev(q), dev(k), dev(v), dev(v), *out, g, si.theta_schedule(dk),
                                     flags=rn.F_ALL)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="BAD_PARAM"):
        rn.retnet_retention_backward(dev(q), dev(k), dev(v), dev(v), *out, g, si.theta_schedule(dk),
                                     workspace=small)


def test_backward_cuda_core_path_with_small_workspace():
    """The same bf16 call with a workspace of only the CUDA-core path's size takes that path
    (fp32 bar), and matches the tensor-core path's result within the bf16 bar."""
    b, L, h, dk, dv = 1, 150, 2, 128, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 77, "bf16")
    do = si.randn((b, L, h, dv), 78, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    rq, rk, rv, _ = oracle.backward(q, k, v, do, g, th, 0, FLAGS)
    small = torch.empty(2 * 4 * b * L * h * dk, dtype=torch.uint8, device="cuda")
    assert rn.retnet_backward_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, g, small.numel()) == 0
    outs = [torch.empty(b, L, h, d, device="cuda") for d in (dk, dk, dv)]
    rn.retnet_retention_backward(dev(q), dev(k), dev(v), dev(do), *outs, g, th, 0, FLAGS, workspace=small)
    torch.cuda.synchronize()
    assert max(err(outs[0], rq), err(outs[1], rk), err(outs[2], rv)) <= TOL_F32


def test_backward_reports_fp16_value_range():
    """A gradient whose scaled value rows (f dO here) leave the fp16 range is reported by
    retnet_fp16_range_errors rather than returned as silent inf."""
    b, L, h, dk, dv = 1, 64, 2, 64, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 91, "bf16")
    do = si.randn((b, L, h, dv), 92, "bf16", std=3e6)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ws = torch.empty(rn.retnet_backward_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    assert rn.retnet_backward_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, g, ws.numel()) == 1
    outs = [torch.empty(b, L, h, d, device="cuda") for d in (dk, dk, dv)]
    rn.retnet_retention_backward(dev(q), dev(k), dev(v), do.cuda(), *outs, g, th, 0, FLAGS, workspace=ws)
    torch.cuda.synchronize()
    assert rn.retnet_fp16_range_errors(clear=True) > 0
