"""Parity of the fused MSR kernel (chunkwise retention + GroupNorm + swish gate in one
tensor-core kernel, the d_v slices of a head in one thread-block cluster) against the fp64
oracle: oracle.msr_epilogue of the oracle's retention output.

Bar: the plain max|err|/rms(out) <= 1e-2 of bf16 inputs on the post-epilogue output (net of a
bf16 output's own rounding).  The GroupNorm divides each row by its own deviation, so a row of
few tokens whose scores nearly cancel magnifies the operand rounding of the retention output;
the fused kernel therefore always runs with split fp16 operands (hi + lo, about 22 significant
bits), which keeps the post-epilogue error near the fp32 level.  gpu_util.err_msr (the
retention bar carried through the normalisation) is printed beside it.
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_BF16, dev, err, err_bf16_out, err_msr, require_gpu

pytestmark = pytest.mark.gpu
FLAGS = rn.F_XPOS | rn.F_SCALE_SQRT_D | rn.F_NORM_D
EPS = 1e-5


@pytest.fixture(autouse=True)
def _gpu(cuda_lib):
    require_gpu()
    rn.retnet_debug_wait_timeouts(clear=True)
    rn.retnet_fp16_range_errors(clear=True)
    yield
    assert rn.retnet_fp16_range_errors(clear=True) == 0  # no tensor-core operand left the fp16 range
    assert rn.retnet_debug_wait_timeouts(clear=True) == 0


def gate(b, L, h, dv, seed):
    return si.randn((b, L, h, dv), seed, "bf16")


def fused(q, k, v, gt, g, th, B, pos0=0, state_in=None, want_state=False, out_dtype=torch.float32,
          workspace=True):
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    ws = None
    if workspace:
        ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    n = rn.retnet_msr_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS, B, g,
                                         0 if ws is None else ws.numel())
    assert n in (1, 2), n
    out = torch.empty(b, L, h, dv, device="cuda", dtype=out_dtype)
    so = torch.empty(b, h, dk, dv, device="cuda") if want_state else None
    rn.retnet_msr_chunkwise(dev(q), dev(k), dev(v), dev(gt), out, g, th, pos0, FLAGS, B, EPS,
                            None if state_in is None else dev(state_in), so, ws)
    torch.cuda.synchronize()
    return out, so, n


def reference(q, k, v, gt, g, th, B, pos0=0, state_in=None):
    y, S, _ = oracle.chunkwise(q, k, v, g, B, th, pos0, FLAGS, state_in=state_in)
    h = q.shape[2]
    return oracle.msr_epilogue(y, gt, h, eps=EPS), y, S


@pytest.mark.parametrize("dk,dv,B,L", [(64, 64, 64, 130), (128, 128, 64, 300), (128, 192, 128, 300),
                                       (256, 256, 64, 200), (256, 256, 256, 520), (64, 256, 512, 513),
                                       (128, 128, 256, 257), (256, 128, 128, 129), (128, 64, 64, 1)])
@pytest.mark.parametrize("workspace", [True, False])
def test_fused_msr_matches_oracle(dk, dv, B, L, workspace):
    b, h = 2, 3
    q, k, v = si.qkv(b, L, h, dk, dv, 300 + dk + B, "bf16")
    gt = gate(b, L, h, dv, 7000 + dv)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref, y, Sref = reference(q, k, v, gt, g, th, B)
    out, so, n = fused(q, k, v, gt, g, th, B, want_state=True, workspace=workspace)
    e = err_msr(out, ref, y, gt, h, EPS)
    e_out = err(out, ref)
    print(f"dk={dk} dv={dv} B={B} L={L} ws={workspace} launches={n}: msr err {e:.3e}, max|err|/rms {e_out:.3e}")
    assert e_out <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


def test_fused_msr_bf16_out_state_in_pos0():
    """bf16 output, a carried-in state and a large start position, against the same bar."""
    b, L, h, dk, dv, B = 2, 333, 4, 256, 256, 256
    q, k, v = si.qkv(b, L, h, dk, dv, 321, "bf16")
    gt = gate(b, L, h, dv, 322)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 323, std=0.05)
    pos0 = (1 << 20) + 77
    ref, y, Sref = reference(q, k, v, gt, g, th, B, pos0=pos0, state_in=S0)
    out, so, _ = fused(q, k, v, gt, g, th, B, pos0=pos0, state_in=S0, want_state=True, out_dtype=torch.bfloat16)
    e = err_bf16_out(out, ref)
    print(f"bf16 out, state in, pos0 {pos0}: max|err|/rms net of bf16 rounding {e:.3e}")
    assert e <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


def test_fused_no_worse_than_two_kernel_path():
    """The fused kernel and chunkwise (split operands) + retnet_msr_epilogue (fp32 between them)
    against the oracle: fusing the epilogue loses no accuracy."""
    b, L, h, dk, dv, B = 2, 700, 4, 128, 256, 128
    q, k, v = si.qkv(b, L, h, dk, dv, 401, "bf16")
    gt = gate(b, L, h, dv, 402)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref, y_ref, _ = reference(q, k, v, gt, g, th, B)
    out, _, _ = fused(q, k, v, gt, g, th, B)
    y = torch.empty(b, L, h, dv, device="cuda")
    rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), y, g, th, 0, FLAGS | rn.F_PRECISE, B)
    two = torch.empty_like(y)
    rn.retnet_msr_epilogue(y, dev(gt).float(), two, h, EPS)  # y and g share one dtype
    torch.cuda.synchronize()
    e_fused, e_two = err(out, ref), err(two, ref)
    print(f"fused {e_fused:.3e}, two kernels {e_two:.3e}")
    assert e_fused <= TOL_BF16 and e_two <= TOL_BF16
    assert e_fused <= 1.5 * e_two + 1e-4


@pytest.mark.parametrize("dk,dv,B,L", [(128, 128, 64, 300), (256, 256, 256, 520)])
def test_fused_msr_with_norm_r(dk, dv, B, L):
    """R~ (§三.3) before the GroupNorm: the key-sum pass writes the row factors into the
    workspace, the fused kernel folds them into its row scale (the GroupNorm then sees each row
    divided by max(|row sum|, 1), which changes the result only through eps)."""
    b, h = 2, 3
    q, k, v = si.qkv(b, L, h, dk, dv, 500 + dk + B, "bf16")
    q = (q.float() + 0.5).to(q.dtype)  # most row sums exceed 1: the normalisation is active
    k = (k.float() + 0.5).to(k.dtype)
    gt = gate(b, L, h, dv, 501)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    flags = FLAGS | rn.F_NORM_R
    y, _, _ = oracle.chunkwise(q, k, v, g, B, th, 0, flags)
    ref = oracle.msr_epilogue(y, gt, h, eps=EPS)
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    n = rn.retnet_msr_chunkwise_launches((b, L, h, dk), dv, rn.BF16, flags, B, g, ws.numel())
    assert n >= 2, n  # the key-sum pass, then the fused kernel (after the conversion pre-pass)
    out = torch.empty(b, L, h, dv, device="cuda")
    rn.retnet_msr_chunkwise(dev(q), dev(k), dev(v), dev(gt), out, g, th, 0, flags, B, EPS, workspace=ws)
    torch.cuda.synchronize()
    e = err(out, ref)
    print(f"fused MSR with R~ dk={dk} dv={dv} B={B} L={L} launches={n}: max|err|/rms {e:.3e}")
    assert e <= TOL_BF16


def test_fused_unsupported_shapes_are_rejected():
    b, L, h, dk = 1, 64, 2, 128
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    # d_v = 320 needs five CTAs a cluster; R~ needs a workspace for its row factors
    for dv, flags in ((320, FLAGS), (128, FLAGS | rn.F_NORM_R)):
        assert rn.retnet_msr_chunkwise_launches((b, L, h, dk), dv, rn.BF16, flags, 64, g) == -5
        q, k, v = si.qkv(b, L, h, dk, dv, 5, "bf16")
        gt = gate(b, L, h, dv, 6)
        out = torch.full((b, L, h, dv), 7.0, device="cuda")
        with pytest.raises(RuntimeError, match="UNSUPPORTED"):
            rn.retnet_msr_chunkwise(dev(q), dev(k), dev(v), dev(gt), out, g, th, 0, flags, 64, EPS)
        assert bool((out == 7.0).all())  # nothing was launched
