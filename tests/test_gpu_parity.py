"""GPU parity through the C interface: every CUDA path against the fp64 oracle.

Bar: max|err|/rms(oracle) <= 1e-4 for fp32 inputs and <= 1e-2 for bf16 inputs, on the raw
retention output and on the MSR epilogue output.  Inputs are the seeded generators of
synth_inputs; both sides see identical values (bf16 inputs upcast exactly for the oracle).
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_BF16, TOL_F32, dev, err, err_bf16_out, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(cuda_lib):
    require_gpu()


def test_config1_tiny_all_modes_fp32():
    """b=1, h=2, d_k=d_v=16, L=64, B=16, fp32: parallel, chunkwise and step-by-step recurrent."""
    b, L, h, dk, dv, B = 1, 64, 2, 16, 16, 16
    q, k, v = si.qkv(b, L, h, dk, dv, 1, "f32")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    qd, kd, vd = dev(q), dev(k), dev(v)
    for flags in range(16):
        ref = oracle.parallel(q, k, v, g, th, 0, flags)
        o = torch.empty_like(vd)
        rn.retnet_retention_parallel(qd, kd, vd, o, g, th, 0, flags)
        assert err(o, ref) <= TOL_F32, ("parallel", flags, err(o, ref))
        o2 = torch.empty_like(vd)
        rn.retnet_retention_chunkwise(qd, kd, vd, o2, g, th, 0, flags, B)
        assert err(o2, ref) <= TOL_F32, ("chunkwise", flags, err(o2, ref))
        S = torch.zeros(b, h, dk, dv, device="cuda")
        z = torch.zeros(b, h, dk, device="cuda")
        outs = []
        for t in range(L):
            ot = torch.empty(b, h, dv, device="cuda")
            rn.retnet_retention_step(dev(q[:, t]), dev(k[:, t]), dev(v[:, t]), ot, S, g, th, t, flags, z)
            outs.append(ot)
        o3 = torch.stack(outs, dim=1)
        assert err(o3, ref) <= TOL_F32, ("step", flags, err(o3, ref))


@pytest.mark.parametrize("B", [1, 16, 33, 64, 100])
def test_chunkwise_fp32_ragged_with_state(B):
    b, L, h, dk, dv = 2, 70, 3, 8, 40
    q, k, v = si.qkv(b, L, h, dk, dv, 21, "f32")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 22, std=0.5)
    z0 = si.randn((b, h, dk), 23, "f32")
    pos0 = 5
    for flags in (oracle.F_ALL, oracle.F_XPOS | oracle.F_NORM_D, 0):
        ref, Sref, zref = oracle.recurrent(q, k, v, g, th, pos0, flags, S0, z0)
        o = torch.empty(b, L, h, dv, device="cuda")
        So = torch.empty(b, h, dk, dv, device="cuda")
        zo = torch.empty(b, h, dk, device="cuda")
        rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), o, g, th, pos0, flags, B, dev(S0), So, dev(z0), zo)
        assert err(o, ref) <= TOL_F32, (flags, err(o, ref))
        assert err(So, Sref) <= TOL_F32
        if flags & oracle.F_NORM_R:
            assert err(zo, zref) <= TOL_F32


def test_chunkwise_state_aliasing_in_place():
    b, L, h, dk, dv = 1, 50, 2, 16, 32
    q, k, v = si.qkv(b, L, h, dk, dv, 24, "f32")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 25, std=0.3)
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, 0, oracle.F_ALL, S0, None)
    S = dev(S0.clone())
    o = torch.empty(b, L, h, dv, device="cuda")
    rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), o, g, th, 0, oracle.F_ALL, 16, S, S)
    assert err(o, ref) <= TOL_F32
    assert err(S, Sref) <= TOL_F32


def test_chunkwise_bf16_inputs_cuda_core_shapes():
    """bf16 inputs on shapes the tensor-core kernel does not take (d_k=48): fp32 CUDA-core path."""
    b, L, h, dk, dv, B = 2, 130, 2, 48, 24, 32
    q, k, v = si.qkv(b, L, h, dk, dv, 26, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref = oracle.parallel(q, k, v, g, th, 0, oracle.F_ALL)
    o = torch.empty(b, L, h, dv, device="cuda")
    rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), o, g, th, 0, oracle.F_ALL, B)
    assert err(o, ref) <= TOL_F32  # exact inputs, fp32 arithmetic
    ob = torch.empty(b, L, h, dv, device="cuda", dtype=torch.bfloat16)
    rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), ob, g, th, 0, oracle.F_ALL, B)
    assert err_bf16_out(ob, ref) <= TOL_BF16


@pytest.mark.parametrize("dv", [48, 42, 520])
def test_step_matches_recurrent_oracle(dv):
    b, h, dk, steps = 3, 4, 32, 12
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 30, std=0.01)
    z0 = si.randn((b, h, dk), 31, "f32")
    toks = [si.decode_token(b, h, dk, dv, 32, t) for t in range(steps)]
    q = torch.stack([t[0] for t in toks], 1)
    k = torch.stack([t[1] for t in toks], 1)
    v = torch.stack([t[2] for t in toks], 1)
    pos0 = 1000
    for flags in (oracle.F_ALL, oracle.F_XPOS | oracle.F_SCALE_SQRT_D | oracle.F_NORM_D):
        ref, Sref, zref = oracle.recurrent(q, k, v, g, th, pos0, flags, S0, z0)
        S, z = dev(S0.clone()), dev(z0.clone())
        outs = []
        for t in range(steps):
            ot = torch.empty(b, h, dv, device="cuda")
            rn.retnet_retention_step(dev(toks[t][0]), dev(toks[t][1]), dev(toks[t][2]), ot, S, g, th, pos0 + t,
                                     flags, z)
            outs.append(ot)
        o = torch.stack(outs, 1)
        assert err(o, ref) <= TOL_F32, (flags, err(o, ref))
        assert err(S, Sref) <= TOL_F32
        if flags & oracle.F_NORM_R:
            assert err(z, zref) <= TOL_F32


def test_prefill_then_decode_equals_parallel():
    b, L, P, h, dk, dv = 2, 90, 67, 2, 16, 32
    q, k, v = si.qkv(b, L, h, dk, dv, 33, "f32")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref = oracle.parallel(q, k, v, g, th, 0, oracle.F_ALL)
    o1 = torch.empty(b, P, h, dv, device="cuda")
    S = torch.empty(b, h, dk, dv, device="cuda")
    z = torch.empty(b, h, dk, device="cuda")
    rn.retnet_retention_chunkwise(dev(q[:, :P]), dev(k[:, :P]), dev(v[:, :P]), o1, g, th, 0, oracle.F_ALL, 16,
                                  None, S, None, z)
    outs = [o1]
    for t in range(P, L):
        ot = torch.empty(b, 1, h, dv, device="cuda")
        rn.retnet_retention_step(dev(q[:, t]), dev(k[:, t]), dev(v[:, t]), ot.view(b, h, dv), S, g, th, t,
                                 oracle.F_ALL, z)
        outs.append(ot)
    assert err(torch.cat(outs, 1), ref) <= TOL_F32


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [8, 64, 256, 1024])
def test_msr_epilogue(dtype, dv):
    tokens, h = 37, 3
    y = si.randn((tokens, h * dv), 40, dtype) * 2
    y = (y.float() + 0.3).to(y.dtype)
    gt = si.randn((tokens, h * dv), 41, dtype)
    ref = oracle.msr_epilogue(y, gt, h, eps=1e-5)
    out = torch.empty(tokens, h * dv, device="cuda", dtype=torch.float32)
    rn.retnet_msr_epilogue(dev(y), dev(gt), out, h, 1e-5)
    assert err(out, ref) <= TOL_F32
    outb = torch.empty(tokens, h * dv, device="cuda", dtype=torch.bfloat16)
    rn.retnet_msr_epilogue(dev(y), dev(gt), outb, h, 1e-5)
    assert err_bf16_out(outb, ref) <= TOL_BF16


def test_causality_bitwise():
    b, L, h, dk, dv, m = 1, 96, 2, 16, 32, 57
    q, k, v = si.qkv(b, L, h, dk, dv, 42, "f32")
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[:, m:] += 3; k2[:, m:] -= 1; v2[:, m:] *= -2
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    for fn in ("parallel", "chunkwise"):
        outs = []
        for (a, bb, c) in ((q, k, v), (q2, k2, v2)):
            o = torch.empty(b, L, h, dv, device="cuda")
            if fn == "parallel":
                rn.retnet_retention_parallel(dev(a), dev(bb), dev(c), o, g, th, 0, oracle.F_ALL)
            else:
                rn.retnet_retention_chunkwise(dev(a), dev(bb), dev(c), o, g, th, 0, oracle.F_ALL, 32)
            outs.append(o.cpu())
        assert torch.equal(outs[0][:, :m], outs[1][:, :m])
        assert not torch.equal(outs[0][:, m:], outs[1][:, m:])


def test_degenerate_sizes():
    g = si.gamma_schedule(1)
    # seqlen 0: state passes through, z too
    S0 = dev(si.decode_state(1, 1, 4, 8, 50, std=1.0))
    z0 = dev(si.randn((1, 1, 4), 51, "f32"))
    So = torch.empty_like(S0)
    zo = torch.empty_like(z0)
    e = torch.empty(1, 0, 1, 4, device="cuda")
    ev = torch.empty(1, 0, 1, 8, device="cuda")
    nox = oracle.F_SCALE_SQRT_D | oracle.F_NORM_D | oracle.F_NORM_R
    rn.retnet_retention_chunkwise(e, e, ev, ev.clone(), g, None, 0, nox, 16, S0, So, z0, zo)
    torch.cuda.synchronize()
    assert torch.equal(So, S0) and torch.equal(zo, z0)
    # seqlen 1, d_k = d_v = 1, no rotation
    q, k, v = si.qkv(1, 1, 1, 1, 1, 52, "f32")
    ref = oracle.parallel(q, k, v, g, None, 0, oracle.F_SCALE_SQRT_D | oracle.F_NORM_D | oracle.F_NORM_R)
    o = torch.empty(1, 1, 1, 1, device="cuda")
    rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), o, g, None, 0,
                                  oracle.F_SCALE_SQRT_D | oracle.F_NORM_D | oracle.F_NORM_R, 64)
    assert err(o, ref) <= TOL_F32
    # closed form on the GPU: d = 1, q = k = v = 1  ->  o_n = (1 - gamma^n) / (1 - gamma)
    L = 200
    ones = torch.ones(1, L, 1, 1, device="cuda")
    o = torch.empty_like(ones)
    gam = np.array([0.96875], np.float32)
    rn.retnet_retention_chunkwise(ones, ones, ones, o, gam, None, 0, 0, 64)
    n = np.arange(1, L + 1)
    geo = -np.expm1(n * np.log1p(-(1 - 0.96875))) / (1 - 0.96875)
    np.testing.assert_allclose(o.cpu().double().numpy()[0, :, 0, 0], geo, rtol=2e-6)


@pytest.mark.parametrize("b,L,h,dk,dv,flags,pos0", [
    (2, 64, 2, 64, 64, oracle.F_XPOS | oracle.F_SCALE_SQRT_D | oracle.F_NORM_D, 0),
    (1, 200, 3, 128, 128, oracle.F_XPOS | oracle.F_SCALE_SQRT_D | oracle.F_NORM_D, 9),
    (2, 512, 2, 128, 64, oracle.F_SCALE_SQRT_D, 0),
    (1, 1, 2, 256, 64, oracle.F_XPOS | oracle.F_NORM_D, 3),
    (1, 700, 2, 64, 128, oracle.F_XPOS | oracle.F_SCALE_SQRT_D | oracle.F_NORM_D, 0)])
def test_parallel_bf16_on_tensor_cores(b, L, h, dk, dv, flags, pos0):
    """bf16 parallel form (§2.3) on the tensor-core kernel: one masked tile of the whole
    sequence up to 512 tokens, 512-token chunks beyond; single fp16 operands at the bf16 bar,
    split operands (RETNET_F_PRECISE) at the fp32 bar."""
    q, k, v = si.qkv(b, L, h, dk, dv, 1700 + L, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref = oracle.parallel(q, k, v, g, th, pos0, flags)
    for fl, tol in ((flags, TOL_BF16), (flags | rn.F_PRECISE, TOL_F32)):
        o = torch.empty(b, L, h, dv, device="cuda")
        rn.retnet_retention_parallel(dev(q), dev(k), dev(v), o, g, th, pos0, fl)
        torch.cuda.synchronize()
        e = err(o, ref)
        print(f"parallel bf16 L={L} dk={dk} flags={fl}: {e:.3e}")
        assert e <= tol
    assert rn.retnet_debug_wait_timeouts(clear=True) == 0
