"""The allocation-free chunkwise entry point (segment states in the library's static device
scratch) against the workspace entry point it mirrors.

In its own file, named to be collected last: the scratch is process-wide device state, and the
test must pass alone as well as after every other test has run kernels in the same process.
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_BF16, TOL_F32, err, require_gpu

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


@pytest.mark.parametrize("b,L,h,dk,dv,B", [(8, 2048, 8, 128, 128, 64), (1, 1100, 2, 256, 64, 128),
                                           (2, 700, 3, 64, 128, 64)])
def test_static_scratch_matches_workspace_call(b, L, h, dk, dv, B):
    """Two calls in a row with different inputs: each bit-equal to retnet_retention_chunkwise_ws
    given a workspace of the scratch's size (same plan, same kernels), and within the bf16 bar
    of the plain call."""
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    assert rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, B, g) == 1
    ws = torch.empty(rn.STATIC_SCRATCH_BYTES, dtype=torch.uint8, device="cuda")
    for call in range(2):
        q, k, v = (x.cuda() for x in si.qkv(b, L, h, dk, dv, 300 + 10 * call + dk, "bf16"))
        s0 = si.decode_state(b, h, dk, dv, 301 + call, std=0.2).cuda()
        o_static, o_ws, o_plain = (torch.empty(b, L, h, dv, device="cuda") for _ in range(3))
        s_static, s_ws = (torch.empty(b, h, dk, dv, device="cuda") for _ in range(2))
        rn.retnet_retention_chunkwise_static(q, k, v, o_static, g, th, 17, FLAGS, B, s0, s_static)
        rn.retnet_retention_chunkwise_ws(q, k, v, o_ws, g, th, 17, FLAGS, B, s0, s_ws, workspace=ws)
        rn.retnet_retention_chunkwise(q, k, v, o_plain, g, th, 17, FLAGS, B, s0)
        torch.cuda.synchronize()
        assert torch.equal(o_static, o_ws), call
        assert torch.equal(s_static, s_ws), call
        assert err(o_static, o_plain.cpu().double().numpy()) <= TOL_BF16


@pytest.mark.parametrize("b,L,h,dk,dv,B,fits", [(2, 700, 3, 64, 128, 64, True), (4, 130, 64, 256, 64, 64, False)])
def test_static_scratch_with_norm_r(b, L, h, dk, dv, B, fits):
    """R~ through the static scratch.  Where its row factors and key-sum values fit the 16 MiB,
    they take the front of the scratch and R~ runs on the tensor-core kernel (key-sum pass +
    split operands); where they do not (64 heads of d_k 256: 16 MiB of key-sum values alone),
    the call runs on the CUDA-core kernel.  Both are checked against the workspace call given a
    workspace of the scratch's size (same plan, same kernels: bit-equal) and against the oracle
    on two heads."""
    g = np.linspace(0.9, 0.999, h).astype(np.float32)
    th = si.theta_schedule(dk)
    flags = FLAGS | rn.F_NORM_R
    n = rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, flags, B, g, rn.STATIC_SCRATCH_BYTES)
    assert (n >= 2) if fits else (n == 1), n
    ws = torch.empty(rn.STATIC_SCRATCH_BYTES, dtype=torch.uint8, device="cuda")
    q, k, v = si.qkv(b, L, h, dk, dv, 350 + dk, "bf16")
    q = (q.float() + 0.3).to(q.dtype)  # most row sums exceed 1: the normalisation is active
    k = (k.float() + 0.3).to(k.dtype)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    for call in range(2):
        o_static, o_ws = (torch.empty(b, L, h, dv, device="cuda") for _ in range(2))
        z_static, z_ws = (torch.empty(b, h, dk, device="cuda") for _ in range(2))
        rn.retnet_retention_chunkwise_static(qd, kd, vd, o_static, g, th, 5, flags, B, z_out=z_static)
        rn.retnet_retention_chunkwise_ws(qd, kd, vd, o_ws, g, th, 5, flags, B, z_out=z_ws, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(o_static, o_ws), call
        assert torch.equal(z_static, z_ws), call
    for hh in (0, h - 1):
        sl = (slice(None), slice(None), slice(hh, hh + 1))
        ref, _, zref = oracle.recurrent(q[sl], k[sl], v[sl], g[hh:hh + 1], th, 5, flags)
        e = err(o_static[sl], ref)
        print(f"static R~ b={b} L={L} h={h} dk={dk} head {hh} launches={n}: {e:.3e}")
        assert e <= (TOL_BF16 if fits else TOL_F32)
        assert err(z_static[:, hh], zref[:, 0]) <= TOL_F32
