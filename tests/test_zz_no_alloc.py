"""The allocation-free chunkwise entry point (segment states in the library's static device
scratch) against the workspace entry point it mirrors.

In its own file, named to be collected last: the scratch is process-wide device state, and the
test must pass alone as well as after every other test has run kernels in the same process.
"""
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import synth_inputs as si
from gpu_util import TOL_BF16, err, require_gpu

pytestmark = pytest.mark.gpu
FLAGS = rn.F_XPOS | rn.F_SCALE_SQRT_D | rn.F_NORM_D


@pytest.fixture(autouse=True)
def _gpu(cuda_lib):
    require_gpu()
    rn.retnet_debug_wait_timeouts(clear=True)
    yield
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
