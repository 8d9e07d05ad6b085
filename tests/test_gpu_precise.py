"""Parity of the tensor-core kernel with split fp16 operands (RETNET_F_PRECISE) against the fp64
oracle ("阅读笔记：RetNet" §2.4 Chunkwise Recurrent Mode, with §2.3's xPos rotation and §三.3's
normalisations).

With split operands every value that the single-copy kernel rounds to fp16 once -- the scaled,
rotated q and k, the masked scores P and the fp16 state copy -- is carried as hi + lo
(hi = fp16(x), lo = fp16(x - hi)), and each product takes the hi*hi, lo*hi and hi*lo terms: the
operands keep about 22 significant bits, the accumulation is fp32, so the result is held to the
fp32 bar (max|err|/rms <= 1e-4) although the inputs are bf16.  Cases cover the in-kernel
converters (no workspace) and the conversion pre-pass (workspace, chunks of several 64-row
sub-blocks), d_k 64/128/256, carried state, positions and a one-token sequence.
"""
import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_F32, dev, err, require_gpu

pytestmark = pytest.mark.gpu
BASE = rn.F_XPOS | rn.F_SCALE_SQRT_D | rn.F_NORM_D


@pytest.fixture(autouse=True)
def _gpu(cuda_lib):
    require_gpu()
    rn.retnet_debug_wait_timeouts(clear=True)
    rn.retnet_fp16_range_errors(clear=True)
    yield
    assert rn.retnet_fp16_range_errors(clear=True) == 0  # no tensor-core operand left the fp16 range
    assert rn.retnet_debug_wait_timeouts(clear=True) == 0


CASES = [
    # dk, dv, B, L, pos0, with_state, workspace
    (64, 64, 64, 130, 0, False, True),
    (128, 128, 64, 300, 5, True, False),
    (128, 192, 128, 300, 0, False, True),
    (256, 128, 128, 129, 0, True, True),
    (256, 256, 256, 520, 1000, True, False),
    (256, 256, 256, 520, 0, False, True),
    (64, 256, 512, 513, 0, False, True),
    (256, 64, 64, 1, 3, True, True),
]


@pytest.mark.parametrize("dk,dv,B,L,pos0,with_state,workspace", CASES)
def test_precise_matches_oracle(dk, dv, B, L, pos0, with_state, workspace):
    b, h = 2, 3
    q, k, v = si.qkv(b, L, h, dk, dv, 1300 + dk + B, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 1301, std=0.05) if with_state else None
    flags = BASE | rn.F_PRECISE
    ref, Sref, _ = oracle.chunkwise(q, k, v, g, B, th, pos0, BASE, state_in=S0)
    assert rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, flags, B, g) == 1
    ws = None
    if workspace:
        ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    n = rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, flags, B, g, 0 if ws is None else ws.numel())
    # no sequence segments with split operands; the pre-pass only for chunks of several sub-blocks
    assert n == (2 if (workspace and B > 64) else 1), n
    o = torch.empty(b, L, h, dv, device="cuda")
    so = torch.empty(b, h, dk, dv, device="cuda")
    rn.retnet_retention_chunkwise_ws(dev(q), dev(k), dev(v), o, g, th, pos0, flags, B,
                                     None if S0 is None else dev(S0), so, workspace=ws)
    torch.cuda.synchronize()
    e, es = err(o, ref), err(so, Sref)
    print(f"precise dk={dk} dv={dv} B={B} L={L} launches={n}: out {e:.3e}, state {es:.3e}")
    assert e <= TOL_F32 and es <= TOL_F32


def test_precise_bf16_output():
    """bf16 output of the split-operand kernel: the output's own rounding (2^-8 relative) is
    then the only error left."""
    b, L, h, dk, dv, B = 1, 384, 2, 128, 128, 128
    q, k, v = si.qkv(b, L, h, dk, dv, 1400, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref, _, _ = oracle.chunkwise(q, k, v, g, B, th, 0, BASE)
    o = torch.empty(b, L, h, dv, device="cuda", dtype=torch.bfloat16)
    rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), o, g, th, 0, BASE | rn.F_PRECISE, B)
    torch.cuda.synchronize()
    got = o.double().cpu().numpy()
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    big = np.abs(ref) > 1e-3 * np.sqrt((ref ** 2).mean())
    assert rel[big].max() <= 2.0 ** -8 * 1.01, rel[big].max()
