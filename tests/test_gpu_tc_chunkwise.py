"""Parity of the tcgen05 tensor-core chunkwise kernel (bf16 inputs) against the fp64 oracle.

Bar: max|err|/rms(oracle) <= 1e-2 on the raw output (the bf16-input tolerance); the
state hand-off is held to the same bar.  Every case asserts first that the call takes
the tensor-core kernel, and last that no bounded wait inside it gave up.
"""
import os

import numpy as np
import pytest
import torch

import linear_attention_sequence_chunkwise_b200 as rn
import oracle
import synth_inputs as si
from gpu_util import TOL_BF16, TOL_F32, dev, err, err_bf16_out, require_gpu

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


def run_tc(q, k, v, g, th, B, flags=FLAGS, pos0=0, state_in=None, want_state=False, out_dtype=torch.float32):
    import os
    b, L, h, dk = q.shape
    dv = v.shape[-1]
    if os.environ.get("RETNET_TC_KERNEL") == "serial" and B > 128:
        pytest.skip("the serial tensor-core kernel takes chunks of at most 128 tokens")
    assert rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, flags, B, g) == 1
    o = torch.empty(b, L, h, dv, device="cuda", dtype=out_dtype)
    so = torch.empty(b, h, dk, dv, device="cuda") if want_state else None
    rn.retnet_retention_chunkwise(dev(q), dev(k), dev(v), o, g, th, pos0, flags, B,
                                  None if state_in is None else dev(state_in), so)
    torch.cuda.synchronize()
    return o, so


@pytest.mark.parametrize("dk,dv,B,L", [(128, 128, 64, 300), (128, 192, 128, 300), (64, 64, 64, 130),
                                       (64, 128, 128, 257), (256, 128, 64, 200), (256, 64, 128, 129),
                                       (128, 64, 64, 1), (128, 64, 64, 64), (128, 64, 128, 128),
                                       (128, 128, 256, 600), (128, 64, 512, 1100), (64, 64, 512, 513),
                                       (256, 64, 256, 520), (256, 128, 512, 700), (128, 64, 256, 100),
                                       (256, 64, 128, 300), (64, 128, 256, 257)])
def test_tc_matches_oracle(dk, dv, B, L):
    b, h = 2, 3
    q, k, v = si.qkv(b, L, h, dk, dv, 60 + dk + B, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, 0, FLAGS)
    o, so = run_tc(q, k, v, g, th, B, want_state=True)
    e = err(o, ref)
    print(f"dk={dk} dv={dv} B={B} L={L}: max|err|/rms = {e:.3e}")
    assert e <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


@pytest.mark.parametrize("b,h,dk,dv,L", [(10, 16, 128, 128, 200), (5, 16, 64, 256, 130)])
def test_tc_wide_slices(b, h, dk, dv, L):
    """Enough (batch, head) pairs for the 128-column d_v slices (chunk 64): same bar."""
    B = 64
    q, k, v = si.qkv(b, L, h, dk, dv, 80 + dk, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, 0, FLAGS)
    o, so = run_tc(q, k, v, g, th, B, want_state=True)
    e = err(o, ref)
    print(f"wide slices b={b} h={h} dk={dk} dv={dv}: max|err|/rms = {e:.3e}")
    assert e <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


@pytest.mark.parametrize("dk,dv,B,L,with_state", [(128, 128, 64, 64 * 9 + 5, False), (128, 64, 64, 64 * 17, True),
                                                  (256, 64, 128, 128 * 8 + 30, True), (64, 128, 256, 256 * 8, False),
                                                  (128, 128, 64, 64 * 33 + 1, True)])
def test_tc_sequence_segments(dk, dv, B, L, with_state):
    """Few (batch, head) pairs and many chunks: the sequence is split over CTAs that replay
    the state over the earlier chunks.  Outputs and the final state against the oracle."""
    b, h = 1, 2
    q, k, v = si.qkv(b, L, h, dk, dv, 90 + dk + B, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 91, std=0.3) if with_state else None
    pos0 = 321 if with_state else 0
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS, S0)
    o, so = run_tc(q, k, v, g, th, B, pos0=pos0, state_in=S0, want_state=True)
    e = err(o, ref)
    print(f"segments dk={dk} dv={dv} B={B} L={L}: max|err|/rms = {e:.3e}")
    assert e <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


@pytest.mark.parametrize("dk,dv,B,L,with_state", [(128, 128, 64, 64 * 9 + 5, True), (128, 64, 64, 64 * 17, False),
                                                  (256, 64, 128, 128 * 8 + 30, True), (64, 128, 256, 256 * 8, True),
                                                  (128, 128, 64, 64 * 33 + 1, False)])
def test_tc_two_pass_segments(dk, dv, B, L, with_state):
    """The workspace form: segment states from a pre-pass launch, every segment's outputs from
    state_in carried over the earlier ones.  Against the oracle, and the workspace sizes that
    allow 2, 3 or 4 segments give the same bar."""
    b, h = 1, 2
    q, k, v = si.qkv(b, L, h, dk, dv, 95 + dk + B, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 96, std=0.3) if with_state else None
    pos0 = 555 if with_state else 0
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS, S0)
    full = rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv))
    for nbytes in (full // 3, 2 * full // 3, full):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o = torch.empty(b, L, h, dv, device="cuda")
        so = torch.empty(b, h, dk, dv, device="cuda")
        rn.retnet_retention_chunkwise_ws(dev(q), dev(k), dev(v), o, g, th, pos0, FLAGS, B,
                                         None if S0 is None else dev(S0), so, workspace=ws)
        torch.cuda.synchronize()
        e = err(o, ref)
        print(f"two-pass dk={dk} dv={dv} B={B} L={L} ws={nbytes}: max|err|/rms = {e:.3e}")
        assert e <= TOL_BF16
        assert err(so, Sref) <= TOL_BF16


@pytest.mark.parametrize("dk,dv,B,L,with_state", [(128, 64, 256, 600, True), (256, 64, 128, 333, False),
                                                  (64, 64, 512, 700, True), (256, 128, 512, 520, True)])
def test_tc_preconverted(dk, dv, B, L, with_state):
    """Chunks of several sub-blocks with a workspace that holds the fp16 copies: a conversion
    pre-pass, then the kernel without converters (for d_k 256 the P pass between them).
    Against the oracle (outputs and state)."""
    b, h = 8, 10  # >= 75 d_v-slice CTAs: no sequence segments
    q, k, v = si.qkv(b, L, h, dk, dv, 110 + dk + B, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 111, std=0.3) if with_state else None
    pos0 = 4321 if with_state else 0
    nbytes = rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv))
    assert rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS, B, g, nbytes) == (3 if dk == 256 else 2)
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS, S0)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o = torch.empty(b, L, h, dv, device="cuda")
    so = torch.empty(b, h, dk, dv, device="cuda")
    rn.retnet_retention_chunkwise_ws(dev(q), dev(k), dev(v), o, g, th, pos0, FLAGS, B,
                                     None if S0 is None else dev(S0), so, workspace=ws)
    torch.cuda.synchronize()
    e = err(o, ref)
    print(f"pre-converted dk={dk} dv={dv} B={B} L={L}: max|err|/rms = {e:.3e}")
    assert e <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


@pytest.mark.parametrize("case", ["dv1024", "pos0_large", "one_token_ws", "gamma_near_one"])
def test_tc_edge_cases(case):
    """Widest value dimension (16 slices), an xPos position near 2^26 (where an fp32 angle is
    off by radians: the kernel reduces p * theta in fp64; the oracle's D~ prefix is a plain
    O(pos0) sum, which bounds how far this can go),
    a single-token call through the workspace form, and heads up to gamma = 1 - 2^-24 (the
    largest fp32 below 1)."""
    b, L, h, dk, dv, B, pos0 = 1, 300, 2, 128, 64, 64, 0
    if case == "dv1024":
        dv = 1024
    elif case == "pos0_large":
        pos0 = (1 << 26) + 12345
    elif case == "one_token_ws":
        L = 1
    elif case == "gamma_near_one":
        h, L = 20, 150
    q, k, v = si.qkv(b, L, h, dk, dv, 120, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    assert rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, B, g) == 1
    S0 = si.decode_state(b, h, dk, dv, 121, std=0.2)
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS, S0)
    o = torch.empty(b, L, h, dv, device="cuda")
    so = torch.empty(b, h, dk, dv, device="cuda")
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    rn.retnet_retention_chunkwise_ws(dev(q), dev(k), dev(v), o, g, th, pos0, FLAGS, B, dev(S0), so, workspace=ws)
    torch.cuda.synchronize()
    e = err(o, ref)
    print(f"edge {case}: max|err|/rms = {e:.3e}")
    assert e <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


def test_tc_launch_count():
    """The launch-count query follows the plan: two launches only for the workspace form with
    segments (few (batch, head) pairs), one otherwise."""
    g = si.gamma_schedule(8)
    ws = rn.retnet_chunkwise_workspace_size((8, 2048, 8, 128, 128))
    assert rn.retnet_chunkwise_launches((8, 2048, 8, 128), 128, rn.BF16, FLAGS, 64, g, ws) == 2
    assert rn.retnet_chunkwise_launches((8, 2048, 8, 128), 128, rn.BF16, FLAGS, 64, g, 0) == 1
    assert rn.retnet_chunkwise_launches((32, 2048, 8, 128), 128, rn.BF16, FLAGS, 64, g, 10 ** 9) == 1
    assert rn.retnet_chunkwise_launches((8, 0, 8, 128), 128, rn.BF16, FLAGS, 64, g, ws) == 0
    assert rn.retnet_chunkwise_launches((8, 2048, 8, 128), 128, rn.F32, FLAGS, 64, g, ws) == 1


def test_tc_two_pass_full_workload():
    """b8/L2048/h8/d128/chunk 64 through the workspace form: within the bf16 bar of the plain
    call's output (the two round the segment-boundary state differently) and of the oracle on
    sampled (batch, head) pairs."""
    b, L, h, dk, dv, B = 8, 2048, 8, 128, 128, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 97, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    qd, kd, vd = dev(q), dev(k), dev(v)
    o1 = torch.empty(b, L, h, dv, device="cuda")
    o2 = torch.empty_like(o1)
    rn.retnet_retention_chunkwise(qd, kd, vd, o1, g, th, 0, FLAGS, B)
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    rn.retnet_retention_chunkwise_ws(qd, kd, vd, o2, g, th, 0, FLAGS, B, workspace=ws)
    torch.cuda.synchronize()
    rms = o1.float().pow(2).mean().sqrt().item()
    assert (o1 - o2).abs().max().item() / rms <= TOL_BF16
    for bb, hh in ((0, 0), (7, 7)):
        sl = lambda x: x[bb:bb + 1, :, hh:hh + 1]
        ref = oracle.recurrent(sl(q).contiguous(), sl(k).contiguous(), sl(v).contiguous(), g[hh:hh + 1], th, 0,
                               FLAGS)[0]
        assert err(sl(o2.cpu()).contiguous(), ref) <= TOL_BF16


@pytest.mark.parametrize("flags", [0, rn.F_XPOS, rn.F_SCALE_SQRT_D, rn.F_NORM_D, FLAGS])
def test_tc_flag_combinations(flags):
    b, L, h, dk, dv, B = 1, 200, 4, 128, 64, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 70, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref = oracle.parallel(q, k, v, g, th, 0, flags)
    o, _ = run_tc(q, k, v, g, th, B, flags=flags)
    assert err(o, ref) <= TOL_BF16


@pytest.mark.parametrize("dk,B", [(128, 64), (128, 256), (256, 512)])
def test_tc_state_in_and_position(dk, B):
    b, L, h, dv = 2, 590, 2, 128
    q, k, v = si.qkv(b, L, h, dk, dv, 71, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 72, std=0.3)
    pos0 = 777
    ref, Sref, _ = oracle.recurrent(q, k, v, g, th, pos0, FLAGS, S0)
    o, so = run_tc(q, k, v, g, th, B, pos0=pos0, state_in=S0, want_state=True)
    assert err(o, ref) <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16


def test_tc_bf16_output():
    b, L, h, dk, dv, B = 2, 256, 2, 128, 128, 128
    q, k, v = si.qkv(b, L, h, dk, dv, 73, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref = oracle.parallel(q, k, v, g, th, 0, FLAGS)
    o, _ = run_tc(q, k, v, g, th, B, out_dtype=torch.bfloat16)
    assert err_bf16_out(o, ref) <= TOL_BF16


def test_tc_causality_bitwise():
    b, L, h, dk, dv, B, m = 1, 300, 2, 128, 64, 64, 150
    q, k, v = si.qkv(b, L, h, dk, dv, 74, "bf16")
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[:, m:] = -q2[:, m:]; k2[:, m:] *= 2; v2[:, m:] += 1
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    o1, _ = run_tc(q, k, v, g, th, B)
    o2, _ = run_tc(q2, k2, v2, g, th, B)
    assert torch.equal(o1[:, :m].cpu(), o2[:, :m].cpu())
    assert not torch.equal(o1[:, m:].cpu(), o2[:, m:].cpu())


def test_tc_prefill_then_decode_matches_parallel():
    b, L, P, h, dk, dv = 2, 160, 128, 2, 128, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 75, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ref = oracle.parallel(q, k, v, g, th, 0, FLAGS)
    o1, S = run_tc(q[:, :P].contiguous(), k[:, :P].contiguous(), v[:, :P].contiguous(), g, th, 64,
                   want_state=True)
    outs = [o1]
    for t in range(P, L):
        ot = torch.empty(b, 1, h, dv, device="cuda")
        rn.retnet_retention_step(dev(q[:, t]), dev(k[:, t]), dev(v[:, t]), ot.view(b, h, dv), S, g, th, t, FLAGS)
        outs.append(ot)
    assert err(torch.cat(outs, 1), ref) <= TOL_BF16


def test_tc_chunkwise_workload_full_size():
    """The benchmark workload in full: batch 8, h 8, d_k = d_v = 128, L 2048, B 64, every output."""
    b, L, h, dk, dv, B = 8, 2048, 8, 128, 128, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 2, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    o, _ = run_tc(q, k, v, g, th, B)
    ref, _, _ = oracle.recurrent(q, k, v, g, th, 0, FLAGS)
    e = err(o, ref)
    print(f"full workload max|err|/rms = {e:.3e}")
    assert e <= TOL_BF16


def test_serial_kernel_variant_in_subprocess():
    """RETNET_TC_KERNEL=serial routes every tensor-core call to the serial kernel; it must
    pass the same parity cases as the pipelined kernel."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, RETNET_TC_KERNEL="serial")
    here = os.path.dirname(os.path.abspath(__file__))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu",
                        "-k", "tc_matches_oracle or tc_state_in or tc_flag", os.path.join(here, "test_gpu_tc_chunkwise.py")],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.mark.parametrize("dk,dv,B,L,pos0,bias,with_state", [
    (128, 128, 64, 300, 0, 0.5, False),   # 128-column slices, one launch after the key sum
    (64, 64, 128, 517, 7, 0.0, True),     # carried-in state and key sum
    (256, 128, 256, 600, 1000, 0.5, True),  # pre-converted, 4 sub-blocks a chunk
    (128, 256, 512, 1100, 0, 0.3, False),
    (128, 128, 64, 64 * 33 + 1, 0, 0.5, True),  # few pairs: two-pass segments after the key sum
    (256, 64, 64, 1, 3, 0.5, True)])
def test_tc_norm_r_matches_oracle(dk, dv, B, L, pos0, bias, with_state):
    """R~ on the tensor-core kernel (workspace form): a key-sum pass writes each row's factor
    1/max(|sum of scores|, 1) and z_out, the kernel folds it into its row scale.  Outputs,
    state and z against the oracle; q and k carry a mean (bias) so that most rows' sums exceed
    1 and the normalisation is active.

    Bar: the plain max|err|/rms <= 1e-2 on the R~-normalised output.  R~ divides each row by
    its own D_n = max(|sum of scores|, 1), which leaves rows of very different sizes (early rows
    keep D ~ 1, later ones are divided by tens), so the rms over the normalised output is small
    against the early rows' values; R~ calls therefore run with split fp16 operands (hi + lo).
    The output scaled back by the oracle's D_n (against the oracle's output without R~, which
    is ref * D_n exactly) is printed and held to the same bar: a wrong row factor on the GPU
    shows there as its relative error."""
    b, h = 2, 3
    q, k, v = si.qkv(b, L, h, dk, dv, 900 + dk + B, "bf16")
    q = (q.float() + bias).to(q.dtype)
    k = (k.float() + bias).to(k.dtype)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 901, std=0.05) if with_state else None
    z0 = si.randn((b, h, dk), 902, "f32", std=3.0) if with_state else None
    ref, Sref, zref = oracle.chunkwise(q, k, v, g, B, th, pos0, oracle.F_ALL, state_in=S0, z_in=z0)
    plain, _, _ = oracle.chunkwise(q, k, v, g, B, th, pos0, FLAGS, state_in=S0, z_in=z0)
    ref, plain = np.asarray(ref), np.asarray(plain)
    # D_n = ||plain_n|| / ||ref_n|| per (token, head) row (ref = plain / D_n)
    D = np.sqrt((plain ** 2).sum(-1, keepdims=True) / np.maximum((ref ** 2).sum(-1, keepdims=True), 1e-300))
    assert np.all(D >= 1 - 1e-9)
    if bias:
        active = np.mean(D[..., 0] > 1 + 1e-9)
        assert active > 0.3, active
    nbytes = rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv))
    n = rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, oracle.F_ALL, B, g, nbytes)
    assert n >= 2, n  # the key-sum pass, then the tensor-core kernel(s)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o = torch.empty(b, L, h, dv, device="cuda")
    so = torch.empty(b, h, dk, dv, device="cuda")
    zo = torch.empty(b, h, dk, device="cuda")
    rn.retnet_retention_chunkwise_ws(dev(q), dev(k), dev(v), o, g, th, pos0, oracle.F_ALL, B,
                                     None if S0 is None else dev(S0), so, None if z0 is None else dev(z0), zo,
                                     workspace=ws)
    torch.cuda.synchronize()
    e = err(o.cpu().double().numpy() * D, plain)
    e_plain = err(o, ref)
    print(f"R~ dk={dk} dv={dv} B={B} L={L} launches={n}: plain max|err|/rms = {e_plain:.3e}, "
          f"rescaled {e:.3e}")
    assert e_plain <= TOL_BF16
    assert e <= TOL_BF16
    assert err(so, Sref) <= TOL_BF16
    assert err(zo, zref) <= TOL_F32


def test_tc_norm_r_needs_room_for_its_factors():
    """R~ with a workspace too small for the row factors takes the CUDA-core kernel (one
    launch); with room, the key-sum pass comes first."""
    g = si.gamma_schedule(4)
    a256 = lambda x: (x + 255) // 256 * 256
    need = a256(2 * 300 * 4 * 4) + a256(2 * 4 * 128 * 64 * 4)  # row factors + key-sum segment values
    assert rn.retnet_chunkwise_launches((2, 300, 4, 128), 64, rn.BF16, oracle.F_ALL, 64, g, need - 256) == 1
    # two key-sum passes (the sequence in segments), then the kernel (no room for a split)
    assert rn.retnet_chunkwise_launches((2, 300, 4, 128), 64, rn.BF16, oracle.F_ALL, 64, g, need) == 3


def test_fp16_range_is_reported():
    """bf16 inputs beyond the fp16 operand range (a value of v above 65504, a q element whose
    rotated, scaled copy exceeds it): the tensor-core kernel rounds them to inf, and the range
    counter says so -- no silent non-finite output.  In-range calls leave it at zero, with
    single and split operands and with the conversion pre-pass."""
    b, L, h, dk, dv = 1, 256, 2, 64, 64
    q, k, v = si.qkv(b, L, h, dk, dv, 1500, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device="cuda")
    v_big = v.clone()
    v_big[0, 70, 1, 5] = 70000.0
    q_big = q.clone()
    q_big[0, 130, 0, 10] = 1.0e5
    for flags in (FLAGS, FLAGS | rn.F_PRECISE):
        for B, wsp in ((64, None), (128, ws)):  # in-kernel converters; conversion pre-pass
            o = torch.empty(b, L, h, dv, device="cuda")
            rn.retnet_fp16_range_errors(clear=True)
            rn.retnet_retention_chunkwise_ws(dev(q), dev(k), dev(v), o, g, th, 0, flags, B, workspace=wsp)
            assert rn.retnet_fp16_range_errors(clear=True) == 0
            assert bool(torch.isfinite(o).all())
            for qq, vv in ((q, v_big), (q_big, v)):
                rn.retnet_retention_chunkwise_ws(dev(qq), dev(k), dev(vv), o, g, th, 0, flags, B, workspace=wsp)
                n = rn.retnet_fp16_range_errors(clear=True)
                print(f"flags={flags} B={B} ws={wsp is not None}: {n} range reports, "
                      f"finite={bool(torch.isfinite(o).all())}")
                assert n > 0


def test_bounded_waits_give_up_and_recover():
    """The give-up path of the kernel's bounded waits.  With the wait budget lowered to 500 SM
    cycles (a testing aid) the roles' waits for one another give up: the call must return (no
    hang), count its give-ups, drain the TMA copies and MMAs already issued and free its tensor
    memory.  After the default budget is restored the same call is bit-identical to one made
    before, and counts nothing.  (A plain launch, no thread-block clusters.)"""
    b, L, h, dk, dv, B = 1, 640, 2, 64, 64, 64
    q, k, v = (dev(x) for x in si.qkv(b, L, h, dk, dv, 1600, "bf16"))
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    assert rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, B, g) == 1
    o_ref, o_bad, o_again = (torch.empty(b, L, h, dv, device="cuda") for _ in range(3))
    rn.retnet_retention_chunkwise(q, k, v, o_ref, g, th, 0, FLAGS, B)
    torch.cuda.synchronize()
    assert rn.retnet_debug_wait_timeouts(clear=True) == 0
    rn.retnet_debug_set_wait_budget(500)
    try:
        rn.retnet_retention_chunkwise(q, k, v, o_bad, g, th, 0, FLAGS, B)
        torch.cuda.synchronize()
        gave_up = rn.retnet_debug_wait_timeouts(clear=True)
    finally:
        rn.retnet_debug_set_wait_budget(0)
    rn.retnet_fp16_range_errors(clear=True)  # (the abandoned call's buffers are undefined)
    print(f"waits that gave up with a 500-cycle budget: {gave_up}")
    assert gave_up > 0
    rn.retnet_retention_chunkwise(q, k, v, o_again, g, th, 0, FLAGS, B)
    torch.cuda.synchronize()
    assert torch.equal(o_again, o_ref)
    assert rn.retnet_debug_wait_timeouts(clear=True) == 0


@pytest.mark.parametrize("dv,B,L,pos0,with_state", [(64, 128, 300, 0, False), (192, 256, 1100, 7, True),
                                                    (128, 512, 513, 0, True), (64, 512, 129, 3, False),
                                                    (512, 128, 400, 0, True)])
def test_tc_p_pass_matches_oracle(dv, B, L, pos0, with_state):
    """d_k 256 with chunks of several 64-row sub-blocks: the P pass computes every masked score
    tile once per head into the workspace and the pipelined kernel loads them beside V (three
    launches: conversion pre-pass, P pass, kernel).  Against the oracle, and bit-identical to the
    same call with a workspace one byte too small for the P tiles (the kernel then forms P itself
    from the same operands, in the same order) and to the same call with the one-CTA-a-tile P
    kernel (RETNET_P_TILE_KERNEL=1) in place of the one-CTA-a-chunk kernel."""
    b, h, dk = 2, 3, 256
    q, k, v = si.qkv(b, L, h, dk, dv, 1800 + B + L, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    S0 = si.decode_state(b, h, dk, dv, 1801, std=0.05) if with_state else None
    ref, Sref, _ = oracle.chunkwise(q, k, v, g, B, th, pos0, FLAGS, state_in=S0)
    full = rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv))
    a256 = lambda x: (x + 255) // 256 * 256
    copies = 2 * a256(b * L * h * dk * 2) + a256(b * L * h * dv * 2)
    tiles = b * h * ((L + B - 1) // B) * ((B // 64) * (B // 64 + 1) // 2)
    small = copies + a256(tiles * 64 * 64 * 2) - 1  # room for the copies, not for the P tiles
    assert rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS, B, g, full) == 3
    assert rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS, B, g, small) == 2
    outs = []
    for nbytes, tile_kernel in ((full, False), (small, False), (full, True)):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o = torch.empty(b, L, h, dv, device="cuda")
        so = torch.empty(b, h, dk, dv, device="cuda")
        if tile_kernel:
            os.environ["RETNET_P_TILE_KERNEL"] = "1"
        try:
            rn.retnet_retention_chunkwise_ws(dev(q), dev(k), dev(v), o, g, th, pos0, FLAGS, B,
                                             None if S0 is None else dev(S0), so, workspace=ws)
            torch.cuda.synchronize()
        finally:
            os.environ.pop("RETNET_P_TILE_KERNEL", None)
        outs.append((o, so))
    e, es = err(outs[0][0], ref), err(outs[0][1], Sref)
    print(f"P pass dv={dv} B={B} L={L}: out {e:.3e}, state {es:.3e}")
    assert e <= TOL_BF16 and es <= TOL_BF16
    for o2, s2 in outs[1:]:
        assert torch.equal(outs[0][0], o2) and torch.equal(outs[0][1], s2)
