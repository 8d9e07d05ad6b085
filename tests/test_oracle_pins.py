"""Pins for the fp64 oracle, against what the pages and the mathematics fix.

Source: "阅读笔记：RetNet" (mzeromiko blog) §2.2 Recurrent Mode, §2.3 Parallel Mode,
§2.4 Chunkwise Recurrent Mode, §三.2 MSR, §三.3 Normalization.  The pages print no
worked numbers, so the pins are: the page's claim that its three forms are equal
(checked between independently written loops), closed forms, special cases that reduce
to a library routine (numpy matmul, numpy complex arithmetic for the page's own
complex xPos form, torch's group_norm/silu), causality, linearity and the state's
closed form.  ``test_oracle_mutants.py`` shows that plausible mistakes fail these.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si

FLAG_COMBOS = list(range(16))


def rel(a, b):
    return float(np.abs(a - b).max() / max(np.sqrt((b ** 2).mean()), 1e-300))


def _inputs(b, L, h, dk, dv, seed):
    q, k, v = si.qkv(b, L, h, dk, dv, seed, "f32")
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


# ---- T1: the page's three forms agree (§2.2 = §2.3 = §2.4) -------------------------------

@pytest.mark.parametrize("h,dk,dv,L,B", [(1, 2, 2, 1, 1), (2, 16, 16, 5, 3), (2, 16, 8, 64, 16),
                                         (1, 2, 4, 70, 64), (2, 16, 16, 70, 16), (2, 4, 6, 33, 7)])
def test_three_forms_agree(h, dk, dv, L, B):
    q, k, v = _inputs(2, L, h, dk, dv, 11 + L + B)
    g = si.gamma_schedule(h)
    th = si.theta_schedule(dk)
    for flags in FLAG_COMBOS:
        for pos0 in (0, 37):
            op = oracle.parallel(q, k, v, g, th, pos0, flags)
            orc, s1, z1 = oracle.recurrent(q, k, v, g, th, pos0, flags)
            och, s2, z2 = oracle.chunkwise(q, k, v, g, B, th, pos0, flags)
            assert rel(orc, op) < 1e-12, (flags, pos0)
            assert rel(och, op) < 1e-12, (flags, pos0)
            assert rel(s2, s1) < 1e-12 and rel(z2, z1) < 1e-12


def test_chunk_one_is_recurrent_and_chunk_L_is_parallel():
    q, k, v = _inputs(1, 40, 2, 8, 8, 5)
    g, th = si.gamma_schedule(2), si.theta_schedule(8)
    orc, _, _ = oracle.recurrent(q, k, v, g, th, 0, oracle.F_ALL)
    o1, _, _ = oracle.chunkwise(q, k, v, g, 1, th, 0, oracle.F_ALL)
    oL, _, _ = oracle.chunkwise(q, k, v, g, 40, th, 0, oracle.F_ALL)
    op = oracle.parallel(q, k, v, g, th, 0, oracle.F_ALL)
    assert rel(o1, orc) < 1e-13
    assert rel(oL, op) < 1e-13


# ---- T2: closed form with d = 1, q = k = v = 1 (§2.2, D_nn = 1) ---------------------------

@pytest.mark.parametrize("gamma", [0.96875, 0.5, 1.0 - 2.0 ** -20])
def test_closed_form_ones(gamma):
    L = 300
    ones = np.ones((1, L, 1, 1))
    g = np.array([gamma])
    n = np.arange(1, L + 1, dtype=np.float64)
    # sum_{j<n} gamma^j = (1 - gamma^n)/(1 - gamma), evaluated without cancellation
    geo = -np.expm1(n * np.log1p(-(1.0 - gamma))) / (1.0 - gamma)
    for fn in ("parallel", "recurrent", "chunkwise"):
        def run(flags):
            if fn == "parallel":
                return oracle.parallel(ones, ones, ones, g, None, 0, flags)
            if fn == "recurrent":
                return oracle.recurrent(ones, ones, ones, g, None, 0, flags)[0]
            return oracle.chunkwise(ones, ones, ones, g, 17, None, 0, flags)[0]
        raw = run(0)[0, :, 0, 0]
        np.testing.assert_allclose(raw, geo, rtol=1e-12)
        nd = run(oracle.F_NORM_D | oracle.F_SCALE_SQRT_D)[0, :, 0, 0]
        np.testing.assert_allclose(nd, np.sqrt(geo), rtol=1e-12)
        nr = run(oracle.F_NORM_D | oracle.F_NORM_R)[0, :, 0, 0]
        np.testing.assert_allclose(nr, np.ones(L), rtol=1e-12)
        # R~ alone: sigma_n = geo_n >= 1, so o_n = geo_n / geo_n = 1 as well.
        np.testing.assert_allclose(run(oracle.F_NORM_R)[0, :, 0, 0], np.ones(L), rtol=1e-12)


def test_norm_r_clamp_keeps_small_rows():
    # q.k small: |sigma| < 1, so the clamp max(|sigma|, 1) leaves the row as is.
    L = 20
    q = np.full((1, L, 1, 1), 0.01)
    k = np.full((1, L, 1, 1), 0.02)
    v = np.full((1, L, 1, 1), 3.0)
    g = np.array([0.9])
    a = oracle.parallel(q, k, v, g, None, 0, 0)
    b = oracle.parallel(q, k, v, g, None, 0, oracle.F_NORM_R)
    np.testing.assert_allclose(a, b, rtol=1e-14)
    # Negative scores: the absolute value is taken and the sign of o is kept.
    qn = -np.ones((1, L, 1, 1)) * 2.0
    kn = np.ones((1, L, 1, 1))
    vn = np.ones((1, L, 1, 1))
    o = oracle.parallel(qn, kn, vn, g, None, 0, oracle.F_NORM_R)[0, :, 0, 0]
    geo = 2.0 * (1 - 0.9 ** np.arange(1, L + 1)) / 0.1
    expect = -geo / np.maximum(geo, 1.0)
    np.testing.assert_allclose(o, expect, rtol=1e-12)


# ---- T3: xPos closed form, d = 2 (§2.1 last equation, §2.3 Theta) -------------------------

@pytest.mark.parametrize("theta0", [0.3, 1.0, 2.5])
def test_xpos_closed_form(theta0):
    L, gamma = 50, 0.9
    q = np.zeros((1, L, 1, 2)); q[..., 0] = 1.0
    k = q.copy()
    v = np.ones((1, L, 1, 1))
    th = np.array([theta0])
    g = np.array([gamma])
    n = np.arange(L)
    w = gamma * np.exp(1j * theta0)
    expect = np.real((1 - w ** (n + 1)) / (1 - w))  # sum_{j<=n} gamma^j cos(j theta0)
    for pos0 in (0, 1000):
        o = oracle.parallel(q, k, v, g, th, pos0, oracle.F_XPOS)[0, :, 0, 0]
        np.testing.assert_allclose(o, expect, rtol=1e-11, atol=1e-12)
        o2 = oracle.recurrent(q, k, v, g, th, pos0, oracle.F_XPOS)[0][0, :, 0, 0]
        np.testing.assert_allclose(o2, expect, rtol=1e-11, atol=1e-12)


def test_xpos_shift_invariance():
    q, k, v = _inputs(1, 30, 2, 16, 8, 9)
    g, th = si.gamma_schedule(2), si.theta_schedule(16)
    f = oracle.F_XPOS | oracle.F_SCALE_SQRT_D
    a = oracle.parallel(q, k, v, g, th, 0, f)
    b = oracle.parallel(q, k, v, g, th, 12345, f)
    assert rel(b, a) < 1e-9  # only the angle's rounding differs


# ---- T4: special cases that reduce to library routines -------------------------------------

def test_matches_numpy_masked_matmul_without_rotation():
    q, k, v = _inputs(2, 45, 3, 8, 5, 4)
    g = np.array([0.96875, 0.8, 0.5])
    o = oracle.parallel(q, k, v, g, None, 0, 0)
    L = q.shape[1]
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    for b in range(2):
        for h in range(3):
            D = np.where(i >= j, g[h] ** (i - j).astype(np.float64), 0.0)
            ref = ((q[b, :, h] @ k[b, :, h].T) * D) @ v[b, :, h]
            assert rel(o[b, :, h], ref) < 1e-13


def test_matches_page_complex_form_with_rotation():
    """o_n = sum_m gamma^(n-m) Re[(Q_n e^{in theta})(K_m e^{im theta})^dagger] v_m, in numpy complex."""
    b_, L, h, dk, dv = 1, 33, 2, 8, 4
    q, k, v = _inputs(b_, L, h, dk, dv, 6)
    g, th = si.gamma_schedule(h).astype(np.float64), si.theta_schedule(dk).astype(np.float64)
    pos0 = 7
    o = oracle.parallel(q, k, v, g, th, pos0, oracle.F_XPOS)
    p = np.arange(L) + pos0
    rot = np.exp(1j * p[:, None] * th[None, :])
    for hh in range(h):
        Qc = (q[0, :, hh, 0::2] + 1j * q[0, :, hh, 1::2]) * rot
        Kc = (k[0, :, hh, 0::2] + 1j * k[0, :, hh, 1::2]) * rot
        S = np.real(Qc @ np.conj(Kc).T)
        i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
        D = np.where(i >= j, g[hh] ** (i - j).astype(np.float64), 0.0)
        ref = (S * D) @ v[0, :, hh]
        assert rel(o[0, :, hh], ref) < 1e-12


def test_normalisations_match_numpy_row_scales():
    """§三.3 applied to the library-computed score matrix: /sqrt(d), D~ rows, R~ rows."""
    q, k, v = _inputs(1, 40, 2, 16, 8, 8)
    g = si.gamma_schedule(2).astype(np.float64)
    o = oracle.parallel(q, k, v, g, None, 0, oracle.F_SCALE_SQRT_D | oracle.F_NORM_D | oracle.F_NORM_R)
    L = 40
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    for hh in range(2):
        D = np.where(i >= j, g[hh] ** (i - j).astype(np.float64), 0.0)
        Dt = D / np.sqrt(D.sum(axis=1, keepdims=True))
        R = (q[0, :, hh] @ k[0, :, hh].T) / math.sqrt(16) * Dt
        Rt = R / np.maximum(np.abs(R.sum(axis=1, keepdims=True)), 1.0)
        assert rel(o[0, :, hh], Rt @ v[0, :, hh]) < 1e-12


# ---- T5: MSR epilogue (§三.2): GroupNorm per head, swish gate --------------------------------

def test_epilogue_matches_torch_group_norm_and_silu():
    tokens, h, dv = 37, 4, 24
    y = si.randn((tokens, h * dv), 3, "f32").double() * 3.0 + 0.5
    gt = si.randn((tokens, h * dv), 4, "f32").double()
    out = oracle.msr_epilogue(y.numpy(), gt.numpy(), h, eps=1e-5)
    ref = torch.nn.functional.group_norm(y, h, eps=1e-5) * torch.nn.functional.silu(gt)
    assert rel(out, ref.numpy()) < 1e-13


def test_epilogue_invariants():
    tokens, h, dv = 16, 2, 32
    y = si.randn((tokens, h * dv), 5, "f32").double().numpy()
    ones_gate = np.full(y.shape, 50.0)  # swish(50) = 50 * sigmoid(50) ~= 50 exactly in fp64
    out = oracle.msr_epilogue(y, ones_gate, h, eps=1e-5) / 50.0
    rows = out.reshape(tokens, h, dv)
    yr = y.reshape(tokens, h, dv)
    var = yr.var(axis=-1)
    np.testing.assert_allclose(rows.mean(axis=-1), 0.0, atol=1e-13)
    np.testing.assert_allclose(rows.var(axis=-1), var / (var + 1e-5), rtol=1e-10)
    # GroupNorm(alpha * head) = GroupNorm(head), up to eps (page §三.3 reason one)
    # with eps > 0 the invariance is exact up to the factor sqrt(var+eps)/sqrt(var+eps/49)
    out2 = oracle.msr_epilogue(y * 7.0, ones_gate, h, eps=1e-5) / 50.0
    ratio = np.sqrt(var + 1e-5) / np.sqrt(var + 1e-5 / 49.0)
    np.testing.assert_allclose(out2.reshape(tokens, h, dv), rows * ratio[..., None], rtol=1e-10,
                               atol=1e-13)
    out3 = oracle.msr_epilogue(y * 7.0, ones_gate, h, eps=0.0) / 50.0
    out4 = oracle.msr_epilogue(y, ones_gate, h, eps=0.0) / 50.0
    assert np.abs(out3 - out4).max() < 1e-12
    # swish(0) = 0
    assert np.all(oracle.msr_epilogue(y, np.zeros_like(y), h) == 0.0)


def test_groupnorm_removes_row_scales():
    """Un-normalised retention and fully normalised retention agree after GroupNorm (§三.3)."""
    q, k, v = _inputs(1, 48, 2, 8, 16, 12)
    g, th = si.gamma_schedule(2), si.theta_schedule(8)
    raw = oracle.parallel(q, k, v, g, th, 0, oracle.F_XPOS)
    nrm = oracle.parallel(q, k, v, g, th, 0, oracle.F_ALL)
    gate = np.ones((1, 48, 32)) * 30.0
    a = oracle.msr_epilogue(raw.reshape(1, 48, 32), gate, 2, eps=0.0)
    b = oracle.msr_epilogue(nrm.reshape(1, 48, 32), gate, 2, eps=0.0)
    assert rel(a, b) < 1e-10


# ---- T6: causality (§2.3: D_nm = 0 for n < m) -----------------------------------------------

def test_causality_bit_exact():
    q, k, v = _inputs(1, 50, 2, 8, 8, 13)
    g, th = si.gamma_schedule(2), si.theta_schedule(8)
    m = 31
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, m:] += 5.0; k2[:, m:] -= 3.0; v2[:, m:] *= -2.0
    for fn in (lambda *a: oracle.parallel(*a, g, th, 0, oracle.F_ALL),
               lambda *a: oracle.recurrent(*a, g, th, 0, oracle.F_ALL)[0],
               lambda *a: oracle.chunkwise(*a, g, 16, th, 0, oracle.F_ALL)[0]):
        a, b = fn(q, k, v), fn(q2, k2, v2)
        assert np.array_equal(a[:, :m], b[:, :m])
        assert not np.array_equal(a[:, m:], b[:, m:])


# ---- T7: state closed form and prefill -> decode hand-off (§2.2 vs §2.4) ---------------------

def test_state_closed_form_and_handoff():
    L, h, dk, dv = 37, 2, 8, 6
    q, k, v = _inputs(2, L, h, dk, dv, 14)
    g, th = si.gamma_schedule(h).astype(np.float64), si.theta_schedule(dk).astype(np.float64)
    _, S, z = oracle.recurrent(q, k, v, g, th, 0, oracle.F_XPOS)
    _, Sc, zc = oracle.chunkwise(q, k, v, g, 10, th, 0, oracle.F_XPOS)
    assert rel(Sc, S) < 1e-13 and rel(zc, z) < 1e-13
    # S_L = sum_m gamma^(L-1-m) k'_m^T v_m with k'_m the rotated key (complex form for the turn)
    p = np.arange(L)
    rot = np.exp(1j * p[:, None] * th[None, :])
    for b in range(2):
        for hh in range(h):
            kc = (k[b, :, hh, 0::2] + 1j * k[b, :, hh, 1::2]) * rot
            kr = np.empty((L, dk)); kr[:, 0::2] = kc.real; kr[:, 1::2] = kc.imag
            w = g[hh] ** (L - 1 - p).astype(np.float64)
            assert rel(S[b, hh], (kr * w[:, None]).T @ v[b, :, hh]) < 1e-12
            assert rel(z[b, hh], (kr * w[:, None]).sum(axis=0)) < 1e-12
    # prefill 0..P-1 with the chunkwise form, then continue token by token from its state
    P = 23
    for flags in (oracle.F_ALL, oracle.F_XPOS | oracle.F_NORM_D):
        full = oracle.parallel(q, k, v, g, th, 0, flags)
        o1, S1, z1 = oracle.chunkwise(q[:, :P], k[:, :P], v[:, :P], g, 8, th, 0, flags)
        o2, _, _ = oracle.recurrent(q[:, P:], k[:, P:], v[:, P:], g, th, P, flags, S1, z1)
        assert rel(np.concatenate([o1, o2], axis=1), full) < 1e-12


# ---- T8: linearity in V (R~ off) ------------------------------------------------------------

def test_linearity_in_v():
    q, k, v = _inputs(1, 30, 2, 8, 8, 15)
    v2 = _inputs(1, 30, 2, 8, 8, 16)[2]
    g, th = si.gamma_schedule(2), si.theta_schedule(8)
    f = oracle.F_XPOS | oracle.F_SCALE_SQRT_D | oracle.F_NORM_D
    a = oracle.chunkwise(q, k, 2.0 * v - 3.0 * v2, g, 8, th, 0, f)[0]
    b = 2.0 * oracle.chunkwise(q, k, v, g, 8, th, 0, f)[0] - 3.0 * oracle.chunkwise(q, k, v2, g, 8, th, 0, f)[0]
    assert rel(a, b) < 1e-13


# ---- golden: the page's gamma schedule (§三.2) -----------------------------------------------

def test_gamma_schedule_golden():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "gamma_schedule_h16.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    want = np.array([float.fromhex(r[1]) for r in rows])
    got = si.gamma_schedule(16).astype(np.float64)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("flags,pos0", [(oracle.F_XPOS | oracle.F_SCALE_SQRT_D | oracle.F_NORM_D, 5), (0, 0),
                                        (oracle.F_XPOS, 123)])
def test_backward_is_the_derivative_of_the_recurrent_form(flags, pos0):
    """oracle.backward against central finite differences of oracle.recurrent (the page's §2.2
    form, with a state before the first token) for L = sum(dO * O): every element of q, k, v
    and the state.  Exact up to the difference quotient's own error (h = 1e-5, fp64)."""
    rng = np.random.default_rng(31)
    b, L, h, dk, dv = 1, 6, 2, 4, 3
    q, k = rng.standard_normal((b, L, h, dk)), rng.standard_normal((b, L, h, dk))
    v, do = rng.standard_normal((b, L, h, dv)), rng.standard_normal((b, L, h, dv))
    S0 = rng.standard_normal((b, h, dk, dv))
    g = np.array([0.9, 0.7])
    th = np.array([0.3, 1.1])
    gq, gk, gv, gs = oracle.backward(q, k, v, do, g, th, pos0, flags, state_in=S0)

    def loss(q_, k_, v_, s_):
        o, _, _ = oracle.recurrent(q_, k_, v_, g, th, pos0, flags, state_in=s_)
        return float((o * do).sum())

    eps = 1e-5
    for name, x, grad in (("q", q, gq), ("k", k, gk), ("v", v, gv), ("state", S0, gs)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": (q, k, v, S0), "k": (q, k, v, S0), "v": (q, k, v, S0), "state": (q, k, v, S0)}[name]
            a_p, a_m = list(args), list(args)
            pos = ["q", "k", "v", "state"].index(name)
            a_p[pos], a_m[pos] = xp, xm
            fd[idx] = (loss(*a_p) - loss(*a_m)) / (2 * eps)
        scale = max(np.abs(fd).max(), 1e-12)
        assert np.abs(grad - fd).max() / scale < 1e-7, (name, np.abs(grad - fd).max() / scale)


def test_backward_without_state_and_linearity():
    """Without a state the state gradient is absent; dv is linear in dO and does not depend on v
    (O is linear in v), checked on two dO."""
    rng = np.random.default_rng(32)
    q, k = rng.standard_normal((2, 9, 1, 4)), rng.standard_normal((2, 9, 1, 4))
    v = rng.standard_normal((2, 9, 1, 2))
    d1, d2 = rng.standard_normal((2, 9, 1, 2)), rng.standard_normal((2, 9, 1, 2))
    g = np.array([0.8])
    _, _, a, s = oracle.backward(q, k, v, d1, g, None, 0, oracle.F_SCALE_SQRT_D)
    _, _, b_, _ = oracle.backward(q, k, 3 * v + 1, d2, g, None, 0, oracle.F_SCALE_SQRT_D)
    _, _, c, _ = oracle.backward(q, k, v, 2 * d1 - d2, g, None, 0, oracle.F_SCALE_SQRT_D)
    assert s is None
    np.testing.assert_allclose(c, 2 * a - b_, rtol=1e-12, atol=1e-12)
