"""The tensor-core gradient computes each gradient sum as a retention output (runs of the
forward kernel): dq through a forward run with query dO, key v, value k~ and start state S0^T;
dk and dv through runs over the reversed sequence, dv with the rotation at the reversed
positions and theta negated.  This checks that decomposition in fp64 with the oracle's own
forward forms against the oracle's gradient (itself pinned by finite differences), so a wrong
reversal, sign or factor in the scheme fails here, on the CPU, whatever the kernels do.
"""
import numpy as np
import pytest

import oracle


def _rotate(x, theta, pos0, sign=1.0):
    """Turn every pair (2j, 2j+1) of x[:, t] by sign * (pos0 + t) * theta_j."""
    y = x.copy()
    L = x.shape[1]
    for t in range(L):
        a = sign * (pos0 + t) * theta
        c, s = np.cos(a), np.sin(a)
        x0, x1 = x[:, t, :, 0::2], x[:, t, :, 1::2]
        y[:, t, :, 0::2] = x0 * c - x1 * s
        y[:, t, :, 1::2] = x0 * s + x1 * c
    return y


@pytest.mark.parametrize("flags,pos0,with_state", [
    (oracle.F_XPOS | oracle.F_SCALE_SQRT_D | oracle.F_NORM_D, 3, True),
    (oracle.F_XPOS, 11, False),
    (oracle.F_SCALE_SQRT_D | oracle.F_NORM_D, 0, True)])
def test_gradient_as_retention_runs(flags, pos0, with_state):
    rng = np.random.default_rng(41)
    b, L, h, dk, dv = 2, 9, 2, 4, 6
    q, k = rng.standard_normal((b, L, h, dk)), rng.standard_normal((b, L, h, dk))
    v, do = rng.standard_normal((b, L, h, dv)), rng.standard_normal((b, L, h, dv))
    S0 = rng.standard_normal((b, h, dk, dv)) if with_state else None
    g = np.array([0.9, 0.75])
    th = np.array([0.4, 1.3])
    xpos = bool(flags & oracle.F_XPOS)
    # row factors f_t of the forward: the D~ part from the oracle's own output on unit inputs
    # (with and without it), the 1/sqrt(d_k) part for this d_k
    ones_q = np.zeros((1, L, h, 1)); ones_q[..., 0] = 1.0
    f = (oracle.parallel(ones_q, ones_q, ones_q, g, None, pos0, flags & oracle.F_NORM_D) /
         oracle.parallel(ones_q, ones_q, ones_q, g, None, pos0, 0))[0, :, :, 0]  # [L][h]
    if flags & oracle.F_SCALE_SQRT_D:
        f = f / np.sqrt(dk)
    qt = _rotate(q, th, pos0) if xpos else q
    kt = _rotate(k, th, pos0) if xpos else k
    rev = lambda x: x[:, ::-1].copy()
    # dq~ / f: forward order, query dO, key v, value k~, start state S0^T
    s0t = None if S0 is None else np.ascontiguousarray(np.swapaxes(S0, 2, 3))
    dq_t, _, _ = oracle.chunkwise(do, v, kt, g, 4, None, 0, 0, state_in=s0t)
    dq = dq_t * f[None, :, :, None]
    dq = _rotate(dq, th, pos0, -1.0) if xpos else dq
    # dk~: reversed, query v, key dO, value f q~
    dk_t = rev(oracle.parallel(rev(v), rev(do), rev(qt * f[None, :, :, None]), g, None, 0, 0))
    dk_ = _rotate(dk_t, th, pos0, -1.0) if xpos else dk_t
    # dv: reversed, query k, key q, value f dO, rotation at the reversed positions with -theta
    dv_ = rev(oracle.parallel(rev(k), rev(q), rev(do * f[None, :, :, None]), g, -th, 0,
                              oracle.F_XPOS if xpos else 0))
    rq, rk, rv, _ = oracle.backward(q, k, v, do, g, th, pos0, flags, state_in=S0)
    for got, ref in ((dq, rq), (dk_, rk), (dv_, rv)):
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)
