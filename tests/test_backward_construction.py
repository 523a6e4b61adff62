"""The data flow of the CUDA backward, replayed in float64 on tiny inputs, against the adjoint
oracle.  No GPU: this checks the construction itself, with every scan run as the plain token
loop.  It covers the reversed scan with unit input weights and decays shifted by one token, the
two scans with the head and state dimensions swapped, the dot products that feed the decay
gradient, and its reverse cumulative sum.  A wrong shift, a missing transpose or a dropped term
in the construction fails here before any kernel runs.
"""
import numpy as np
import pytest

import oracle


def _scan(x, w, dec_dt, A, B, C, init):
    """h_t = exp(dec_dt_t A_h) h_{t-1} + w_t x_t B_t^T, y_t = h_t C_t, per head (B, C per head)."""
    b, L, H, _ = x.shape
    E, K = x.shape[3], B.shape[3]
    y = np.zeros((b, L, H, E))
    fin = np.zeros((b, H, E, K))
    for bi in range(b):
        for h in range(H):
            s = np.zeros((E, K)) if init is None else init[bi, h].copy()
            for t in range(L):
                s = np.exp(dec_dt[bi, t, h] * A[h]) * s + w[bi, t, h] * np.outer(x[bi, t, h],
                                                                                B[bi, t, h])
                y[bi, t, h] = s @ C[bi, t, h]
            fin[bi, h] = s
    return y, fin


@pytest.mark.parametrize("seed,with_init,with_dfinal", [(11, True, True), (12, False, True),
                                                       (13, True, False)])
def test_backward_construction_matches_adjoint_oracle(seed, with_init, with_dfinal):
    rng = np.random.default_rng(seed)
    b, L, H, G, P, N = 2, 9, 4, 2, 3, 5
    x = rng.standard_normal((b, L, H, P))
    dt = rng.uniform(0.01, 0.3, (b, L, H))
    A = -rng.uniform(0.5, 2.0, H)
    B = rng.standard_normal((b, L, G, N))
    C = rng.standard_normal((b, L, G, N))
    D = rng.standard_normal(H)
    dy = rng.standard_normal((b, L, H, P))
    init = rng.standard_normal((b, H, P, N)) if with_init else None
    dfinal = rng.standard_normal((b, H, P, N)) if with_dfinal else None
    ref = oracle.ssd_scan_bwd(x, dt, A, B, C, D, dy, init, dfinal)

    hpg = H // G
    Bh, Ch = np.repeat(B, hpg, axis=2), np.repeat(C, hpg, axis=2)
    rev = lambda v: v[:, ::-1]
    T = lambda v: None if v is None else np.swapaxes(v, 2, 3)
    ones = np.ones_like(dt)
    dtr = np.zeros_like(dt)              # decays of the reversed sequence, shifted by one token
    dtr[:, 1:] = dt[:, ::-1][:, :-1]

    # g_t B_t: the scan of the reversed sequence, x' = dy, B' = C, C' = B, unit weights, from dfinal
    gb_rev, g0 = _scan(rev(dy), ones, dtr, A, rev(Ch), rev(Bh), dfinal)
    dx = D[None, None, :, None] * dy + dt[..., None] * rev(gb_rev)
    dinit = np.exp(dt[:, 0, :] * A)[..., None, None] * g0
    # dB: reversed, head dimension N, state dimension P (x'' = C, B'' = dy, C'' = x), from dfinal^T
    yb, _ = _scan(rev(Ch), ones, dtr, A, rev(dy), rev(x), T(dfinal))
    dB = (dt[..., None] * rev(yb)).reshape(b, L, G, hpg, N).sum(3)
    ddt_in = np.einsum("blhn,blhn->blh", rev(yb), Bh)            # <x_t, g_t B_t>
    # dC: forward, x'' = B, B'' = x, C'' = dy, weights dt, from init^T
    yc, fin_t = _scan(Bh, dt, dt, A, x, dy, T(init))
    dC = yc.reshape(b, L, G, hpg, N).sum(3)
    ydot = np.einsum("blhn,blhn->blh", yc, Ch)                   # <dy_t, y_t - D x_t>
    # the decay gradient: q, its reverse cumsum, ddt and dA; dD
    q = ydot - dt * ddt_in
    if dfinal is not None:
        q[:, -1] += np.einsum("bhnp,bhnp->bh", T(dfinal), fin_t)
    dl = np.cumsum(q[:, ::-1], axis=1)[:, ::-1]
    ddt = ddt_in + A * dl
    dA = np.einsum("blh,blh->h", dt, dl)
    dD = np.einsum("blhp,blhp->h", dy, x)

    got = dict(dx=dx, ddt=ddt, dA=dA, dB=dB, dC=dC, dD=dD, dinit=dinit)
    for k, v in got.items():
        scale = max(np.abs(ref[k]).max(), 1e-30)
        assert np.abs(v - ref[k]).max() <= 1e-12 * scale, k
