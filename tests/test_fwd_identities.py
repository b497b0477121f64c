"""The factored decay form of the tensor-core forward (and, at the end, the head-pair kernel's
exact form factored by quarters), checked on the CPU against the oracle.
Per 128-token block with within-block cumsum A_cs and reference m (the middle of its range):

    X''[s]  = exp(m - A_cs[s]) dt_s x_s
    G'[l,s] = (C_l . B_s) for s < l, (C_l . B_l) + D / dt_l on the diagonal, 0 above
    Y       = C (exp(m) S_in)^T + G' X''            y_l = exp(A_cs[l] - m) Y_l
    S_out   = exp(A_cs[last]) S_in + exp(A_cs[last] - m) X''^T B

(the decay exp(A_cs[l] - A_cs[s]) split into a row factor and a column factor at m). Evaluated
directly in numpy fp64, it must give the recurrence's y and final state."""
import math

import numpy as np
import pytest

import oracle


def factored_forward(x, dt, A, Bm, Cm, D, h0, blk=128):
    L, P = x.shape
    N = Bm.shape[1]
    S = h0.copy() if h0 is not None else np.zeros((P, N))
    y = np.zeros((L, P))
    for lo in range(0, L, blk):
        hi = min(L, lo + blk)
        acs = np.cumsum(dt[lo:hi] * A)
        m = 0.5 * (acs.max() + acs.min())
        Xpp = (np.exp(m - acs) * dt[lo:hi])[:, None] * x[lo:hi]
        Gp = np.tril(Cm[lo:hi] @ Bm[lo:hi].T)
        Gp[np.diag_indices(hi - lo)] += D / dt[lo:hi]
        Y = Cm[lo:hi] @ (math.exp(m) * S).T + Gp @ Xpp
        y[lo:hi] = np.exp(acs - m)[:, None] * Y
        S = math.exp(acs[-1]) * S + math.exp(acs[-1] - m) * Xpp.T @ Bm[lo:hi]
    return y, S


@pytest.mark.parametrize("L,with_h0,blk", [(300, True, 128), (128, False, 128), (77, True, 32), (1, True, 128)])
def test_factored_form_equals_recurrence(L, with_h0, blk):
    rng = np.random.default_rng(L + blk)
    P, N = 4, 6
    x = rng.standard_normal((L, P))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), L))
    A, D = -7.0, 0.8
    Bm = rng.standard_normal((L, N)) / math.sqrt(N)
    Cm = rng.standard_normal((L, N)) / math.sqrt(N)
    h0 = rng.standard_normal((P, N)) * 0.1 if with_h0 else None
    y, hf = factored_forward(x, dt, A, Bm, Cm, D, h0, blk)
    yr, hr = oracle.recurrent(x[None, :, None, :], dt[None, :, None], np.array([A]), Bm[None, :, None, :],
                              Cm[None, :, None, :], np.array([D]), h0[None, None] if h0 is not None else None)
    np.testing.assert_allclose(y, yr[0, :, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(hf, hr[0, 0], rtol=1e-10, atol=1e-12)


def test_reference_point_is_free():
    """Any m gives the same result in exact arithmetic; the kernel's choice (the middle of the
    range) only bounds the factors' magnitudes."""
    rng = np.random.default_rng(9)
    L, P, N = 128, 3, 5
    x, Bm, Cm = rng.standard_normal((L, P)), rng.standard_normal((L, N)), rng.standard_normal((L, N))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), L))
    acs = np.cumsum(dt * -5.0)
    outs = []
    for m in (acs.max(), 0.5 * (acs.max() + acs.min()), acs.min()):
        Xpp = (np.exp(m - acs) * dt)[:, None] * x
        outs.append(np.exp(acs - m)[:, None] * (np.tril(Cm @ Bm.T) @ Xpp))
    np.testing.assert_allclose(outs[0], outs[1], rtol=1e-10)
    np.testing.assert_allclose(outs[2], outs[1], rtol=1e-10)


def quarter_exact_forward(x, dt, A, Bm, Cm, D, h0, blk=128, q=32):
    """The head-pair kernel's exact form, per block: with mid_k the middle of quarter k's span of
    A_cs (bounds: the cumsum before the quarter and at its end),
        X'''[s]  = exp(mid_q(s) - A_cs[s]) dt_s x_s
        G'[l,s]  = (C_l . B_s) exp(A_cs[l] - mid_q(s))  for s <= l, 0 above
        B'[s]    = exp(A_cs[last] - A_cs[s]) dt_s B_s,   C~[l] = exp(A_cs[l]) C_l
        y        = C~ S_in^T + G' X''' + D x,            S_out = exp(A_cs[last]) S_in + x^T B'"""
    L, P = x.shape
    N = Bm.shape[1]
    S = h0.copy() if h0 is not None else np.zeros((P, N))
    y = np.zeros((L, P))
    for lo in range(0, L, blk):
        hi = min(L, lo + blk)
        n = hi - lo
        acs = np.cumsum(dt[lo:hi] * A)
        tot = acs[-1]
        quarter = np.arange(n) // q
        bounds = [0.0] + [acs[min(n, (k + 1) * q) - 1] for k in range((n + q - 1) // q)]
        mid = np.array([0.5 * (bounds[k] + bounds[k + 1]) for k in range(len(bounds) - 1)])
        X3 = (np.exp(mid[quarter] - acs) * dt[lo:hi])[:, None] * x[lo:hi]
        Gp = np.tril((Cm[lo:hi] @ Bm[lo:hi].T) * np.exp(acs[:, None] - mid[quarter][None, :]))
        Bp = (np.exp(tot - acs) * dt[lo:hi])[:, None] * Bm[lo:hi]
        Ct = np.exp(acs)[:, None] * Cm[lo:hi]
        y[lo:hi] = Ct @ S.T + Gp @ X3 + D * x[lo:hi]
        S = math.exp(tot) * S + x[lo:hi].T @ Bp
    return y, S


@pytest.mark.parametrize("L,A,dt_scale,zero_dt", [(300, -7.0, 1.0, False), (128, -16.0, 8.0, True),
                                                   (77, -3.0, 20.0, False), (1, -1.0, 1.0, False)])
def test_quarter_factored_exact_form_equals_recurrence(L, A, dt_scale, zero_dt):
    """Narrow and wide decays (one block here spans up to 343 of A_cs in natural log, 494 in
    the kernel's log2 units, far past the factored form's 192; one quarter up to 94) and zero
    step sizes, whose skip term comes from the raw x."""
    rng = np.random.default_rng(L + int(-A))
    P, N = 4, 6
    x = rng.standard_normal((L, P))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), L)) * dt_scale
    if zero_dt:
        dt[5] = 0.0
        dt[70] = 0.0
    D = 0.8
    Bm = rng.standard_normal((L, N)) / math.sqrt(N)
    Cm = rng.standard_normal((L, N)) / math.sqrt(N)
    h0 = rng.standard_normal((P, N)) * 0.1
    y, hf = quarter_exact_forward(x, dt, A, Bm, Cm, D, h0)
    yr, hr = oracle.recurrent(x[None, :, None, :], dt[None, :, None], np.array([A]), Bm[None, :, None, :],
                              Cm[None, :, None, :], np.array([D]), h0[None, None])
    np.testing.assert_allclose(y, yr[0, :, 0], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(hf, hr[0, 0], rtol=1e-9, atol=1e-12)
