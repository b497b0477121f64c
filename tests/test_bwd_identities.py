"""The chunked backward's decomposition, checked on the CPU against the oracle's token-by-token
adjoint. The tensor-core backward forms the log-decay gradient of token t inside its chunk as

    G_t = sum_{u<t} (K_u - R_u) + sum_{l>=t} T_l + sum_{s<t} U_s + exp(A_cs[Q-1]) <Gend, S_in>

with M[l,s] = (C_l.B_s)(dy_l.x_s) dt_s exp(A_cs[l] - A_cs[s]) for l > s in the chunk,
K_s = sum_l M[l,s], R_l = sum_s M[l,s], T_l = exp(A_cs[l]) dy_l^T S_in C_l,
U_s = exp(A_cs[Q-1] - A_cs[s]) dt_s x_s^T Gend B_s, and then ddt_t = A G_t + x_t . u_t,
dA = sum_t dt_t G_t. Here those formulas are evaluated directly in numpy (fp64), from the
oracle's chunk states, and must give the oracle's ddt and dA."""
import math

import numpy as np
import pytest

import oracle


def chunk_local_ddt(x, dt, A, Bm, Cm, h0, dy, dhf, Q, mistake=None):
    """One (batch row, head) stream, G = H = 1: ddt [L] and dA from the chunk-local formulas."""
    L, P = x.shape
    N = Bm.shape[1]
    nc = (L + Q - 1) // Q
    a = dt * A
    r = oracle.chunked(x[None, :, None, :], dt[None, :, None], np.array([A]), Bm[None, :, None, :],
                       Cm[None, :, None, :], None, h0[None, None] if h0 is not None else None, chunk=Q)
    S_in = r["S_in"][0, 0]                      # [nc, P, N]
    # reverse state pass: Gend[c] = gradient of the state leaving chunk c
    Gend = np.zeros((nc, P, N))
    run = dhf.copy() if dhf is not None else np.zeros((P, N))
    for c in range(nc - 1, -1, -1):
        lo, hi = c * Q, min(L, (c + 1) * Q)
        acs = np.cumsum(a[lo:hi])
        Gend[c] = run
        Rc = np.einsum("l,lp,ln->pn", np.exp(acs), dy[lo:hi], Cm[lo:hi])
        run = math.exp(acs[-1]) * run + Rc
    ddt = np.zeros(L)
    dA = 0.0
    for c in range(nc):
        lo, hi = c * Q, min(L, (c + 1) * Q)
        q = hi - lo
        acs = np.cumsum(a[lo:hi])
        xs, dts, Bs, Cs, dys = x[lo:hi], dt[lo:hi], Bm[lo:hi], Cm[lo:hi], dy[lo:hi]
        dec = np.exp(acs[:, None] - acs[None, :])                     # [l, s]
        strict = np.tril(np.ones((q, q), dtype=bool), k=-1)           # l > s
        M = np.where(strict, (Cs @ Bs.T) * (dys @ xs.T) * dts[None, :] * np.where(strict, dec, 0.0), 0.0)
        K = M.sum(axis=0)                                            # over l, per s
        R = M.sum(axis=1)                                            # over s, per l
        T = np.exp(acs) * np.einsum("lp,pn,ln->l", dys, S_in[c], Cs)
        U = np.exp(acs[-1] - acs) * dts * np.einsum("sp,pn,sn->s", xs, Gend[c], Bs)
        E = math.exp(acs[-1]) * np.sum(Gend[c] * S_in[c])
        KR_excl = np.cumsum(K - R) if mistake == "inclusive_pairs" else np.concatenate([[0.0], np.cumsum(K - R)[:-1]])
        if mistake == "no_pairs":
            KR_excl = np.zeros(q)
        if mistake == "no_state_product":
            E = 0.0
        U_excl = np.concatenate([[0.0], np.cumsum(U)[:-1]])
        T_incl_suffix = np.cumsum(T[::-1])[::-1]
        G = KR_excl + U_excl + T_incl_suffix + E
        # u_t = sum_{l >= t} exp(acs_l - acs_t) (C_l . B_t) dy_l + exp(acs_end - acs_t) Gend B_t
        causal = np.tril(np.ones((q, q), dtype=bool))                 # l >= s
        W1 = np.where(causal, (Cs @ Bs.T) * np.where(causal, dec, 0.0), 0.0)
        u = W1.T @ dys + np.exp(acs[-1] - acs)[:, None] * (Bs @ Gend[c].T)
        ddt[lo:hi] = A * G + np.sum(xs * u, axis=1)
        dA += float(np.sum(dts * G))
    return ddt, dA


@pytest.mark.parametrize("Q,L,with_h0,with_dhf", [(8, 37, True, True), (5, 20, False, True), (16, 16, True, False),
                                                  (64, 70, True, True)])
def test_chunk_local_log_decay_gradient_matches_adjoint(Q, L, with_h0, with_dhf):
    rng = np.random.default_rng(Q * 100 + L)
    P, N = 3, 4
    x = rng.standard_normal((L, P))
    dt = np.exp(rng.uniform(math.log(1e-2), math.log(0.5), L))
    A = -3.0
    Bm = rng.standard_normal((L, N)) / 2
    Cm = rng.standard_normal((L, N)) / 2
    h0 = rng.standard_normal((P, N)) if with_h0 else None
    dy = rng.standard_normal((L, P))
    dhf = rng.standard_normal((P, N)) if with_dhf else None
    ddt, dA = chunk_local_ddt(x, dt, A, Bm, Cm, h0, dy, dhf, Q)
    ref = oracle.backward(x[None, :, None, :], dt[None, :, None], np.array([A]), Bm[None, :, None, :],
                          Cm[None, :, None, :], None, h0[None, None] if h0 is not None else None,
                          dy[None, :, None, :], dhf[None, None] if dhf is not None else None)
    np.testing.assert_allclose(ddt, ref["ddt"][0, :, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dA, ref["dA"][0], rtol=1e-10)


@pytest.mark.parametrize("mistake", ["inclusive_pairs", "no_pairs", "no_state_product"])
def test_planted_mistakes_in_the_decomposition_are_caught(mistake):
    rng = np.random.default_rng(3)
    L, P, N, Q = 37, 3, 4, 8
    x = rng.standard_normal((L, P))
    dt = np.exp(rng.uniform(math.log(1e-2), math.log(0.5), L))
    Bm, Cm = rng.standard_normal((L, N)) / 2, rng.standard_normal((L, N)) / 2
    h0, dy, dhf = rng.standard_normal((P, N)), rng.standard_normal((L, P)), rng.standard_normal((P, N))
    ddt, _ = chunk_local_ddt(x, dt, -3.0, Bm, Cm, h0, dy, dhf, Q, mistake)
    ref = oracle.backward(x[None, :, None, :], dt[None, :, None], np.array([-3.0]), Bm[None, :, None, :],
                          Cm[None, :, None, :], None, h0[None, None], dy[None, :, None, :], dhf[None, None])
    err = np.max(np.abs(ddt - ref["ddt"][0, :, 0])) / np.max(np.abs(ref["ddt"]))
    assert err > 1e-3

