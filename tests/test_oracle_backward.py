"""Pins of the oracle's backward pass (the gradient of sum(dy * y) + sum(dh_final * h_final)
through the recurrence) against facts that do not come from the backward itself:
central finite differences of the forward (both the recurrence and the masked quadratic
form), a closed form, and planted mistakes that those checks must catch."""
import math

import numpy as np
import pytest

import oracle

NAMES = ("x", "dt", "A", "Bm", "Cm", "D", "h0")
GRAD = {"x": "dx", "dt": "ddt", "A": "dA", "Bm": "dB", "Cm": "dC", "D": "dD", "h0": "dh0"}


def rand_problem(rng, Bsz=2, L=9, H=4, P=2, G=2, N=3):
    x = rng.standard_normal((Bsz, L, H, P))
    dt = np.exp(rng.uniform(math.log(1e-2), math.log(0.5), (Bsz, L, H)))
    A = -np.exp(rng.uniform(0, math.log(16), H))
    Bm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    Cm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((Bsz, H, P, N))
    dy = rng.standard_normal((Bsz, L, H, P))
    dhf = rng.standard_normal((Bsz, H, P, N))
    return dict(x=x, dt=dt, A=A, Bm=Bm, Cm=Cm, D=D, h0=h0), dy, dhf


def loss(forward, inp, dy, dhf):
    y, hf = forward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["D"], inp["h0"])
    return float(np.sum(dy * y) + (np.sum(dhf * hf) if dhf is not None else 0.0))


def finite_difference(forward, inp, dy, dhf, name, eps=1e-6):
    """Central difference of the loss for every element of one input."""
    base = inp[name]
    g = np.empty_like(base)
    for idx in np.ndindex(base.shape):
        saved = base[idx]
        base[idx] = saved + eps
        lp = loss(forward, inp, dy, dhf)
        base[idx] = saved - eps
        lm = loss(forward, inp, dy, dhf)
        base[idx] = saved
        g[idx] = (lp - lm) / (2 * eps)
    return g


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


@pytest.mark.parametrize("seed,with_dhf", [(0, True), (1, False)])
def test_backward_matches_finite_differences_of_recurrence(seed, with_dhf):
    rng = np.random.default_rng(seed)
    inp, dy, dhf = rand_problem(rng)
    dhf = dhf if with_dhf else None
    got = oracle.backward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["D"], inp["h0"],
                          dy, dhf, seg=4)
    for name in NAMES:
        fd = finite_difference(oracle.recurrent, inp, dy, dhf, name)
        assert rel(got[GRAD[name]], fd) < 1e-7, name


def test_backward_matches_finite_differences_of_quadratic_form():
    """The same check against the O(L^2) masked-matrix form of the forward, which shares
    no code with the recurrence."""
    rng = np.random.default_rng(2)
    inp, dy, dhf = rand_problem(rng, Bsz=1, L=7, H=2, P=2, G=1, N=3)
    got = oracle.backward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["D"], inp["h0"],
                          dy, dhf, seg=3)
    for name in NAMES:
        fd = finite_difference(oracle.quadratic, inp, dy, dhf, name)
        assert rel(got[GRAD[name]], fd) < 1e-7, name


def test_backward_without_skip_and_initial_state():
    """D = None and h0 = None are a zero skip and a zero initial state; dh0 is still the
    gradient for that zero state (checked by differences around h0 = 0)."""
    rng = np.random.default_rng(3)
    inp, dy, dhf = rand_problem(rng, Bsz=1, L=6, H=2, P=2, G=1, N=2)
    got = oracle.backward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], None, None, dy, dhf)
    inp0 = dict(inp, D=np.zeros_like(inp["D"]), h0=np.zeros_like(inp["h0"]))
    ref = oracle.backward(inp0["x"], inp0["dt"], inp0["A"], inp0["Bm"], inp0["Cm"], inp0["D"],
                          inp0["h0"], dy, dhf)
    for k in ("dx", "ddt", "dA", "dB", "dC", "dh0"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-13, atol=1e-13)
    fd = finite_difference(oracle.recurrent, inp0, dy, dhf, "h0")
    assert rel(got["dh0"], fd) < 1e-7


@pytest.mark.parametrize("seg", [1, 2, 5, 64])
def test_segment_length_does_not_change_gradients(seg):
    """The reverse sweep recomputes states per segment; the segment length is a storage
    choice and must not change the result beyond rounding."""
    rng = np.random.default_rng(4)
    inp, dy, dhf = rand_problem(rng, L=23)
    args = (inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["D"], inp["h0"], dy, dhf)
    ref = oracle.backward(*args, seg=23)
    got = oracle.backward(*args, seg=seg)
    for k in ref:
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-12, atol=1e-12)


def test_closed_form_initial_state_only():
    """x = 0 and dy nonzero only at the last token T: with c_t = dt_0 + ... + dt_t,
      loss = e^{A c_T} dy_T^T h0 C_T, so
      dh0 = e^{A c_T} dy_T C_T^T, dC_T = e^{A c_T} h0^T dy_T, dC_t = 0 (t < T),
      dA = c_T loss, ddt_t = A loss (every t), dB = 0,
      dx_t = dt_t e^{A (c_T - c_t)} (C_T . B_t) dy_T + D dy_t."""
    rng = np.random.default_rng(6)
    L, P, N = 11, 3, 4
    dt = np.exp(rng.uniform(math.log(1e-2), math.log(0.5), (1, L, 1)))
    A = np.array([-2.5])
    Bm = rng.standard_normal((1, L, 1, N))
    Cm = rng.standard_normal((1, L, 1, N))
    D = np.array([0.7])
    h0 = rng.standard_normal((1, 1, P, N))
    x = np.zeros((1, L, 1, P))
    dy = np.zeros((1, L, 1, P))
    dy[0, L - 1, 0] = rng.standard_normal(P)
    got = oracle.backward(x, dt, A, Bm, Cm, D, h0, dy, None, seg=4)
    c = np.cumsum(dt[0, :, 0])
    e = math.exp(A[0] * c[-1])
    dyT, CT = dy[0, -1, 0], Cm[0, -1, 0]
    lossv = e * dyT @ h0[0, 0] @ CT
    np.testing.assert_allclose(got["dh0"][0, 0], e * np.outer(dyT, CT), rtol=1e-12)
    want_dC = np.zeros((L, N))
    want_dC[-1] = e * h0[0, 0].T @ dyT
    np.testing.assert_allclose(got["dC"][0, :, 0], want_dC, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(got["dA"][0], c[-1] * lossv, rtol=1e-12)
    np.testing.assert_allclose(got["ddt"][0, :, 0], np.full(L, A[0] * lossv), rtol=1e-11)
    np.testing.assert_allclose(got["dB"], 0.0, atol=0)
    want_dx = np.array([dt[0, t, 0] * math.exp(A[0] * (c[-1] - c[t])) * (CT @ Bm[0, t, 0]) * dyT
                        for t in range(L)])
    want_dx[-1] += D[0] * dyT
    np.testing.assert_allclose(got["dx"][0, :, 0], want_dx, rtol=1e-12, atol=1e-15)


# ---- planted mistakes: a plain Python adjoint, correct or with one mistake planted ----------

def _py_adjoint(inp, dy, dhf, mistake=None):
    x, dt, A, Bm, Cm, D, h0 = (inp[k] for k in NAMES)
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2:]
    out = {"dx": np.zeros_like(x), "ddt": np.zeros_like(dt), "dA": np.zeros(H),
           "dB": np.zeros_like(Bm), "dC": np.zeros_like(Cm), "dD": np.zeros(H),
           "dh0": np.zeros_like(h0)}
    for b in range(Bsz):
        for h in range(H):
            g = h // (H // G)
            S = [h0[b, h].copy()]
            for t in range(L):
                a = math.exp(dt[b, t, h] * A[h])
                S.append(a * S[-1] + dt[b, t, h] * np.outer(x[b, t, h], Bm[b, t, g]))
            Gb = dhf[b, h].copy()
            for t in reversed(range(L)):
                a = math.exp(dt[b, t, h] * A[h])
                if mistake != "decay_before_output":
                    Gb = Gb + np.outer(dy[b, t, h], Cm[b, t, g])
                out["dC"][b, t, g] += (S[t] if mistake == "dC_previous_state" else S[t + 1]).T @ dy[b, t, h]
                out["dD"][h] += dy[b, t, h] @ x[b, t, h]
                gB = Gb @ Bm[b, t, g]
                out["dx"][b, t, h] = D[h] * dy[b, t, h] + dt[b, t, h] * gB
                out["dB"][b, t, g] += dt[b, t, h] * Gb.T @ x[b, t, h]
                prev = S[t + 1] if mistake == "state_after_token" else S[t]
                inner = np.sum(Gb * prev)
                out["ddt"][b, t, h] = x[b, t, h] @ gB + A[h] * a * inner
                out["dA"][h] += dt[b, t, h] * a * inner
                Gb = a * Gb
                if mistake == "decay_before_output":
                    Gb = Gb + a * np.outer(dy[b, t, h], Cm[b, t, g])
            out["dh0"][b, h] = Gb
    return out


def test_python_adjoint_agrees_with_oracle():
    rng = np.random.default_rng(7)
    inp, dy, dhf = rand_problem(rng)
    ref = oracle.backward(*(inp[k] for k in NAMES), dy, dhf, seg=2)
    got = _py_adjoint(inp, dy, dhf)
    for k in ref:
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mistake,name", [("state_after_token", "dt"), ("state_after_token", "A"),
                                          ("decay_before_output", "x"), ("decay_before_output", "Bm"),
                                          ("dC_previous_state", "Cm")])
def test_planted_mistakes_are_caught(mistake, name):
    rng = np.random.default_rng(8)
    inp, dy, dhf = rand_problem(rng, Bsz=1, L=6, H=2, P=2, G=1, N=2)
    bad = _py_adjoint(inp, dy, dhf, mistake)
    fd = finite_difference(oracle.recurrent, inp, dy, dhf, name)
    assert rel(bad[GRAD[name]], fd) > 1e-3
