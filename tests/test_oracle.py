"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
a hand-worked example, closed forms, library routines for special cases, and the
equivalences the SSD pages state (recurrence = masked quadratic form = chunked
algorithm; A = 0 is linear attention; state passing across a split)."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_problem(rng, Bsz=2, L=37, H=4, P=3, G=2, N=5, h0=True, A_scale=1.0):
    x = rng.standard_normal((Bsz, L, H, P))
    dt = np.exp(rng.uniform(math.log(1e-2), math.log(0.5), (Bsz, L, H)))
    A = -np.exp(rng.uniform(0, math.log(16), H)) * A_scale
    Bm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    Cm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    D = rng.standard_normal(H)
    h = rng.standard_normal((Bsz, H, P, N)) if h0 else None
    return x, dt, A, Bm, Cm, D, h


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---- hand-worked example (tests/golden) -------------------------------------------------

def test_handworked_example():
    g = json.load(open(os.path.join(GOLDEN, "handworked_decay_half.json")))
    i, e = g["inputs"], g["expected"]
    L = len(i["x"])
    x = np.array(i["x"]).reshape(1, L, 1, 1)
    dt = np.array(i["dt"]).reshape(1, L, 1)
    A = np.array([i["A"]])
    Bm = np.array(i["B"]).reshape(1, L, 1, 2)
    Cm = np.array(i["C"]).reshape(1, L, 1, 2)
    D = np.array([i["D"]])
    h0 = np.array(i["h0"]).reshape(1, 1, 1, 2)
    y, hf, st = oracle.recurrent(x, dt, A, Bm, Cm, D, h0, store_states=True)
    tol = g["tolerance"]
    np.testing.assert_allclose(y.ravel(), e["y"], atol=tol, rtol=0)
    np.testing.assert_allclose(hf.ravel(), e["h_final"], atol=tol, rtol=0)
    np.testing.assert_allclose(st.reshape(L, 2), e["states"], atol=tol, rtol=0)
    # the other forms reproduce it too
    yq, hq = oracle.quadratic(x, dt, A, Bm, Cm, D, h0)
    np.testing.assert_allclose(yq.ravel(), e["y"], atol=tol, rtol=0)
    np.testing.assert_allclose(hq.ravel(), e["h_final"], atol=tol, rtol=0)
    for Q in (1, 2, 3):
        r = oracle.chunked(x, dt, A, Bm, Cm, D, h0, chunk=Q)
        np.testing.assert_allclose(r["y"].ravel(), e["y"], atol=tol, rtol=0)
    # verify + select
    yv, so = oracle.verify(h0, x, dt, A, Bm, Cm, D)
    np.testing.assert_allclose(yv.ravel(), e["y"], atol=tol, rtol=0)
    for a, want in e["kept"].items():
        kept = oracle.select_state(h0, so, np.array([int(a)], dtype=np.int32))
        np.testing.assert_allclose(kept.ravel(), want, atol=tol, rtol=0)


# ---- closed forms -----------------------------------------------------------------------

@pytest.mark.parametrize("delta,alpha", [(0.05, -3.0), (0.3, -0.7), (1.0, -0.01)])
def test_closed_form_geometric_series(delta, alpha):
    """P=N=1, x=B=C=1, constant dt and A: h_t = dt (1 - r^(t+1)) / (1 - r), r = exp(dt A)."""
    L = 200
    x = np.ones((1, L, 1, 1))
    dt = np.full((1, L, 1), delta)
    A = np.array([alpha])
    Bm = np.ones((1, L, 1, 1))
    Cm = np.ones((1, L, 1, 1))
    y, hf = oracle.recurrent(x, dt, A, Bm, Cm)
    r = math.exp(delta * alpha)
    t = np.arange(L)
    want = delta * (1 - r ** (t + 1)) / (1 - r)
    assert rel(y.ravel(), want) < 1e-12
    assert abs(hf.ravel()[0] - want[-1]) < 1e-12 * abs(want[-1])


def test_zero_decay_rate_is_cumulative_sum():
    """A = 0, dt = 1, B = C = 1: the state is the running sum of x (numpy cumsum)."""
    rng = np.random.default_rng(11)
    L, P = 500, 4
    x = rng.standard_normal((1, L, 1, P))
    ones = np.ones((1, L, 1, 1))
    y, hf = oracle.recurrent(x, np.ones((1, L, 1)), np.zeros(1), ones, ones, np.array([0.0]))
    np.testing.assert_allclose(y[0, :, 0, :], np.cumsum(x[0, :, 0, :], axis=0), rtol=1e-12, atol=1e-12)


def test_memoryless_limit():
    """A very negative decay rate forgets the past: h_t = dt_t x_t B_t^T and
    y_t = dt_t (C_t . B_t) x_t + D x_t (catches an off-by-one between B, C and t)."""
    rng = np.random.default_rng(5)
    x, dt, A, Bm, Cm, D, _ = rand_problem(rng, L=20, h0=False)
    A = np.full_like(A, -1e6)
    y, hf = oracle.recurrent(x, dt, A, Bm, Cm, D)
    H, G = x.shape[2], Bm.shape[2]
    for h in range(H):
        g = h // (H // G)
        cb = np.sum(Cm[:, :, g, :] * Bm[:, :, g, :], axis=-1)  # [B, L]
        want = (dt[:, :, h] * cb)[..., None] * x[:, :, h, :] + D[h] * x[:, :, h, :]
        np.testing.assert_allclose(y[:, :, h, :], want, rtol=1e-12, atol=1e-12)
        want_h = dt[:, -1, h, None, None] * x[:, -1, h, :, None] * Bm[:, -1, g, None, :]
        np.testing.assert_allclose(hf[:, h], want_h, rtol=1e-12, atol=1e-12)


def test_single_token_from_state():
    """L = 1 from h0: y_0 = C_0 (e^{dt A} h0 + dt x_0 B_0^T) + D x_0, written element-wise."""
    rng = np.random.default_rng(8)
    x, dt, A, Bm, Cm, D, h0 = rand_problem(rng, Bsz=1, L=1, H=2, P=2, G=1, N=3)
    y, hf = oracle.recurrent(x, dt, A, Bm, Cm, D, h0)
    for h in range(2):
        for p in range(2):
            s = [math.exp(dt[0, 0, h] * A[h]) * h0[0, h, p, n] + dt[0, 0, h] * x[0, 0, h, p] * Bm[0, 0, 0, n]
                 for n in range(3)]
            yy = sum(s[n] * Cm[0, 0, 0, n] for n in range(3)) + D[h] * x[0, 0, h, p]
            assert abs(y[0, 0, h, p] - yy) < 1e-13
            np.testing.assert_allclose(hf[0, h, p], s, rtol=1e-13, atol=1e-15)


# ---- equivalences the pages state --------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_recurrence_equals_quadratic_form(seed):
    rng = np.random.default_rng(seed)
    prob = rand_problem(rng, Bsz=2, L=29, H=4, P=3, G=2, N=5)
    y1, h1 = oracle.recurrent(*prob)
    y2, h2 = oracle.quadratic(*prob)
    assert rel(y1, y2) < 1e-12
    assert rel(h1, h2) < 1e-12


def test_zero_decay_rate_is_causal_linear_attention():
    rng = np.random.default_rng(3)
    x, dt, A, Bm, Cm, D, _ = rand_problem(rng, Bsz=2, L=33, H=4, P=3, G=4, N=6, h0=False)
    y1, _ = oracle.recurrent(x, dt, np.zeros_like(A), Bm, Cm, D)
    y2 = oracle.linear_attention(x, dt, Bm, Cm, D)
    assert rel(y1, y2) < 1e-12


@pytest.mark.parametrize("Q", [1, 2, 7, 8, 16, 64, 75, 200])
def test_chunked_equals_recurrence(Q):
    """Chunk-size invariance, ragged last chunk included (L = 75)."""
    rng = np.random.default_rng(4)
    prob = rand_problem(rng, Bsz=2, L=75, H=4, P=3, G=2, N=5)
    y1, h1 = oracle.recurrent(*prob)
    r = oracle.chunked(*prob, chunk=Q)
    assert rel(r["y"], y1) < 1e-11
    assert rel(r["h_final"], h1) < 1e-11


def test_chunk_states_are_states_at_chunk_boundaries():
    """S_in[c] is the recurrence's state after token c*Q - 1 (h0 for c = 0)."""
    rng = np.random.default_rng(9)
    prob = rand_problem(rng, Bsz=1, L=40, H=2, P=2, G=1, N=3)
    _, _, st = oracle.recurrent(*prob, store_states=True)
    Q = 8
    r = oracle.chunked(*prob, chunk=Q)
    h0 = prob[-1]
    np.testing.assert_allclose(r["S_in"][:, :, 0], h0, rtol=1e-12, atol=1e-14)
    for c in range(1, 5):
        np.testing.assert_allclose(r["S_in"][:, :, c], st[:, c * Q - 1], rtol=1e-11, atol=1e-13)
    # a chunk state from a zero start equals the recurrence run on that chunk alone with h0 = 0
    x, dt, A, Bm, Cm, D, _ = prob
    sl = slice(16, 24)
    _, hc = oracle.recurrent(x[:, sl], dt[:, sl], A, Bm[:, sl], Cm[:, sl], D, None)
    np.testing.assert_allclose(r["states"][:, :, 2], hc, rtol=1e-11, atol=1e-13)


def test_split_with_carried_state_equals_unsplit():
    rng = np.random.default_rng(6)
    x, dt, A, Bm, Cm, D, h0 = rand_problem(rng, Bsz=2, L=64, H=4, P=3, G=2, N=5)
    y, hf = oracle.recurrent(x, dt, A, Bm, Cm, D, h0)
    L1 = 23
    ya, ha = oracle.recurrent(x[:, :L1], dt[:, :L1], A, Bm[:, :L1], Cm[:, :L1], D, h0)
    yb, hb = oracle.recurrent(x[:, L1:], dt[:, L1:], A, Bm[:, L1:], Cm[:, L1:], D, ha)
    assert rel(np.concatenate([ya, yb], axis=1), y) < 1e-13
    assert rel(hb, hf) < 1e-13


def test_linearity_in_input_and_initial_state():
    rng = np.random.default_rng(7)
    x, dt, A, Bm, Cm, D, h0 = rand_problem(rng)
    y, hf = oracle.recurrent(x, dt, A, Bm, Cm, D, h0)
    y1, h1 = oracle.recurrent(x, dt, A, Bm, Cm, D, None)
    y2, h2 = oracle.recurrent(np.zeros_like(x), dt, A, Bm, Cm, D, h0)
    assert rel(y1 + y2, y) < 1e-13
    assert rel(h1 + h2, hf) < 1e-13


def test_groups_equal_replicated_heads():
    rng = np.random.default_rng(10)
    x, dt, A, Bm, Cm, D, h0 = rand_problem(rng, H=6, G=2)
    y, hf = oracle.recurrent(x, dt, A, Bm, Cm, D, h0)
    Br, Cr = np.repeat(Bm, 3, axis=2), np.repeat(Cm, 3, axis=2)
    yr, hr = oracle.recurrent(x, dt, A, Br, Cr, D, h0)
    assert rel(yr, y) < 1e-15 and rel(hr, hf) < 1e-15


# ---- verify / select ------------------------------------------------------------------

def test_verify_states_equal_prefix_final_states():
    rng = np.random.default_rng(12)
    x, dt, A, Bm, Cm, D, h0 = rand_problem(rng, Bsz=3, L=8, H=4, P=3, G=2, N=5)
    yv, so = oracle.verify(h0, x, dt, A, Bm, Cm, D)
    for k in range(8):
        yk, hk = oracle.recurrent(x[:, :k + 1], dt[:, :k + 1], A, Bm[:, :k + 1], Cm[:, :k + 1], D, h0)
        np.testing.assert_array_equal(so[:, k], hk)
        np.testing.assert_array_equal(yv[:, k], yk[:, k])


def test_select_state_indexing():
    rng = np.random.default_rng(13)
    Bsz, K, H, P, N = 9, 8, 2, 3, 4
    h0 = rng.standard_normal((Bsz, H, P, N))
    so = rng.standard_normal((Bsz, K, H, P, N))
    acc = np.arange(Bsz, dtype=np.int32)  # 0..8 covers a = 0 and a = K
    kept = oracle.select_state(h0, so, acc)
    np.testing.assert_array_equal(kept[0], h0[0])
    for b in range(1, Bsz):
        np.testing.assert_array_equal(kept[b], so[b, b - 1])
    with pytest.raises(ValueError):
        oracle.select_state(h0, so, np.full(Bsz, K + 1, dtype=np.int32))


def test_thread_count_does_not_change_result():
    rng = np.random.default_rng(14)
    prob = rand_problem(rng, Bsz=3, L=50, H=8, P=4, G=2, N=8)
    y1, h1 = oracle.recurrent(*prob, threads=1)
    y4, h4 = oracle.recurrent(*prob, threads=4)
    np.testing.assert_array_equal(y1, y4)
    np.testing.assert_array_equal(h1, h4)


# ---- planted mistakes: each must be caught by one of the pins above -----------------------

def _mutant_add_then_decay(x, dt, A, Bm, Cm, D, h0):
    """Wrong order: S = exp(dt A) (S + dt x B^T)."""
    Bsz, L, H, P = x.shape
    y = np.zeros_like(x)
    for b in range(Bsz):
        for h in range(H):
            S = np.zeros((P, Bm.shape[3])) if h0 is None else h0[b, h].copy()
            for t in range(L):
                g = h // (H // Bm.shape[2])
                S = math.exp(dt[b, t, h] * A[h]) * (S + dt[b, t, h] * np.outer(x[b, t, h], Bm[b, t, g]))
                y[b, t, h] = S @ Cm[b, t, g] + D[h] * x[b, t, h]
    return y


def _mutant_previous_C(x, dt, A, Bm, Cm, D, h0):
    """Wrong index: output read with C_{t-1}."""
    Cs = np.concatenate([Cm[:, :1], Cm[:, :-1]], axis=1)
    return oracle.recurrent(x, dt, A, Bm, Cs, D, h0)[0]


@pytest.mark.parametrize("mutant", [_mutant_add_then_decay, _mutant_previous_C])
def test_planted_mistakes_are_caught(mutant):
    g = json.load(open(os.path.join(GOLDEN, "handworked_decay_half.json")))
    i, e = g["inputs"], g["expected"]
    L = len(i["x"])
    args = (np.array(i["x"]).reshape(1, L, 1, 1), np.array(i["dt"]).reshape(1, L, 1),
            np.array([i["A"]]), np.array(i["B"]).reshape(1, L, 1, 2),
            np.array(i["C"]).reshape(1, L, 1, 2), np.array([i["D"]]),
            np.array(i["h0"]).reshape(1, 1, 1, 2))
    y = mutant(*args)
    assert np.max(np.abs(y.ravel() - np.array(e["y"]))) > 1e-3
