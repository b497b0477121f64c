"""Pins of the oracle's Mamba-2 block operations (convolution + split + step size, gated grouped
RMSNorm, the mixer composition) against library routines, closed forms and invariants."""
import math

import numpy as np
import pytest
from scipy.special import expit

import oracle


def conv_problem(rng, Bsz=2, L=37, H=2, P=4, G=1, N=3, W=4, bias=True):
    Cc = H * P + 2 * G * N
    xbc = rng.standard_normal((Bsz, L, Cc))
    dt_raw = rng.standard_normal((Bsz, L, H))
    w = rng.standard_normal((Cc, W))
    b = rng.standard_normal(Cc) if bias else None
    dtb = rng.standard_normal(H)
    return xbc, dt_raw, w, b, dtb


@pytest.mark.parametrize("W", [1, 2, 3, 4])
def test_conv_equals_numpy_convolve(W):
    """Each channel is numpy's full convolution with the reversed taps, cut to the first L
    outputs (causal), plus the bias, through SiLU (scipy's logistic)."""
    rng = np.random.default_rng(W)
    H, P, G, N = 2, 4, 1, 3
    xbc, dt_raw, w, b, dtb = conv_problem(rng, W=W)
    x, Bm, Cm, dt = oracle.conv_split(xbc, dt_raw, w, b, dtb, nheads=H, headdim=P, ngroups=G, dstate=N)
    Bsz, L, Cc = xbc.shape
    act = np.concatenate([x.reshape(Bsz, L, H * P), Bm.reshape(Bsz, L, G * N), Cm.reshape(Bsz, L, G * N)], axis=-1)
    for bb in range(Bsz):
        for c in range(Cc):
            pre = np.convolve(xbc[bb, :, c], w[c, ::-1])[:L] + b[c]
            np.testing.assert_allclose(act[bb, :, c], pre * expit(pre), rtol=1e-12, atol=1e-14)


def test_conv_impulse_response():
    """A unit impulse at token t0 in channel c gives silu(b_c + w[c, W-1-(t-t0)]) for
    t0 <= t < t0 + W and silu(b_c) elsewhere; no other channel moves."""
    H, P, G, N, W, L, t0 = 1, 2, 1, 2, 4, 12, 5
    Cc = H * P + 2 * G * N
    rng = np.random.default_rng(3)
    w = rng.standard_normal((Cc, W))
    b = rng.standard_normal(Cc)
    for c in range(Cc):
        xbc = np.zeros((1, L, Cc))
        xbc[0, t0, c] = 1.0
        x, Bm, Cm, _ = oracle.conv_split(xbc, np.zeros((1, L, H)), w, b, None, nheads=H, headdim=P, ngroups=G,
                                         dstate=N)
        act = np.concatenate([x.reshape(1, L, -1), Bm.reshape(1, L, -1), Cm.reshape(1, L, -1)], axis=-1)[0]
        for t in range(L):
            for cc in range(Cc):
                pre = b[cc]
                if cc == c and t0 <= t < t0 + W:
                    pre += w[c, W - 1 - (t - t0)]
                want = pre / (1 + math.exp(-pre))
                assert abs(act[t, cc] - want) < 1e-14


def test_split_order_and_step_size():
    """Channels [0, HP) are x (head-major), then B, then C; dt = softplus(dt_raw + bias) with
    softplus(v) = log(1 + e^v) (numpy logaddexp)."""
    rng = np.random.default_rng(4)
    H, P, G, N = 2, 3, 2, 2
    xbc, dt_raw, w, b, dtb = conv_problem(rng, Bsz=1, L=5, H=H, P=P, G=G, N=N, W=1)
    w[:] = 1.0
    b[:] = 0.0
    x, Bm, Cm, dt = oracle.conv_split(xbc, dt_raw, w, b, dtb, nheads=H, headdim=P, ngroups=G, dstate=N)
    s = xbc * expit(xbc)
    np.testing.assert_allclose(x[0, :, 1, 2], s[0, :, 1 * P + 2], rtol=1e-13)
    np.testing.assert_allclose(Bm[0, :, 1, 0], s[0, :, H * P + 1 * N + 0], rtol=1e-13)
    np.testing.assert_allclose(Cm[0, :, 0, 1], s[0, :, H * P + G * N + 1], rtol=1e-13)
    np.testing.assert_allclose(dt, np.logaddexp(0.0, dt_raw + dtb), rtol=1e-13)
    assert abs(oracle.softplus(np.array([0.0]))[0] - math.log(2.0)) < 1e-15


def test_rmsnorm_unit_rms_per_group():
    """weight = 1, eps = 0: every group of the output has mean square 1."""
    rng = np.random.default_rng(5)
    y, z = rng.standard_normal((3, 7, 256)), rng.standard_normal((3, 7, 256))
    out = oracle.gated_rmsnorm(y, z, np.ones(256), ngroups=4, eps=0.0)
    ms = np.mean(out.reshape(3, 7, 4, 64) ** 2, axis=-1)
    np.testing.assert_allclose(ms, 1.0, rtol=1e-12)


def test_rmsnorm_invariances():
    """eps = 0: scaling y by a positive constant changes nothing; a constant gate z = c on every
    channel multiplies g by silu(c), which the norm removes; groups are independent."""
    rng = np.random.default_rng(6)
    y, z, w = rng.standard_normal((2, 256)), rng.standard_normal((2, 256)), rng.standard_normal(256)
    a = oracle.gated_rmsnorm(y, z, w, ngroups=4, eps=0.0)
    np.testing.assert_allclose(oracle.gated_rmsnorm(3.7 * y, z, w, ngroups=4, eps=0.0), a, rtol=1e-12)
    c = oracle.gated_rmsnorm(y, np.full_like(z, 1.3), w, ngroups=4, eps=0.0)
    ref = y.reshape(2, 4, 64)
    ref = (ref / np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))).reshape(2, 256) * w
    np.testing.assert_allclose(c, ref, rtol=1e-12)
    y2 = y.copy()
    y2[:, 64:128] *= -5.0
    b = oracle.gated_rmsnorm(y2, z, w, ngroups=4, eps=0.0)
    np.testing.assert_allclose(b[:, :64], a[:, :64], rtol=1e-13)
    np.testing.assert_allclose(b[:, 128:], a[:, 128:], rtol=1e-13)


def test_mixer_reduces_to_pieces():
    """The mixer with identity-like projections: in_proj copies u into the z, xBC and dt_raw
    columns, out_proj reads the normed channels back. It must equal the pieces run by hand."""
    rng = np.random.default_rng(7)
    H, P, G, N, L = 2, 2, 1, 2, 9
    HP, GN = H * P, G * N
    Dp = 2 * HP + 2 * GN + H
    u = rng.standard_normal((1, L, Dp)) * 0.5
    in_w = np.eye(Dp)
    out_w = np.eye(HP)
    conv_w, conv_b = rng.standard_normal((HP + 2 * GN, 4)) * 0.5, rng.standard_normal(HP + 2 * GN) * 0.1
    dtb = np.full(H, -2.0)
    A, D, nw = -np.array([1.0, 3.0]), np.array([0.5, -0.25]), rng.standard_normal(HP)
    out, hf = oracle.mamba2_mixer(u, in_w, conv_w, conv_b, dtb, A, D, nw, out_w, nheads=H, headdim=P, ngroups=G,
                                  dstate=N, norm_groups=1, eps=1e-6)
    z, xbc, dtr = u[..., :HP], u[..., HP:2 * HP + 2 * GN], u[..., 2 * HP + 2 * GN:]
    x, Bm, Cm, dt = oracle.conv_split(xbc, dtr, conv_w, conv_b, dtb, nheads=H, headdim=P, ngroups=G, dstate=N)
    y, hf2 = oracle.recurrent(x, dt, A, Bm, Cm, D)
    want = oracle.gated_rmsnorm(y.reshape(1, L, HP), z, nw, ngroups=1, eps=1e-6)
    np.testing.assert_allclose(out, want, rtol=1e-13)
    np.testing.assert_allclose(hf, hf2, rtol=1e-13)


def test_mixer_one_token_closed_form():
    """One token from a zero state, with random projections, written out by hand: the causal
    convolution sees only its last tap, the state is dt x B^T, y = dt (B . C) x + D x, then the
    gate, the grouped norm and the output projection. Pins the column order of the input
    projection's row, the tap alignment, the step-size map and the order of the steps."""
    rng = np.random.default_rng(11)
    H, P, G, N, W, dm = 4, 2, 2, 3, 4, 5
    HP, GN = H * P, G * N
    Dp = 2 * HP + 2 * GN + H
    u = rng.standard_normal((1, 1, dm))
    in_w = rng.standard_normal((Dp, dm)) * 0.4
    out_w = rng.standard_normal((dm, HP)) * 0.4
    conv_w = rng.standard_normal((HP + 2 * GN, W)) * 0.5
    conv_b = rng.standard_normal(HP + 2 * GN) * 0.1
    dtb = rng.uniform(-2.0, 0.0, H)
    A, D = -rng.uniform(0.5, 3.0, H), rng.standard_normal(H)
    nw = 1.0 + 0.1 * rng.standard_normal(HP)
    eps = 1e-6
    out, hf = oracle.mamba2_mixer(u, in_w, conv_w, conv_b, dtb, A, D, nw, out_w, nheads=H, headdim=P, ngroups=G,
                                  dstate=N, norm_groups=2, eps=eps)

    row = [sum(in_w[c, k] * u[0, 0, k] for k in range(dm)) for c in range(Dp)]
    z = row[:HP]
    act = [0.0] * (HP + 2 * GN)
    for c in range(HP + 2 * GN):
        v = conv_w[c, W - 1] * row[HP + c] + conv_b[c]  # only the newest tap sees a token
        act[c] = v / (1.0 + math.exp(-v))
    xs, Bs, Cs = act[:HP], act[HP:HP + GN], act[HP + GN:]
    y = [0.0] * HP
    state = np.zeros((H, P, N))
    for h in range(H):
        dt = math.log1p(math.exp(row[2 * HP + 2 * GN + h] + dtb[h]))
        g = h // (H // G)
        bc = sum(Bs[g * N + n] * Cs[g * N + n] for n in range(N))
        for p in range(P):
            xv = xs[h * P + p]
            y[h * P + p] = dt * bc * xv + D[h] * xv
            for n in range(N):
                state[h, p, n] = dt * xv * Bs[g * N + n]
    gated = [y[c] * z[c] / (1.0 + math.exp(-z[c])) for c in range(HP)]
    normed = [0.0] * HP
    gs = HP // 2
    for k in range(2):
        ms = sum(gated[c] ** 2 for c in range(k * gs, (k + 1) * gs)) / gs
        for c in range(k * gs, (k + 1) * gs):
            normed[c] = nw[c] * gated[c] / math.sqrt(ms + eps)
    want = [sum(out_w[j, c] * normed[c] for c in range(HP)) for j in range(dm)]
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(hf[0], state, rtol=1e-12, atol=1e-15)
