"""fp64 CPU oracle for the Mamba-2 SSD layer forward pass and speculative verify.

TEST INFRASTRUCTURE. Only tests/, the smoke check and the benchmark's CPU-baseline
leg import this package. It shares no code with the CUDA library and never calls it.

Forms (each in fp64 on the already-rounded inputs, layouts as in the library):
  recurrent          the plain definition, token by token (C, OpenMP over (b, h)):
                     "A Visual Guide to Mamba and SSMs", "The Recurrent
                     Representation" and "What is a SSM" (D skip); Mamba-2 SSD
                     write-up, "SSD 层" (scalar A per head).
  quadratic          y = M (dt * x) + D x with M[t, s] = (C_t . B_s) exp(sum_{k=s+1..t} a_k),
                     plus the initial-state term: Mamba-2 SSD write-up,
                     contributions list and "SSD 层的对偶注意力" (SSM = semiseparable
                     matrix = structured masked attention; "token-mixing matrix M").
  linear_attention   the A = 0 case, causal linear attention with (x, B, C) as
                     (V, K, Q): "distilling Llama into Mamba" write-up,
                     "从 Llama 到 Mamba".
  chunked            the 4-step chunked algorithm (within-chunk decay cumsum,
                     diagonal blocks, chunk states, inter-chunk state passing,
                     state-to-output): Mamba-2 SSD write-up, "SSD 算法：分块矩阵分解"
                     and "SSD 算法：分块和状态传递". Step 3 is a sequential loop
                     over chunks (the scan runs over a short sequence).
  verify             K tokens of the recurrence from a saved state, returning the
                     state after every token; select_state keeps the state at the
                     accepted position: "distilling Llama into Mamba" write-up,
                     "推测解码".
  conv_split         the Mamba-2 block's convolution step: causal depthwise
                     convolution of the x, B, C channels of the input projection,
                     SiLU, split; dt = softplus(dt_raw + bias): "A Visual Guide to
                     Mamba and SSMs", "The Mamba Block" (convolution before the SSM).
  gated_rmsnorm      y * silu(z), normalised by its root mean square over groups of
                     channels, times a weight: SSD write-up, "张量并行" (grouped norm).
  mamba2_mixer       input projection, conv_split, the SSD recurrence, gated norm,
                     output projection, in that order (Mamba-2 "parallel projection"
                     block, SSD write-up "张量并行" and the Bi-Mamba summary's list of
                     Mamba-2 layers).
  backward           the gradient of sum(dy * y) + sum(dh_final * h_final) with
                     respect to every input: the recurrence differentiated token
                     by token in reverse (C, OpenMP over (b, h)); the states are
                     recomputed per segment in the reverse sweep instead of being
                     stored, as "A Visual Guide to Mamba and SSMs",
                     "Recomputation", describes for the backward pass.
Layouts: x [B,L,H,P], dt [B,L,H], A [H], Bm/Cm [B,L,G,N], D [H], h0 [B,H,P,N];
head h uses group g = h // (H // G).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, dp = ctypes.c_int64, ctypes.POINTER(ctypes.c_double)
        lib.oracle_ssd_recurrent.argtypes = [i64] * 6 + [dp] * 10 + [ctypes.c_int]
        lib.oracle_ssd_recurrent.restype = ctypes.c_int
        lib.oracle_ssd_backward.argtypes = [i64] * 6 + [dp] * 9 + [dp] * 7 + [i64, ctypes.c_int]
        lib.oracle_ssd_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def recurrent(x, dt, A, Bm, Cm, D=None, h0=None, *, store_states=False, threads=0):
    """Token-by-token recurrence. Returns (y, h_final) or (y, h_final, states)."""
    x, dt, A, Bm, Cm, D, h0 = map(_f64, (x, dt, A, Bm, Cm, D, h0))
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    assert dt.shape == (Bsz, L, H) and A.shape == (H,) and Bm.shape == Cm.shape == (Bsz, L, G, N)
    assert H % G == 0
    y = np.empty_like(x)
    hf = np.empty((Bsz, H, P, N))
    st = np.empty((Bsz, L, H, P, N)) if store_states else None
    rc = _load().oracle_ssd_recurrent(Bsz, L, H, P, G, N, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm),
                                      _ptr(Cm), _ptr(D), _ptr(h0), _ptr(y), _ptr(hf), _ptr(st),
                                      int(threads))
    if rc != 0:
        raise RuntimeError("oracle_ssd_recurrent failed")
    return (y, hf, st) if store_states else (y, hf)


def backward(x, dt, A, Bm, Cm, D, h0, dy, dh_final=None, *, seg=64, threads=0):
    """Gradient of sum(dy * y) + sum(dh_final * h_final) through the recurrence.

    D and h0 may be None (no skip / zero initial state), dh_final None (= 0).
    Returns a dict: dx [B,L,H,P], ddt [B,L,H], dA [H], dB [B,L,G,N], dC [B,L,G,N],
    dD [H], dh0 [B,H,P,N] (the gradient for the initial state, also when h0 is None)."""
    x, dt, A, Bm, Cm, D, h0, dy, dh_final = map(_f64, (x, dt, A, Bm, Cm, D, h0, dy, dh_final))
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    assert dt.shape == (Bsz, L, H) and A.shape == (H,) and Bm.shape == Cm.shape == (Bsz, L, G, N)
    assert dy.shape == x.shape and H % G == 0
    out = {"dx": np.empty_like(x), "ddt": np.empty_like(dt), "dA": np.empty(H),
           "dB": np.empty_like(Bm), "dC": np.empty_like(Cm), "dD": np.empty(H),
           "dh0": np.empty((Bsz, H, P, N))}
    rc = _load().oracle_ssd_backward(
        Bsz, L, H, P, G, N, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(h0),
        _ptr(dy), _ptr(dh_final), _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dA"]),
        _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dh0"]), int(seg), int(threads))
    if rc != 0:
        raise RuntimeError("oracle_ssd_backward failed")
    return out


def _heads_to_groups(Bm, H):
    G = Bm.shape[2]
    return np.repeat(Bm, H // G, axis=2)  # [B, L, H, N], head h -> group h // (H // G)


def quadratic(x, dt, A, Bm, Cm, D=None, h0=None):
    """The SSM as one masked matrix per (b, h) (brute force, O(L^2); small L only)."""
    x, dt, A, Bm, Cm, D, h0 = map(_f64, (x, dt, A, Bm, Cm, D, h0))
    Bsz, L, H, P = x.shape
    N = Bm.shape[3]
    Bh, Ch = _heads_to_groups(Bm, H), _heads_to_groups(Cm, H)
    y = np.zeros_like(x)
    hf = np.zeros((Bsz, H, P, N))
    for b in range(Bsz):
        for h in range(H):
            a = dt[b, :, h] * A[h]
            # decay from token s to token t: exp(a_{s+1} + ... + a_t), each sum taken directly
            dec = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    dec[t, s] = np.exp(np.sum(a[s + 1:t + 1]))
            M = (Ch[b, :, h, :] @ Bh[b, :, h, :].T) * dec  # [t, s], zero above the diagonal
            u = dt[b, :, h, None] * x[b, :, h, :]  # [L, P]
            yb = M @ u
            # final state: sum_s exp(a_{s+1..L-1}) u_s B_s^T
            w = np.array([np.exp(np.sum(a[s + 1:])) for s in range(L)])
            hfb = (w[:, None] * u).T @ Bh[b, :, h, :]
            if h0 is not None:
                lead = np.array([np.exp(np.sum(a[:t + 1])) for t in range(L)])  # exp(a_0..a_t)
                yb = yb + lead[:, None] * (Ch[b, :, h, :] @ h0[b, h].T)
                hfb = hfb + np.exp(np.sum(a)) * h0[b, h]
            if D is not None:
                yb = yb + D[h] * x[b, :, h, :]
            y[b, :, h, :] = yb
            hf[b, h] = hfb
    return y, hf


def linear_attention(x, dt, Bm, Cm, D=None):
    """A = 0: y_t = sum_{s<=t} (C_t . B_s) dt_s x_s + D x_t (causal linear attention)."""
    x, dt, Bm, Cm, D = map(_f64, (x, dt, Bm, Cm, D))
    Bsz, L, H, P = x.shape
    Bh, Ch = _heads_to_groups(Bm, H), _heads_to_groups(Cm, H)
    y = np.zeros_like(x)
    for b in range(Bsz):
        for h in range(H):
            Q_, K_, V_ = Ch[b, :, h, :], Bh[b, :, h, :], dt[b, :, h, None] * x[b, :, h, :]
            scores = np.tril(Q_ @ K_.T)
            y[b, :, h, :] = scores @ V_ + (D[h] * x[b, :, h, :] if D is not None else 0.0)
    return y


def chunked(x, dt, A, Bm, Cm, D=None, h0=None, *, chunk):
    """The 4-step chunked algorithm in fp64, returning its intermediates.

    Returns dict with
      A_cs    [B, H, nc, Q]   within-chunk inclusive cumsum of a = dt * A (padded with 0)
      states  [B, H, nc, P, N] chunk states from a zero start (step 2)
      S_in    [B, H, nc, P, N] state entering each chunk (step 3)
      y, h_final
    The last chunk may be shorter than `chunk`.
    """
    x, dt, A, Bm, Cm, D, h0 = map(_f64, (x, dt, A, Bm, Cm, D, h0))
    Bsz, L, H, P = x.shape
    N = Bm.shape[3]
    Q = int(chunk)
    nc = (L + Q - 1) // Q
    Bh, Ch = _heads_to_groups(Bm, H), _heads_to_groups(Cm, H)
    a = dt * A[None, None, :]  # [B, L, H]
    A_cs = np.zeros((Bsz, H, nc, Q))
    states = np.zeros((Bsz, H, nc, P, N))
    S_in = np.zeros((Bsz, H, nc, P, N))
    y = np.zeros_like(x)
    chunk_total = np.zeros((Bsz, H, nc))
    for c in range(nc):
        lo, hi = c * Q, min(L, (c + 1) * Q)
        q = hi - lo
        acs = np.cumsum(a[:, lo:hi, :], axis=1)  # step 0, [B, q, H]
        A_cs[:, :, c, :q] = acs.transpose(0, 2, 1)
        chunk_total[:, :, c] = acs[:, -1, :]
        # step 1: diagonal block, (C B^T o L) (dt x) with L[l, s] = exp(acs_l - acs_s) for s <= l
        seg = acs[:, :, None, :] - acs[:, None, :, :]  # [B, l, s, H]
        causal = np.tril(np.ones((q, q), dtype=bool))[None, :, :, None]
        Lmask = np.where(causal, np.exp(np.where(causal, seg, 0.0)), 0.0)
        CB = np.einsum("blhn,bshn->blsh", Ch[:, lo:hi], Bh[:, lo:hi])
        u = dt[:, lo:hi, :, None] * x[:, lo:hi]  # [B, q, H, P]
        y[:, lo:hi] = np.einsum("blsh,bshp->blhp", CB * Lmask, u)
        # step 2: chunk state from a zero start, decayed to the end of the chunk
        w = np.exp(acs[:, -1:, :] - acs)  # [B, q, H]
        states[:, :, c] = np.einsum("bsh,bshp,bshn->bhpn", w, u, Bh[:, lo:hi])
    # step 3: state passing across chunks
    S = np.zeros((Bsz, H, P, N)) if h0 is None else h0.copy()
    for c in range(nc):
        S_in[:, :, c] = S
        S = np.exp(chunk_total[:, :, c])[:, :, None, None] * S + states[:, :, c]
    h_final = S
    # step 4: state -> output, plus the D skip
    for c in range(nc):
        lo, hi = c * Q, min(L, (c + 1) * Q)
        q = hi - lo
        lead = np.exp(A_cs[:, :, c, :q]).transpose(0, 2, 1)  # [B, q, H]
        y[:, lo:hi] += lead[..., None] * np.einsum("blhn,bhpn->blhp", Ch[:, lo:hi], S_in[:, :, c])
    if D is not None:
        y += D[None, None, :, None] * x
    return {"A_cs": A_cs, "states": states, "S_in": S_in, "y": y, "h_final": h_final,
            "chunk_total": chunk_total}


def verify(h0, x, dt, A, Bm, Cm, D=None):
    """K draft tokens from h0. Returns (y [B,K,H,P], states_out [B,K,H,P,N]),
    states_out[:, k] being the state after token k."""
    y, _, st = recurrent(x, dt, A, Bm, Cm, D, h0, store_states=True)
    return y, st


def select_state(h0, states_out, accepted):
    """Kept state per batch row: h0 when 0 tokens were accepted, else the state
    after the last accepted token (states_out[b, a - 1]). Copies bits, no arithmetic."""
    Bsz, K = states_out.shape[:2]
    out = np.empty_like(h0)
    for b in range(Bsz):
        a = int(accepted[b])
        if not 0 <= a <= K:
            raise ValueError("accepted index out of range")
        out[b] = h0[b] if a == 0 else states_out[b, a - 1]
    return out


# ---- the Mamba-2 block around the SSD layer ---------------------------------------------

def silu(v):
    return v / (1.0 + np.exp(-v))


def softplus(v):
    return np.log1p(np.exp(-np.abs(v))) + np.maximum(v, 0.0)


def conv_split(xbc, dt_raw, conv_w, conv_b, dt_bias, *, nheads, headdim, ngroups, dstate):
    """Causal depthwise convolution over tokens of each of the Cc = H*P + 2*G*N channels of xbc
    [B, L, Cc] with taps conv_w [Cc, W] (tap W-1 on the current token, inputs before the first
    token are zero), plus conv_b [Cc] (or None), then SiLU; split into x [B,L,H,P], B, C
    [B,L,G,N]. dt = softplus(dt_raw + dt_bias) [B,L,H]. Written as the sum over taps."""
    xbc, dt_raw, conv_w, conv_b, dt_bias = map(_f64, (xbc, dt_raw, conv_w, conv_b, dt_bias))
    Bsz, L, Cc = xbc.shape
    W = conv_w.shape[1]
    H, P, G, N = nheads, headdim, ngroups, dstate
    assert Cc == H * P + 2 * G * N and dt_raw.shape == (Bsz, L, H)
    acc = np.zeros_like(xbc) if conv_b is None else np.broadcast_to(conv_b, xbc.shape).copy()
    for j in range(W):
        shift = W - 1 - j  # tap j reads token t - shift
        if shift == 0:
            acc += conv_w[:, j] * xbc
        elif shift < L:
            acc[:, shift:, :] += conv_w[:, j] * xbc[:, :L - shift, :]
    act = silu(acc)
    x = act[..., :H * P].reshape(Bsz, L, H, P)
    Bm = act[..., H * P:H * P + G * N].reshape(Bsz, L, G, N)
    Cm = act[..., H * P + G * N:].reshape(Bsz, L, G, N)
    dt = softplus(dt_raw + (0.0 if dt_bias is None else dt_bias))
    return x, Bm, Cm, dt


def gated_rmsnorm(y, z, weight, *, ngroups, eps):
    """g = y * silu(z); per group of dim / ngroups consecutive channels,
    out = weight * g / sqrt(mean(g^2) + eps). y, z [..., dim]."""
    y, z, weight = map(_f64, (y, z, weight))
    dim = y.shape[-1]
    g = y * silu(z)
    gg = g.reshape(*g.shape[:-1], ngroups, dim // ngroups)
    r = 1.0 / np.sqrt(np.mean(gg * gg, axis=-1, keepdims=True) + eps)
    return (gg * r).reshape(g.shape) * weight


def mamba2_mixer(u, in_proj_w, conv_w, conv_b, dt_bias, A, D, norm_w, out_proj_w, *, nheads, headdim, ngroups,
                 dstate, norm_groups, eps, h0=None):
    """The Mamba-2 mixer forward. u [B, L, d_model]; in_proj_w [2*H*P + 2*G*N + H, d_model] gives
    each token's row [z | x B C | dt_raw]; out_proj_w [d_model, H*P]. Returns (out, h_final)."""
    u, in_proj_w, out_proj_w = map(_f64, (u, in_proj_w, out_proj_w))
    H, P, G, N = nheads, headdim, ngroups, dstate
    HP, GN = H * P, G * N
    zxbcdt = u @ in_proj_w.T
    z, xbc, dt_raw = zxbcdt[..., :HP], zxbcdt[..., HP:2 * HP + 2 * GN], zxbcdt[..., 2 * HP + 2 * GN:]
    x, Bm, Cm, dt = conv_split(xbc, dt_raw, conv_w, conv_b, dt_bias, nheads=H, headdim=P, ngroups=G, dstate=N)
    y, hf = recurrent(x, dt, A, Bm, Cm, D, h0)
    o = gated_rmsnorm(y.reshape(*y.shape[:2], HP), z, norm_w, ngroups=norm_groups, eps=eps)
    return o @ out_proj_w.T, hf

