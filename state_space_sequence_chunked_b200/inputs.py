"""Seeded synthetic inputs for the SSD forward and verify workloads.

This module draws random tensors and rounds them to the storage dtype. It holds
none of the method's arithmetic, so both the CUDA path (through the package
binding) and the fp64 oracle can consume what it returns.

Distributions (the SSD problem statement: input-dependent B, C and step size,
a scalar decay rate per head, a per-head skip weight D):
    x   ~ N(0, 1)                       [B, L, H, P]
    dt  = exp(U(ln 1e-3, ln 1e-1))      [B, L, H]     ("loguniform", the default), or
    dt  = softplus(N(0, 1) + b_h),      [B, L, H]     ("softplus": a projection output plus a
          b_h ~ U(-7, -2.3) per head                   per-head bias, as a Mamba-2 layer forms it)
    A_h = -exp(U(ln 1, ln 16))          [H]           (always fp32)
    B,C ~ N(0, 1) / sqrt(N)             [B, L, G, N]
    D   ~ N(0, 1)                       [H]           (always fp32)
    h0  ~ N(0, h0_std) or zeros         [B, H, P, N]  (always fp32)
    accepted ~ U{0..K}                  [B] int32     (verify workloads only)
Draws are fp64 from numpy's PCG64 generator seeded with `seed`, taken in the
fixed order x, dt, A, B, C, D, h0, accepted. Values stored as bf16 are rounded
fp64 -> fp32 -> bf16, each step round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int  # K for verify workloads
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str  # "f32" or "bf16": storage dtype of x, dt, B, C and y
    h0_std: float
    seed: int
    verify: bool = False
    dt_dist: str = "loguniform"  # or "softplus" (see the module docstring)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


# The workloads: a tiny fp32 case, a 130M-like layer, the 2.7B-like layer (the headline
# shape), a long-context large-state case, a spec-decode verify, and the headline shape
# with softplus-distributed step sizes.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 4, 16, 16, 1, 64, "f32", 0.0, 0),
    "mamba2_130m": Workload("mamba2_130m", 8, 2048, 24, 64, 128, 1, 256, "bf16", 0.0, 1),
    "mamba2_2p7b": Workload("mamba2_2p7b", 4, 8192, 80, 64, 128, 1, 256, "bf16", 0.0, 2),
    "long_n256": Workload("long_n256", 1, 65536, 80, 64, 256, 1, 256, "bf16", 0.1, 3),
    "verify_k8": Workload("verify_k8", 64, 8, 32, 128, 128, 8, 8, "bf16", 0.1, 4, verify=True),
    # the headline shape with step sizes spread as a trained layer's are (long tail to dt ~ 1+)
    "mamba2_2p7b_softplus_dt": Workload("mamba2_2p7b_softplus_dt", 4, 8192, 80, 64, 128, 1, 256, "bf16", 0.0, 5,
                                        dt_dist="softplus"),
}


def round_f32(a: np.ndarray) -> np.ndarray:
    """fp64 -> fp32, round to nearest even."""
    return np.asarray(a, dtype=np.float64).astype(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 -> bf16 (round to nearest even), returned as uint16 bit patterns."""
    u = round_f32(a).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


class Tensor:
    """A drawn tensor: its storage bits and, on demand, the exact fp64 value of each element."""

    def __init__(self, f64: np.ndarray, dtype: str):
        if dtype == "bf16":
            self.bits = bf16_bits(f64)
        elif dtype == "f32":
            self.bits = round_f32(f64)
        else:
            raise ValueError(dtype)
        self.dtype = dtype
        self.shape = self.bits.shape
        self._value = None

    def values(self, index=...) -> np.ndarray:
        """fp64 copy of the stored values (optionally of `bits[index]` only)."""
        b = self.bits[index]
        if self.dtype == "bf16":
            return bf16_to_f64(b)
        return b.astype(np.float64)

    @property
    def value(self) -> np.ndarray:
        if self._value is None:
            self._value = self.values()
        return self._value

    def torch(self, device="cpu"):
        import torch

        if self.dtype == "bf16":
            t = torch.from_numpy(self.bits.view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(self.bits)
        return t.to(device)


def draw(wl: Workload, *, batch=None, seqlen=None, seed=None, h0_std=None, zero_A=False):
    """Draw the inputs of workload `wl` (optionally overriding batch/seqlen/seed).

    Returns a dict of Tensor objects: x, dt, B, C (storage dtype wl.dtype),
    A, D, h0 (fp32) and, for verify workloads, `accepted` (np.int32 array).
    `h0` is None when its std is 0 (the zero initial state).
    """
    Bsz = wl.batch if batch is None else batch
    L = wl.seqlen if seqlen is None else seqlen
    H, P, N, G = wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    std = wl.h0_std if h0_std is None else h0_std
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    x = rng.standard_normal((Bsz, L, H, P))
    if wl.dt_dist == "softplus":
        v = rng.standard_normal((Bsz, L, H)) + rng.uniform(-7.0, -2.3, size=(H,))
        dt = np.logaddexp(0.0, v)  # softplus, overflow-free
    else:
        dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=(Bsz, L, H)))
    A = -np.exp(rng.uniform(0.0, math.log(16.0), size=(H,)))
    Bm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    Cm = rng.standard_normal((Bsz, L, G, N)) / math.sqrt(N)
    D = rng.standard_normal((H,))
    h0 = rng.standard_normal((Bsz, H, P, N)) * std if std > 0 else None
    out = {
        "x": Tensor(x, wl.dtype),
        "dt": Tensor(dt, wl.dtype),
        "A": Tensor(np.zeros_like(A) if zero_A else A, "f32"),
        "B": Tensor(Bm, wl.dtype),
        "C": Tensor(Cm, wl.dtype),
        "D": Tensor(D, "f32"),
        "h0": Tensor(h0, "f32") if h0 is not None else None,
    }
    del x, Bm, Cm
    if wl.verify:
        out["accepted"] = rng.integers(0, L + 1, size=(Bsz,), dtype=np.int64).astype(np.int32)
    return out


def draw_cotangents(wl: Workload, *, batch=None, seqlen=None, seed=None, dh_std=1.0):
    """Cotangents for the backward pass of workload `wl`: dy ~ N(0, 1) [B,L,H,P] in the
    storage dtype and dh_final ~ N(0, dh_std) [B,H,P,N] fp32 (None when dh_std is 0).
    Drawn from their own stream (seed + 10007), so the forward inputs are unchanged."""
    Bsz = wl.batch if batch is None else batch
    L = wl.seqlen if seqlen is None else seqlen
    H, P, N = wl.nheads, wl.headdim, wl.dstate
    rng = np.random.default_rng((wl.seed if seed is None else seed) + 10007)
    dy = rng.standard_normal((Bsz, L, H, P))
    dhf = rng.standard_normal((Bsz, H, P, N)) * dh_std if dh_std > 0 else None
    return {"dy": Tensor(dy, wl.dtype), "dh_final": Tensor(dhf, "f32") if dhf is not None else None}


def draw_mixer(*, batch, seqlen, d_model, nheads, headdim, ngroups, dstate, conv_width=4, dtype="bf16", seed=0):
    """Input and random-init weights of one Mamba-2 mixer (no trained weights exist here).
    u ~ N(0, 1) [B, L, d_model]; in_proj ~ N(0, 1/d_model) [2HP + 2GN + H, d_model] and
    out_proj ~ N(0, 1/HP) [d_model, HP] in the storage dtype; fp32 conv taps ~ N(0, 1/W), conv
    bias ~ N(0, 0.01), dt bias ~ U(-7, -2.3) (softplus of it lies near [1e-3, 1e-1]),
    A = -exp(U(0, ln 16)), D ~ N(0, 1), norm weight ~ 1 + N(0, 0.01)."""
    HP, GN = nheads * headdim, ngroups * dstate
    Dp, Cc = 2 * HP + 2 * GN + nheads, HP + 2 * GN
    rng = np.random.default_rng(seed)
    out = {
        "u": Tensor(rng.standard_normal((batch, seqlen, d_model)), dtype),
        "in_proj": Tensor(rng.standard_normal((Dp, d_model)) / math.sqrt(d_model), dtype),
        "conv_w": Tensor(rng.standard_normal((Cc, conv_width)) / math.sqrt(conv_width), "f32"),
        "conv_b": Tensor(rng.standard_normal(Cc) * 0.1, "f32"),
        "dt_bias": Tensor(rng.uniform(-7.0, -2.3, size=nheads), "f32"),
        "A": Tensor(-np.exp(rng.uniform(0.0, math.log(16.0), size=nheads)), "f32"),
        "D": Tensor(rng.standard_normal(nheads), "f32"),
        "norm_w": Tensor(1.0 + 0.1 * rng.standard_normal(HP), "f32"),
        "out_proj": Tensor(rng.standard_normal((d_model, HP)) / math.sqrt(HP), dtype),
    }
    return out
