"""The Mamba-2 mixer forward around the SSD layer.

Order of operations (the Mamba-2 "parallel projection" block: every SSM parameter is a
projection of the layer input, Mamba-2 SSD write-up, "张量并行"; the convolution before the
SSM, "A Visual Guide to Mamba and SSMs", "The Mamba Block"):

    zxbcdt = u in_proj^T                      plain GEMM (cuBLAS)        [B, L, 2HP + 2GN + H]
    x, B, C, dt = ssd_conv_split(...)         libssd kernel
    y, h_final = ssd_fwd(x, dt, A, B, C, D)   libssd kernel(s)
    o = ssd_gated_rmsnorm(y, z)               libssd kernel
    out = o out_proj^T                        plain GEMM (cuBLAS)        [B, L, d_model]

The two projections are dense matrix products with no fused work, so they go to the vendor
GEMM (through torch.matmul); everything between them runs in libssd.
"""
from __future__ import annotations

import dataclasses

import torch

from . import _binding as ssd


@dataclasses.dataclass
class MixerConfig:
    d_model: int
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    conv_width: int = 4
    norm_groups: int = 1
    chunk: int = 256
    eps: float = 1e-5

    @property
    def d_inner(self) -> int:
        return self.nheads * self.headdim

    @property
    def d_in_proj(self) -> int:
        return 2 * self.d_inner + 2 * self.ngroups * self.dstate + self.nheads


@dataclasses.dataclass
class MixerWeights:
    in_proj: torch.Tensor    # [d_in_proj, d_model], input dtype
    conv_w: torch.Tensor     # [H*P + 2*G*N, W] fp32
    conv_b: torch.Tensor     # [H*P + 2*G*N] fp32
    dt_bias: torch.Tensor    # [H] fp32
    A: torch.Tensor          # [H] fp32, negative
    D: torch.Tensor          # [H] fp32
    norm_w: torch.Tensor     # [H*P] fp32
    out_proj: torch.Tensor   # [d_model, H*P], input dtype


def mixer_fwd(u: torch.Tensor, w: MixerWeights, cfg: MixerConfig, h0=None, stream=None):
    """u [B, L, d_model] -> (out [B, L, d_model], h_final [B, H, P, N])."""
    HP, GN = cfg.d_inner, cfg.ngroups * cfg.dstate
    zxbcdt = torch.matmul(u, w.in_proj.t())
    z = zxbcdt[..., :HP]
    xbc = zxbcdt[..., HP:2 * HP + 2 * GN]
    dt_raw = zxbcdt[..., 2 * HP + 2 * GN:]
    s = ssd.ssd_conv_split(xbc, dt_raw, w.conv_w, w.conv_b, w.dt_bias, nheads=cfg.nheads, headdim=cfg.headdim,
                           ngroups=cfg.ngroups, dstate=cfg.dstate, stream=stream)
    y, hf = ssd.ssd_fwd(s["x"], s["dt"], w.A, s["B"], s["C"], w.D, h0, chunk=cfg.chunk, stream=stream)
    Bsz, L = u.shape[:2]
    o = ssd.ssd_gated_rmsnorm(y.view(Bsz, L, HP), z, w.norm_w, ngroups=cfg.norm_groups, eps=cfg.eps, stream=stream)
    return torch.matmul(o, w.out_proj.t()), hf
