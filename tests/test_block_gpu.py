"""GPU parity of the Mamba-2 block operations against the fp64 oracle: ssd_conv_split and
ssd_gated_rmsnorm through the C ABI, and the whole mixer forward (cuBLAS projections around
libssd kernels). max|out - ref| / max|ref| <= 1e-4 for fp32 and <= 2e-2 for bf16."""
import numpy as np
import pytest
import torch

import oracle
from ssd_cases import TOL, rel_err, to_np
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs, mamba2

pytestmark = pytest.mark.gpu


def tdt(dtype):
    return torch.float32 if dtype == "f32" else torch.bfloat16


def as_stored(a, dtype):
    """fp64 values of a after rounding to the storage dtype (what both sides consume)."""
    return inputs.Tensor(a, dtype).value


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("W,bias,L", [(4, True, 200), (1, False, 64), (3, True, 1), (2, True, 130)])
def test_conv_split(cuda_device, dtype, W, bias, L):
    rng = np.random.default_rng(W * 100 + L)
    Bsz, H, P, G, N = 2, 4, 16, 2, 8
    HP, GN = H * P, G * N
    Dp = 2 * HP + 2 * GN + H + 4   # a wider row (even length), as a projection output with padding
    row = as_stored(rng.standard_normal((Bsz, L, Dp)), dtype)
    w = as_stored(rng.standard_normal((HP + 2 * GN, W)) / np.sqrt(W), "f32")
    b = as_stored(rng.standard_normal(HP + 2 * GN) * 0.1, "f32") if bias else None
    dtb = as_stored(rng.uniform(-3, 0, H), "f32")
    xbc_np, dt_np = row[..., HP:2 * HP + 2 * GN], row[..., 2 * HP + 2 * GN:2 * HP + 2 * GN + H]
    ref = oracle.conv_split(xbc_np, dt_np, w, b, dtb, nheads=H, headdim=P, ngroups=G, dstate=N)
    rt = torch.from_numpy(row).to(cuda_device, tdt(dtype))
    o = ssd.ssd_conv_split(rt[..., HP:2 * HP + 2 * GN], rt[..., 2 * HP + 2 * GN:2 * HP + 2 * GN + H],
                           torch.from_numpy(w).float().to(cuda_device),
                           torch.from_numpy(b).float().to(cuda_device) if bias else None,
                           torch.from_numpy(dtb).float().to(cuda_device), nheads=H, headdim=P, ngroups=G, dstate=N)
    torch.cuda.synchronize()
    for k, r in zip(("x", "B", "C", "dt"), ref):
        assert rel_err(to_np(o[k]), r) <= TOL[dtype], k


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dim,ngroups", [(256, 1), (512, 8), (5120, 1), (5120, 8), (8192, 64)])
@pytest.mark.parametrize("zoff,zpad", [(8, 16), (2, 10)])  # 16-byte aligned z rows, and not
def test_gated_rmsnorm(cuda_device, dtype, dim, ngroups, zoff, zpad):
    rng = np.random.default_rng(dim + ngroups)
    rows = 37
    y = as_stored(rng.standard_normal((rows, dim)), dtype)
    zrow = as_stored(rng.standard_normal((rows, dim + zpad)), dtype)  # z: a column slice of wider rows
    w = as_stored(1 + 0.1 * rng.standard_normal(dim), "f32")
    ref = oracle.gated_rmsnorm(y, zrow[:, zoff:zoff + dim], w, ngroups=ngroups, eps=1e-5)
    zt = torch.from_numpy(zrow).to(cuda_device, tdt(dtype))
    out = ssd.ssd_gated_rmsnorm(torch.from_numpy(y).to(cuda_device, tdt(dtype)), zt[:, zoff:zoff + dim],
                                torch.from_numpy(w).float().to(cuda_device), ngroups=ngroups, eps=1e-5)
    torch.cuda.synchronize()
    assert rel_err(to_np(out), ref) <= TOL[dtype]


@pytest.mark.parametrize("L,h0", [(300, False), (257, True)])
def test_mixer_forward(cuda_device, L, h0):
    """The whole mixer (bf16, P = 64, N = 128: the tensor-core SSD path) against the oracle's
    composition in fp64 on the same rounded input and weights."""
    cfg = mamba2.MixerConfig(d_model=256, nheads=4, headdim=64, ngroups=1, dstate=128, norm_groups=2)
    d = inputs.draw_mixer(batch=2, seqlen=L, d_model=cfg.d_model, nheads=cfg.nheads, headdim=cfg.headdim,
                          ngroups=cfg.ngroups, dstate=cfg.dstate, seed=L)
    g = {k: v.torch(cuda_device) for k, v in d.items()}
    w = mamba2.MixerWeights(in_proj=g["in_proj"], conv_w=g["conv_w"], conv_b=g["conv_b"], dt_bias=g["dt_bias"],
                            A=g["A"], D=g["D"], norm_w=g["norm_w"], out_proj=g["out_proj"])
    h0v = np.random.default_rng(1).standard_normal((2, cfg.nheads, cfg.headdim, cfg.dstate)) * 0.1 if h0 else None
    h0t = torch.from_numpy(h0v).float().to(cuda_device) if h0 else None
    out, hf = mamba2.mixer_fwd(g["u"], w, cfg, h0=h0t)
    torch.cuda.synchronize()
    ref, href = oracle.mamba2_mixer(d["u"].value, d["in_proj"].value, d["conv_w"].value, d["conv_b"].value,
                                    d["dt_bias"].value, d["A"].value, d["D"].value, d["norm_w"].value,
                                    d["out_proj"].value, nheads=cfg.nheads, headdim=cfg.headdim, ngroups=cfg.ngroups,
                                    dstate=cfg.dstate, norm_groups=cfg.norm_groups, eps=cfg.eps,
                                    h0=as_stored(h0v, "f32") if h0 else None)
    assert rel_err(to_np(out), ref) <= 2e-2
    assert rel_err(to_np(hf), href) <= 2e-2
