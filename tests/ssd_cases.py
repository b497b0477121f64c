"""Shared helpers for the GPU parity tests: run the CUDA path through the binding
on seeded inputs, and compute the oracle on the same rounded values (whole
problem for small sizes, sampled (b, h) streams for the full-size workloads)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU output"
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().double().numpy()


def gpu_inputs(d, device):
    g = {k: d[k].torch(device) for k in ("x", "dt", "A", "B", "C", "D")}
    g["h0"] = d["h0"].torch(device) if d["h0"] is not None else None
    return g


def plan_of(d, chunk):
    Bsz, L, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    code = ssd.SSD_BF16 if d["x"].dtype == "bf16" else ssd.SSD_F32
    return ssd.fwd_plan(Bsz, L, H, P, G, N, code, chunk)


def run_fwd(d, chunk, device, *, use_D=True, use_h0=True, nan_fill=True):
    """Run ssd_fwd; also checks the device status word that the tensor-core path
    leaves at the start of its workspace (0 = no bounded wait ran out)."""
    g = gpu_inputs(d, device)
    y = torch.empty_like(g["x"])
    hf = torch.empty(g["x"].shape[0], g["x"].shape[2], g["x"].shape[3], g["B"].shape[3], device=device)
    if nan_fill:
        y.fill_(float("nan"))
        hf.fill_(float("nan"))
    plan = plan_of(d, chunk)
    ws = torch.full((max(plan["workspace_bytes"], 16),), 0xAB, dtype=torch.uint8, device=device)
    ssd.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"] if use_D else None,
                g["h0"] if use_h0 else None, chunk=chunk, y=y, h_final=hf, workspace=ws)
    torch.cuda.synchronize()
    if plan["path"] == "tcgen05":
        assert int(ws[:4].view(torch.int32).item()) == 0, "device status word set"
    return y, hf


def oracle_full(d, *, use_D=True, use_h0=True):
    h0 = d["h0"].value if (use_h0 and d["h0"] is not None) else None
    return oracle.recurrent(d["x"].value, d["dt"].value, d["A"].value, d["B"].value, d["C"].value,
                            d["D"].value if use_D else None, h0)


def oracle_stream(d, b, h):
    """Oracle y[b, :, h, :] and h_final[b, h] of one stream, from the sliced inputs."""
    H = d["x"].shape[2]
    G = d["B"].shape[2]
    g = h // (H // G)
    x = d["x"].values((slice(b, b + 1), slice(None), slice(h, h + 1)))
    dt = d["dt"].values((slice(b, b + 1), slice(None), slice(h, h + 1)))
    Bm = d["B"].values((slice(b, b + 1), slice(None), slice(g, g + 1)))
    Cm = d["C"].values((slice(b, b + 1), slice(None), slice(g, g + 1)))
    A = d["A"].value[h:h + 1]
    D = d["D"].value[h:h + 1]
    h0 = d["h0"].values((slice(b, b + 1), slice(h, h + 1))) if d["h0"] is not None else None
    y, hf = oracle.recurrent(x, dt, A, Bm, Cm, D, h0)
    return y[0, :, 0, :], hf[0, 0]


def sample_streams(Bsz, H, n, seed=123):
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (Bsz - 1, H - 1)}
    while len(picks) < min(n, Bsz * H):
        picks.add((int(rng.integers(Bsz)), int(rng.integers(H))))
    return sorted(picks)


def draw(name, **kw):
    return inputs.draw(inputs.WORKLOADS[name], **kw)


GRADS = ("dx", "ddt", "dA", "dB", "dC", "dD", "dh0")


def run_bwd(d, cot, chunk, device, *, use_D=True, use_h0=True, use_dhf=True):
    """ssd_bwd through the binding, outputs pre-filled with NaN; returns numpy fp64 arrays."""
    g = gpu_inputs(d, device)
    dy = cot["dy"].torch(device)
    dhf = cot["dh_final"].torch(device) if (use_dhf and cot["dh_final"] is not None) else None
    out = {"dx": torch.full_like(g["x"], float("nan")), "ddt": torch.full_like(g["dt"], float("nan")),
           "dB": torch.full_like(g["B"], float("nan")), "dC": torch.full_like(g["C"], float("nan")),
           "dA": torch.full_like(g["A"], float("nan")), "dD": torch.full_like(g["D"], float("nan")),
           "dh0": torch.full((g["x"].shape[0], g["x"].shape[2], g["x"].shape[3], g["B"].shape[3]), float("nan"),
                             device=device)}
    ssd.ssd_bwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"] if use_D else None,
                g["h0"] if use_h0 else None, dy, dhf, chunk=chunk, out=out)
    torch.cuda.synchronize()
    return {k: to_np(v) for k, v in out.items()}


def oracle_bwd(d, cot, *, use_D=True, use_h0=True, use_dhf=True, batch_rows=None):
    """The oracle's gradients; batch_rows=(lo, hi) restricts it to those rows (dA and dD then
    cover only them)."""
    sl = slice(None) if batch_rows is None else slice(*batch_rows)
    v = lambda t: t.values((sl,)) if t is not None else None
    h0 = v(d["h0"]) if use_h0 else None
    dhf = v(cot["dh_final"]) if use_dhf else None
    return oracle.backward(v(d["x"]), v(d["dt"]), d["A"].value, v(d["B"]), v(d["C"]),
                           d["D"].value if use_D else None, h0, v(cot["dy"]), dhf)
