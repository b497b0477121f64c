"""GPU parity of ssd_bwd against the fp64 oracle's backward (the recurrence differentiated
token by token): for every gradient, max|g - g_ref| / max|g_ref| <= 1e-4 for fp32 inputs and
<= 2e-2 for bf16 inputs."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from ssd_cases import GRADS, TOL, draw, oracle_bwd, rel_err, run_bwd
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def check(d, cot, chunk, dev, names=GRADS, **kw):
    got = run_bwd(d, cot, chunk, dev, **kw)
    ref = oracle_bwd(d, cot, **kw)
    tol = TOL[d["x"].dtype]
    errs = {k: rel_err(got[k], ref[k]) for k in names}
    assert all(e <= tol for e in errs.values()), errs
    return errs


def cot_of(wl_name, d, **kw):
    wl = inputs.WORKLOADS[wl_name]
    Bsz, L = d["x"].shape[:2]
    return inputs.draw_cotangents(wl, batch=Bsz, seqlen=L, **kw)


def test_tiny_fp32_workload(cuda_device):
    """B1 L256 H4 P16 N16, chunk 64, with h0 and dh_final."""
    d = draw("tiny_fp32", h0_std=0.5)
    errs = check(d, cot_of("tiny_fp32", d), 64, cuda_device)
    assert max(errs.values()) < 2e-5, errs


@pytest.mark.parametrize("chunk", [1, 7, 64, 100, 256])
def test_fp32_any_chunk_ragged(cuda_device, chunk):
    d = draw("tiny_fp32", seqlen=201, h0_std=0.5)
    check(d, cot_of("tiny_fp32", d, seed=chunk), chunk, cuda_device)


BF16_CASES = [
    # (batch, seqlen, nheads, headdim, ngroups, dstate, chunk, h0_std)
    (2, 600, 4, 64, 1, 128, 256, 0.0),     # several chunks, ragged tail, heads share a group
    (1, 700, 6, 64, 2, 128, 256, 0.1),     # groups, initial state
    (2, 300, 4, 64, 4, 256, 256, 0.1),     # N = 256, one group per head
    (1, 257, 2, 64, 1, 128, 128, 0.0),     # tail of one token
    (3, 100, 3, 32, 1, 64, 64, 0.2),
    (1, 50, 2, 128, 1, 128, 256, 0.1),     # shorter than a chunk
    (1, 1, 2, 64, 1, 128, 256, 0.1),       # a single token
    (1, 90, 2, 200, 1, 40, 32, 0.1),       # headdim and dstate not multiples of 32
    (1, 64, 2, 256, 1, 256, 64, 0.1),      # the largest tiles
    (1, 300, 2, 64, 1, 128, 100, 0.1),     # tensor-core path, chunk not a multiple of the 64-token tile
    (2, 130, 4, 64, 2, 64, 48, 0.0),       # tensor-core path, chunk below one tile, groups
]


@pytest.mark.parametrize("case", BF16_CASES)
def test_bf16_small(cuda_device, case):
    Bsz, L, H, P, G, N, Q, std = case
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_130m"], batch=Bsz, seqlen=L, nheads=H, headdim=P,
                             ngroups=G, dstate=N, chunk=Q, h0_std=std, seed=2000 + L)
    d = inputs.draw(wl)
    cot = inputs.draw_cotangents(wl)
    check(d, cot, Q, cuda_device)


@pytest.mark.parametrize("use_D,use_h0,use_dhf", [(False, False, False), (True, False, True), (False, True, False)])
def test_optional_inputs(cuda_device, use_D, use_h0, use_dhf):
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_130m"], batch=2, seqlen=400, nheads=4, h0_std=0.3, seed=78)
    d = inputs.draw(wl)
    check(d, inputs.draw_cotangents(wl), 256, cuda_device, use_D=use_D, use_h0=use_h0, use_dhf=use_dhf)


def test_optional_outputs_may_be_null(cuda_device):
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_130m"], batch=1, seqlen=300, nheads=2, h0_std=0.3, seed=79)
    d = inputs.draw(wl)
    cot = inputs.draw_cotangents(wl)
    g = {k: d[k].torch(cuda_device) for k in ("x", "dt", "A", "B", "C", "D")}
    o = ssd.ssd_bwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], d["h0"].torch(cuda_device),
                    cot["dy"].torch(cuda_device), cot["dh_final"].torch(cuda_device), chunk=256,
                    want_dD=False, want_dh0=False)
    torch.cuda.synchronize()
    assert o["dD"] is None and o["dh0"] is None
    ref = oracle_bwd(d, cot)
    for k in ("dx", "ddt", "dA", "dB", "dC"):
        assert rel_err(o[k].float().cpu().double().numpy(), ref[k]) <= TOL["bf16"], k


def test_empty_sequence_and_batch(cuda_device):
    H, P, N = 3, 16, 8
    dhf = torch.randn(2, H, P, N, device=cuda_device)
    A = -torch.rand(H, device=cuda_device)
    x = torch.empty(2, 0, H, P, device=cuda_device)
    dt = torch.empty(2, 0, H, device=cuda_device)
    Bm = torch.empty(2, 0, 1, N, device=cuda_device)
    o = ssd.ssd_bwd(x, dt, A, Bm, Bm, None, None, torch.empty_like(x), dhf, chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o["dh0"], dhf)
    assert torch.all(o["dA"] == 0) and torch.all(o["dD"] == 0)
    o = ssd.ssd_bwd(x, dt, A, Bm, Bm, None, None, torch.empty_like(x), None, chunk=64)
    torch.cuda.synchronize()
    assert torch.all(o["dh0"] == 0)
    x0 = torch.empty(0, 5, H, P, device=cuda_device)
    o = ssd.ssd_bwd(x0, torch.empty(0, 5, H, device=cuda_device), A, torch.empty(0, 5, 1, N, device=cuda_device),
                    torch.empty(0, 5, 1, N, device=cuda_device), None, None, torch.empty_like(x0), None, chunk=64)
    torch.cuda.synchronize()
    assert torch.all(o["dA"] == 0) and torch.all(o["dD"] == 0)


def test_workload_mamba2_130m(cuda_device):
    """B8 L2048 H24 P64 N128, chunk 256, every gradient against the whole oracle."""
    d = draw("mamba2_130m")
    check(d, cot_of("mamba2_130m", d), 256, cuda_device)


def test_workload_mamba2_2p7b_row0(cuda_device):
    """B4 L8192 H80 P64 N128 (the launch the benchmark times): the per-row gradients of
    batch row 0 against the oracle on that row, dD against its plain reduction over
    every row, and dA from a launch on row 0 alone."""
    d = draw("mamba2_2p7b")
    cot = cot_of("mamba2_2p7b", d)
    got = run_bwd(d, cot, 256, cuda_device)
    ref = oracle_bwd(d, cot, batch_rows=(0, 1))
    tol = TOL["bf16"]
    for k in ("dx", "ddt", "dB", "dC", "dh0"):
        assert rel_err(got[k][:1], ref[k]) <= tol, k
    # dD_h = sum over (b, t, p) of dy * x: a plain reduction, every row
    H = d["x"].shape[2]
    dD = np.zeros(H)
    for b in range(d["x"].shape[0]):
        xb = d["x"].values((slice(b, b + 1),))
        dyb = cot["dy"].values((slice(b, b + 1),))
        dD += np.einsum("blhp,blhp->h", xb, dyb)
    assert rel_err(got["dD"], dD) <= tol
    row = {k: (v if v is None or k in ("A", "D") else _Row(v)) for k, v in d.items()}
    got1 = run_bwd(row, {k: _Row(v) if v is not None else None for k, v in cot.items()}, 256, cuda_device)
    assert rel_err(got1["dA"], ref["dA"]) <= tol


class _Row:
    """Batch row 0 of a drawn tensor, with the same interface as inputs.Tensor."""

    def __init__(self, t):
        self.t, self.dtype, self.shape = t, t.dtype, (1,) + t.shape[1:]

    def values(self, index=...):
        return self.t.values((slice(0, 1),))[index]

    @property
    def value(self):
        return self.values()

    def torch(self, device="cpu"):
        return self.t.torch(device)[:1].clone()


@pytest.mark.parametrize("h", [0, 79])
def test_workload_long_n256_sampled_heads(cuda_device, h):
    """B1 L65536 H80 P64 N256 with h0: dx, ddt, dh0, dA and dD of one head depend on that head's
    stream alone, so the oracle runs on the one head."""
    d = draw("long_n256")
    cot = cot_of("long_n256", d)
    got = run_bwd(d, cot, 256, cuda_device)
    sl = lambda t, ax: t.values((slice(None),) * ax + (slice(h, h + 1),))
    ref = oracle.backward(sl(d["x"], 2), sl(d["dt"], 2), d["A"].value[h:h + 1], d["B"].value, d["C"].value,
                          d["D"].value[h:h + 1], sl(d["h0"], 1), sl(cot["dy"], 2), sl(cot["dh_final"], 1))
    tol = TOL["bf16"]
    assert rel_err(got["dx"][:, :, h:h + 1], ref["dx"]) <= tol
    assert rel_err(got["ddt"][:, :, h:h + 1], ref["ddt"]) <= tol
    assert rel_err(got["dh0"][:, h:h + 1], ref["dh0"]) <= tol
    assert rel_err(got["dA"][h:h + 1], ref["dA"]) <= tol
    assert rel_err(got["dD"][h:h + 1], ref["dD"]) <= tol
