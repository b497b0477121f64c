"""Context-parallel kernels on one GPU: R ranks are emulated one after another on the
same device (each "rank" is a plain sequence of launches on its own segment; the
all-gather becomes a stack of the per-rank results, so no kernel waits on another).
The concatenated outputs and the last segment's end state must match the oracle over
the whole sequence, and, at the long-context shape, the single-GPU forward."""
import dataclasses

import numpy as np
import pytest
import torch

from ssd_cases import TOL, gpu_inputs, oracle_full, oracle_stream, rel_err, to_np
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs
from state_space_sequence_chunked_b200.context_parallel import segment_bounds, ssd_fwd_context_parallel

pytestmark = pytest.mark.gpu


def emulate(g, R, chunk):
    """Per-rank forward + decay, the gathered tensors, then combine and correct per rank."""
    L = g["x"].shape[1]
    segs, ys, hs, bds, tots = [], [], [], [], []
    for r in range(R):
        lo, hi = segment_bounds(L, R, r)
        sl = lambda k: g[k][:, lo:hi].clone()  # its own allocation, as on a real rank (16-byte aligned)
        y, h = ssd.ssd_fwd(sl("x"), sl("dt"), g["A"], sl("B"), sl("C"), g["D"], g["h0"] if r == 0 else None,
                           chunk=chunk)
        bd, tot = ssd.ssd_cp_decay(sl("dt"), g["A"])
        segs.append((lo, hi)); ys.append(y); hs.append(h); bds.append(bd); tots.append(tot)
    states, totals = torch.stack(hs), torch.stack(tots)
    ends = []
    status = torch.zeros(4, dtype=torch.int32, device=g["x"].device)
    for r in range(R):
        lo, hi = segs[r]
        s_in, h_end = ssd.ssd_cp_combine(states, totals, r)
        if r > 0:
            ssd.ssd_cp_correct(g["dt"][:, lo:hi].clone(), g["A"], g["C"][:, lo:hi].clone(), bds[r], s_in, ys[r],
                               status=status)
        ends.append(h_end)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0, "a bounded wait of the correction ran out"
    return torch.cat(ys, dim=1), ends


CASES = [
    # (workload, overrides, R): the tensor-core correction (bf16, P = 64, N = 128), fp32 on CUDA
    # cores, bf16 with a head dimension the tiles do not take, ragged segments
    ("mamba2_130m", dict(batch=2, seqlen=1000, nheads=4, h0_std=0.2, seed=301), 3),
    ("mamba2_130m", dict(batch=1, seqlen=700, nheads=6, ngroups=2, h0_std=0.0, seed=302), 2),
    ("tiny_fp32", dict(batch=2, seqlen=300, h0_std=0.3, seed=303), 4),
    ("mamba2_130m", dict(batch=2, seqlen=389, nheads=4, headdim=16, dstate=32, h0_std=0.1, seed=304), 3),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-R{c[2]}-{i}" for i, c in enumerate(CASES)])
def test_emulated_ranks_match_the_oracle(cuda_device, case):
    name, over, R = case
    wl = dataclasses.replace(inputs.WORKLOADS[name], **over)
    d = inputs.draw(wl)
    g = gpu_inputs(d, cuda_device)
    y, ends = emulate(g, R, wl.chunk)
    yr, hr = oracle_full(d)
    tol = TOL[wl.dtype]
    assert rel_err(to_np(y), yr) <= tol
    assert rel_err(to_np(ends[-1]), hr) <= tol


def test_decay_sums(cuda_device):
    """Block and total sums of dt*A against fp64 sums (fp32 accumulation tolerance)."""
    d = inputs.draw(inputs.WORKLOADS["mamba2_130m"], batch=2, seqlen=1000, seed=305)
    g = gpu_inputs(d, cuda_device)
    bd, tot = ssd.ssd_cp_decay(g["dt"], g["A"])
    torch.cuda.synchronize()
    a = d["dt"].value * d["A"].value[None, None, :]
    want = np.stack([a[:, k * 128:(k + 1) * 128].sum(axis=1) for k in range(8)], axis=-1)
    assert np.max(np.abs(to_np(bd) - want)) <= 1e-5 * np.max(np.abs(want))
    assert np.max(np.abs(to_np(tot) - a.sum(axis=1))) <= 1e-5 * np.max(np.abs(a.sum(axis=1)))


def test_long_context_shape_eight_ranks(cuda_device):
    """The long-context large-state shape (B1 L65536 H80 P64 N256, h0 ~ N(0, 0.1)) cut into 8
    segments: the tensor-core correction at N = 256, against the single-GPU forward over the
    whole sequence, and against the oracle on sampled heads."""
    wl = inputs.WORKLOADS["long_n256"]
    d = inputs.draw(wl)
    g = gpu_inputs(d, cuda_device)
    y, ends = emulate(g, 8, wl.chunk)
    y1, h1 = ssd.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["h0"], chunk=wl.chunk)
    torch.cuda.synchronize()
    assert rel_err(to_np(y), to_np(y1)) <= TOL["bf16"]
    assert rel_err(to_np(ends[-1]), to_np(h1)) <= TOL["bf16"]
    for h in (0, 79):
        yr, hr = oracle_stream(d, 0, h)
        assert rel_err(to_np(y[0, :, h]), yr) <= TOL["bf16"]
        assert rel_err(to_np(ends[-1][0, h]), hr) <= TOL["bf16"]


def test_one_rank_is_the_plain_forward(cuda_device):
    d = inputs.draw(inputs.WORKLOADS["mamba2_130m"], batch=1, seqlen=300, seed=306, h0_std=0.1)
    g = gpu_inputs(d, cuda_device)
    y, h = ssd_fwd_context_parallel(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["h0"], chunk=256)
    y1, h1 = ssd.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["h0"], chunk=256)
    torch.cuda.synchronize()
    assert torch.equal(y.float(), y1.float()) and torch.equal(h, h1)
