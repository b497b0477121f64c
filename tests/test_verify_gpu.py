"""GPU parity of ssd_verify against the oracle, and bit-exact ssd_select_state."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from ssd_cases import TOL, draw, gpu_inputs, rel_err, to_np
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def run_verify(d, dev):
    g = gpu_inputs(d, dev)
    y, so = ssd.ssd_verify(g["h0"], g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"])
    torch.cuda.synchronize()
    return g, y, so


def oracle_rows(d, rows):
    sl = (slice(rows[0], rows[1]),)
    return oracle.verify(d["h0"].values(sl), d["x"].values(sl), d["dt"].values(sl), d["A"].value,
                         d["B"].values(sl), d["C"].values(sl), d["D"].value)


def test_verify_workload_sampled_rows(cuda_device):
    """Full verify workload (B64 K8 H32 P128 N128 G8); rows 0-3 and 60-63 against the oracle."""
    d = draw("verify_k8")
    g, y, so = run_verify(d, cuda_device)
    for rows in ((0, 4), (60, 64)):
        yr, sr = oracle_rows(d, rows)
        assert rel_err(to_np(y[rows[0]:rows[1]]), yr) <= TOL["bf16"]
        assert rel_err(to_np(so[rows[0]:rows[1]]), sr) <= TOL["bf16"]
    # selection with the drawn accepted indices, checked bit for bit
    acc = torch.from_numpy(d["accepted"]).to(cuda_device)
    kept = ssd.ssd_select_state(g["h0"], so, acc)
    torch.cuda.synchronize()
    for b in range(d["accepted"].shape[0]):
        a = int(d["accepted"][b])
        want = g["h0"][b] if a == 0 else so[b, a - 1]
        assert torch.equal(kept[b].view(torch.int32), want.view(torch.int32)), b


@pytest.mark.parametrize("K,H,P,G,N,dtype", [(1, 4, 64, 1, 128, "bf16"), (3, 4, 16, 2, 16, "f32"),
                                              (8, 8, 128, 8, 256, "bf16"), (5, 2, 8, 1, 4, "f32")])
def test_verify_small_full(cuda_device, K, H, P, G, N, dtype):
    wl = dataclasses.replace(inputs.WORKLOADS["verify_k8"], batch=3, seqlen=K, nheads=H, headdim=P,
                             ngroups=G, dstate=N, dtype=dtype, seed=40 + K)
    d = inputs.draw(wl)
    g, y, so = run_verify(d, cuda_device)
    yr, sr = oracle_rows(d, (0, 3))
    assert rel_err(to_np(y), yr) <= TOL[dtype]
    assert rel_err(to_np(so), sr) <= TOL[dtype]


def test_verify_matches_fwd_final_states(cuda_device):
    """states_out[k] from verify equals h_final of a forward run over the first k+1 tokens."""
    wl = dataclasses.replace(inputs.WORKLOADS["verify_k8"], batch=2, nheads=4, ngroups=2, seed=9)
    d = inputs.draw(wl)
    g, y, so = run_verify(d, cuda_device)
    for k in range(8):
        sl = lambda t: t[:, :k + 1].contiguous()
        yf, hf = ssd.ssd_fwd(sl(g["x"]), sl(g["dt"]), g["A"], sl(g["B"]), sl(g["C"]), g["D"], g["h0"], chunk=4)
        torch.cuda.synchronize()
        assert rel_err(to_np(so[:, k]), to_np(hf)) <= 1e-3
        assert rel_err(to_np(y[:, k]), to_np(yf[:, k])) <= TOL["bf16"]


def test_select_every_index_and_out_of_range(cuda_device):
    Bsz, K, H, P, N = 12, 8, 3, 16, 8
    h0 = torch.randn(Bsz, H, P, N, device=cuda_device)
    so = torch.randn(Bsz, K, H, P, N, device=cuda_device)
    acc = torch.tensor([0, 1, 2, 3, 4, 5, 6, 7, 8, -1, 9, 8], dtype=torch.int32, device=cuda_device)
    kept = ssd.ssd_select_state(h0, so, acc)
    torch.cuda.synchronize()
    for b in range(9):
        want = h0[b] if b == 0 else so[b, b - 1]
        assert torch.equal(kept[b].view(torch.int32), want.view(torch.int32))
    assert torch.isnan(kept[9]).all() and torch.isnan(kept[10]).all()
    assert torch.equal(kept[11], so[11, 7])
