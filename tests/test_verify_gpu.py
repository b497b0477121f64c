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


def test_verify_workload_every_row(cuda_device):
    """Full verify workload (B64 K8 H32 P128 N128 G8): every row against the oracle, each row
    (its K outputs and K states) on its own scale."""
    d = draw("verify_k8")
    g, y, so = run_verify(d, cuda_device)
    Bsz = d["x"].shape[0]
    yr, sr = oracle_rows(d, (0, Bsz))
    yg, sg = to_np(y), to_np(so)
    for b in range(Bsz):
        assert rel_err(yg[b], yr[b]) <= TOL["bf16"], b
        assert rel_err(sg[b], sr[b]) <= TOL["bf16"], b
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


def test_verify_outputs_only_and_advance_state_full_workload(cuda_device):
    """The flow that keeps one state instead of K (full verify workload): verify with no
    states_out (the chunked form over the K tokens) matches the oracle and the recurrent form,
    and the state recomputed for the drawn accepted counts equals ssd_select_state over the
    stored states bit for bit, also in place."""
    d = draw("verify_k8")
    g, y, so = run_verify(d, cuda_device)
    y2, none = ssd.ssd_verify(g["h0"], g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], return_states=False)
    acc = torch.from_numpy(d["accepted"]).to(cuda_device)
    kept = ssd.ssd_select_state(g["h0"], so, acc)
    adv = ssd.ssd_advance_state(g["h0"], g["x"], g["dt"], g["A"], g["B"], acc)
    inplace = g["h0"].clone()
    ret = ssd.ssd_advance_state(inplace, g["x"], g["dt"], g["A"], g["B"], acc, h_keep=inplace)
    torch.cuda.synchronize()
    assert none is None and ret is inplace
    assert rel_err(to_np(y2), to_np(y)) <= 1e-2
    yr, _ = oracle_rows(d, (0, d["x"].shape[0]))
    y2n = to_np(y2)
    for b in range(y2n.shape[0]):
        assert rel_err(y2n[b], yr[b]) <= TOL["bf16"], b
    assert torch.equal(adv.view(torch.int32), kept.view(torch.int32))
    assert torch.equal(inplace.view(torch.int32), kept.view(torch.int32))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_advance_state_every_count(cuda_device, dtype):
    """Every accepted count 0..K on its own row, plus two out-of-range rows (NaN), against the
    stored verify states bit for bit and against the oracle's state after that many tokens."""
    K = 6
    wl = dataclasses.replace(inputs.WORKLOADS["verify_k8"], batch=K + 3, seqlen=K, nheads=4, headdim=32,
                             ngroups=2, dstate=64, dtype=dtype, seed=77)
    d = inputs.draw(wl)
    g, y, so = run_verify(d, cuda_device)
    acc_list = list(range(K + 1)) + [-1, K + 1]
    acc = torch.tensor(acc_list, dtype=torch.int32, device=cuda_device)
    adv = ssd.ssd_advance_state(g["h0"], g["x"], g["dt"], g["A"], g["B"], acc)
    torch.cuda.synchronize()
    _, sr = oracle_rows(d, (0, K + 3))
    h0r = d["h0"].value
    for b, a in enumerate(acc_list):
        if a < 0 or a > K:
            assert torch.isnan(adv[b]).all()
            continue
        want = g["h0"][b] if a == 0 else so[b, a - 1]
        assert torch.equal(adv[b].view(torch.int32), want.view(torch.int32)), b
        ref = h0r[b] if a == 0 else sr[b, a - 1]
        assert rel_err(to_np(adv[b]), ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,H,P,G,N", [("bf16", 32, 128, 8, 128), ("f32", 4, 16, 2, 16), ("bf16", 3, 8, 1, 256)])
def test_decode_step(cuda_device, dtype, H, P, G, N):
    """One token in place: equals ssd_verify with K = 1 bit for bit (y and state), and the oracle."""
    wl = dataclasses.replace(inputs.WORKLOADS["verify_k8"], batch=5, seqlen=1, nheads=H, headdim=P, ngroups=G,
                             dstate=N, dtype=dtype, seed=91)
    d = inputs.draw(wl)
    g, y, so = run_verify(d, cuda_device)
    state = g["h0"].clone()
    yd = ssd.ssd_decode_step(state, g["x"][:, 0].contiguous(), g["dt"][:, 0].contiguous(), g["A"],
                             g["B"][:, 0].contiguous(), g["C"][:, 0].contiguous(), g["D"])
    torch.cuda.synchronize()
    assert torch.equal(state.view(torch.int32), so[:, 0].view(torch.int32))
    assert torch.equal(yd.float(), y[:, 0].float())
    yr, sr = oracle_rows(d, (0, 5))
    assert rel_err(to_np(yd), yr[:, 0]) <= TOL[dtype]
    assert rel_err(to_np(state), sr[:, 0]) <= TOL[dtype]


@pytest.mark.parametrize("K,H,P,G,N,dtype", [(1, 4, 64, 1, 128, "bf16"), (3, 4, 16, 2, 16, "f32"),
                                              (8, 8, 128, 8, 256, "bf16"), (5, 2, 8, 1, 4, "f32"),
                                              (64, 2, 16, 1, 32, "f32")])
def test_verify_outputs_only_small(cuda_device, K, H, P, G, N, dtype):
    """Outputs only (chunked form over K tokens) against the oracle, K from 1 to the maximum."""
    wl = dataclasses.replace(inputs.WORKLOADS["verify_k8"], batch=3, seqlen=K, nheads=H, headdim=P,
                             ngroups=G, dstate=N, dtype=dtype, seed=140 + K)
    d = inputs.draw(wl)
    g = gpu_inputs(d, cuda_device)
    y, none = ssd.ssd_verify(g["h0"], g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], return_states=False)
    torch.cuda.synchronize()
    yr, _ = oracle_rows(d, (0, 3))
    assert none is None and rel_err(to_np(y), yr) <= TOL[dtype]
