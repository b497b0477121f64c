"""GPU parity of ssd_fwd against the fp64 oracle: max|y - y_ref| / max|y_ref| and
the same for the final state, <= 1e-4 for fp32 inputs and <= 2e-2 for bf16."""
import dataclasses

import numpy as np
import pytest
import torch

from ssd_cases import TOL, draw, oracle_full, oracle_stream, plan_of, rel_err, run_fwd, sample_streams, to_np
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs

pytestmark = pytest.mark.gpu


def check_full(d, chunk, dev, **kw):
    y, hf = run_fwd(d, chunk, dev, **kw)
    yr, hr = oracle_full(d, **kw)
    tol = TOL[d["x"].dtype]
    ey, eh = rel_err(to_np(y), yr), rel_err(to_np(hf), hr)
    assert ey <= tol and eh <= tol, (ey, eh)
    return ey, eh


def test_tiny_fp32_workload(cuda_device):
    """The fp32 workload at full size (B1 L256 H4 P16 N16, chunk 64)."""
    d = draw("tiny_fp32")
    ey, eh = check_full(d, 64, cuda_device)
    assert ey < 1e-5


@pytest.mark.parametrize("chunk", [1, 7, 64, 100, 256])
def test_tiny_fp32_any_chunk(cuda_device, chunk):
    d = draw("tiny_fp32", seqlen=201, h0_std=0.5)
    check_full(d, chunk, cuda_device)


BF16_CASES = [
    # (batch, seqlen, nheads, headdim, ngroups, dstate, chunk, h0_std)
    (2, 600, 4, 64, 1, 128, 256, 0.0),     # several chunks, ragged tail
    (1, 700, 6, 64, 2, 128, 256, 0.1),     # groups, initial state
    (2, 300, 4, 64, 4, 256, 256, 0.1),     # N = 256, one group per head
    (1, 257, 2, 64, 1, 128, 128, 0.0),     # tail of one token
    (3, 100, 3, 32, 1, 64, 64, 0.2),
    (1, 50, 2, 128, 1, 128, 256, 0.1),     # sequence shorter than a chunk
    (1, 1, 2, 64, 1, 128, 256, 0.1),       # a single token
]


@pytest.mark.parametrize("case", BF16_CASES)
def test_bf16_small(cuda_device, case):
    Bsz, L, H, P, G, N, Q, std = case
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_130m"], batch=Bsz, seqlen=L, nheads=H, headdim=P,
                             ngroups=G, dstate=N, chunk=Q, h0_std=std, seed=1000 + L)
    d = inputs.draw(wl)
    check_full(d, Q, cuda_device)


def test_no_D_no_h0(cuda_device):
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_130m"], batch=2, seqlen=400, nheads=4, h0_std=0.3, seed=77)
    d = inputs.draw(wl)
    check_full(d, 256, cuda_device, use_D=False, use_h0=False)
    check_full(d, 256, cuda_device, use_D=True, use_h0=False)


def test_seqlen_zero_copies_initial_state(cuda_device):
    h0 = torch.randn(2, 3, 16, 8, device=cuda_device)
    x = torch.empty(2, 0, 3, 16, device=cuda_device)
    dt = torch.empty(2, 0, 3, device=cuda_device)
    Bm = torch.empty(2, 0, 1, 8, device=cuda_device)
    A = -torch.rand(3, device=cuda_device)
    y, hf = ssd.ssd_fwd(x, dt, A, Bm, Bm, None, h0, chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(hf, h0)
    y, hf = ssd.ssd_fwd(x, dt, A, Bm, Bm, None, None, chunk=64)
    torch.cuda.synchronize()
    assert torch.count_nonzero(hf) == 0


@pytest.mark.parametrize("name", ["mamba2_130m", "mamba2_2p7b", "long_n256"])
def test_bf16_workloads_take_the_tensor_core_path(name):
    wl = inputs.WORKLOADS[name]
    d = inputs.draw(wl, batch=1, seqlen=8)
    assert plan_of(d, wl.chunk)["path"] == "tcgen05"


def _tc_case(seed, **kw):
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_130m"], batch=1, seqlen=128, nheads=1, h0_std=0.5, seed=seed)
    return inputs.draw(dataclasses.replace(wl, **kw))


def _zeroed(d, *names):
    d = dict(d)
    for n in names:
        if n == "h0":
            d["h0"] = None
            continue
        t = d[n]
        z = object.__new__(type(t))
        z.__dict__.update(t.__dict__)
        z.bits = np.zeros_like(t.bits)
        z._value = None
        d[n] = z
    return d


@pytest.mark.parametrize("nheads", [1, 2])
@pytest.mark.parametrize("what", ["skip", "state_to_output", "diagonal_block", "all"])
def test_tensor_core_products_in_isolation(cuda_device, what, nheads):
    """One 128-token block with all but one product switched off, so a wrong
    operand layout shows up as exactly one failing case:
    skip: dt = 0, h0 = 0 -> y = D x;  state_to_output: dt = 0, x = 0, D = 0 -> y = C h0^T;
    diagonal_block: h0 = 0, D = 0 -> y = (C B^T o L) (dt x), h_final = chunk state.
    One head runs the one-head kernel, two heads the head-pair kernel (dt = 0 on valid
    tokens sends a pair task to its single-head exact form)."""
    d = _tc_case(7, nheads=nheads)
    zero = {"skip": ("dt", "h0"), "state_to_output": ("dt", "x", "D"), "diagonal_block": ("h0", "D"),
            "all": ()}[what]
    d = _zeroed(d, *zero)
    assert plan_of(d, 128)["path"] == "tcgen05"
    check_full(d, 128, cuda_device)


@pytest.mark.parametrize("chunk", [128, 256])
def test_wide_decay_and_zero_step_blocks(cuda_device, chunk):
    """The tensor-core path evaluates a block in factored form only when its decay range
    is small enough (2^128 for the one-head kernel, 2^192 for the head-pair kernel) and no
    token has |dt| < 2^-40; other blocks take the elementwise form. Here the kinds alternate
    within streams: head 0 has one block with dt = 1 (range 128 * 2 * log2 e = 369), head 1
    has A = 0 (no decay), head 2 has one token with dt = 0, head 3 decays by 2^-11.5 per
    token everywhere, head 4 has one block of range 128 * 0.9 * log2 e = 166 (factored by
    the pair kernel, elementwise by the one-head kernel) and head 5 one of range 191."""
    d = _tc_case(21, batch=2, seqlen=700, nheads=6, h0_std=0.2)
    dt = d["dt"].value.copy()
    dt[0, 128:256, 0] = 1.0
    dt[1, 300, 2] = 0.0
    dt[:, :, 3] = 0.5
    dt[0, 256:384, 4] = 0.9
    dt[1, 384:512, 5] = 1.0
    d["dt"] = inputs.Tensor(dt, "bf16")
    d["A"] = inputs.Tensor(np.array([-2.0, 0.0, -4.0, -16.0, -1.0, -1.035]), "f32")
    assert plan_of(d, chunk)["path"] == "tcgen05"
    check_full(d, chunk, cuda_device)


@pytest.mark.parametrize("chunk", [128, 256])
def test_tensor_core_path_matches_cuda_core_path(cuda_device, chunk):
    """Same inputs through both CUDA paths (chunk 64 selects the fp32 CUDA-core path)."""
    d = _tc_case(11, batch=2, seqlen=777, nheads=4, ngroups=2, h0_std=0.2)
    assert plan_of(d, chunk)["path"] == "tcgen05" and plan_of(d, 64)["path"] == "simt"
    y1, h1 = run_fwd(d, chunk, cuda_device)
    y2, h2 = run_fwd(d, 64, cuda_device)
    assert rel_err(to_np(y1), to_np(y2)) <= 2e-2
    assert rel_err(to_np(h1), to_np(h2)) <= 2e-2


@pytest.mark.parametrize("name,nstreams", [("mamba2_130m", 6), ("mamba2_2p7b", 4), ("long_n256", 3)])
def test_full_size_sampled_streams(cuda_device, name, nstreams):
    """Full-size workloads in the benchmark's launch configuration; sampled (b, h)
    streams are recomputed one by one by the oracle over the whole sequence."""
    wl = inputs.WORKLOADS[name]
    d = draw(name)
    y, hf = run_fwd(d, wl.chunk, cuda_device)
    yn = y.float()
    assert not torch.isnan(yn).any()
    assert not torch.isnan(hf).any()
    tol = TOL[wl.dtype]
    for (b, h) in sample_streams(wl.batch, wl.nheads, nstreams):
        yr, hr = oracle_stream(d, b, h)
        ey = rel_err(yn[b, :, h, :].cpu().double().numpy(), yr)
        eh = rel_err(hf[b, h].cpu().double().numpy(), hr)
        assert ey <= tol and eh <= tol, (b, h, ey, eh)
