"""The tensor-core forward's bounded waits, made to run out on purpose.

Every wait of the fused kernels (on a shared-memory barrier phase, or on the counter
through which a CTA hands a cut stream's state to the next) gives up after a limit,
raises the CTA's abort flag and sets bit 0 of the status word at the start of the
workspace. Here the limit is cut to 1 us through the library's test hook, on shapes
with at least as many streams as SMs (so streams are cut between CTAs and states are
handed over), for both kernels: head pairs (an even head count at N = 128) and single
heads (an odd head count, or N = 256). The call must come back, report SSD_ERR_TIMEOUT through ssd_fwd_status,
and leave the GPU usable: the next call, with the normal limit, must match the oracle
(it allocates the same tensor memory, which the aborted CTAs therefore released).
No fault, trap or unbounded wait is involved."""
import dataclasses

import pytest
import torch

from ssd_cases import TOL, gpu_inputs, oracle_stream, plan_of, rel_err
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs

pytestmark = pytest.mark.gpu

SSD_ERR_TIMEOUT = 6


def _case(dstate, nheads, seed):
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_2p7b"], batch=1, seqlen=2048, nheads=nheads,
                             dstate=dstate, seed=seed)
    return wl, inputs.draw(wl)


@pytest.mark.parametrize("dstate,nheads", [(128, 320), (256, 320), (128, 161), (256, 161)])
def test_wait_limit_runs_out_then_next_call_is_exact(cuda_device, dstate, nheads):
    wl, d = _case(dstate, nheads, 900 + dstate)
    plan = plan_of(d, wl.chunk)
    assert plan["path"] == "tcgen05"
    g = gpu_inputs(d, cuda_device)
    shape = (wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.ngroups, wl.dstate)
    ws = torch.zeros(plan["workspace_bytes"], dtype=torch.uint8, device=cuda_device)
    y = torch.empty_like(g["x"])
    hf = torch.empty(wl.batch, wl.nheads, wl.headdim, wl.dstate, device=cuda_device)

    ssd.set_wait_limit_us(1)
    try:
        with pytest.raises(ssd.SSDError) as err:  # check=True reads the status word after the launch
            ssd.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], None, chunk=wl.chunk, y=y, h_final=hf,
                        workspace=ws, check=True)
    finally:
        ssd.set_wait_limit_us(0)
    assert err.value.status == SSD_ERR_TIMEOUT
    word = int(ws[:4].view(torch.int32).item())
    assert word & 1, f"no wait ran out (status word {word})"
    assert ssd.fwd_status(shape, ssd.SSD_BF16, wl.chunk, ws) == SSD_ERR_TIMEOUT

    # the same call at the normal limit: status clear, results exact
    y.fill_(float("nan"))
    hf.fill_(float("nan"))
    ssd.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], None, chunk=wl.chunk, y=y, h_final=hf,
                workspace=ws, check=True)
    assert int(ws[:4].view(torch.int32).item()) == 0
    yn = y.float()
    for (b, h) in [(0, 0), (0, nheads // 2 + 1), (0, nheads - 1)]:
        yr, hr = oracle_stream(d, b, h)
        ey = rel_err(yn[b, :, h, :].cpu().double().numpy(), yr)
        eh = rel_err(hf[b, h].cpu().double().numpy(), hr)
        assert ey <= TOL["bf16"] and eh <= TOL["bf16"], (b, h, ey, eh)
