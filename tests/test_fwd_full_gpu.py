"""Exhaustive full-size parity of ssd_fwd: every (batch, head) stream of each bf16
forward workload, in the benchmark's launch configuration, against the fp64 oracle
(the token-by-token recurrence) over the whole sequence. Per stream:
max|y - y_ref| / max|y_ref| and the same for the final state, <= 2e-2.

Also the shapes that cut streams between CTAs (at least as many streams as SMs,
so a stream's state is handed from one CTA to the next inside a block sequence),
for both tensor-core kernels, with a nonzero initial state."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from ssd_cases import TOL, plan_of, run_fwd
from state_space_sequence_chunked_b200 import inputs

pytestmark = pytest.mark.gpu

HEAD_BLOCK = 16  # heads per oracle call (bounds host memory on the long workload)


def stream_errors(d, y, hf):
    """Per-stream relative errors of y [B,L,H,P] and hf [B,H,P,N] (torch, on the GPU)."""
    Bsz, L, H, P = d["x"].shape
    G = d["B"].shape[2]
    hpg = H // G
    ey = np.zeros((Bsz, H))
    eh = np.zeros((Bsz, H))
    for h0 in range(0, H, HEAD_BLOCK):
        h1 = min(H, h0 + HEAD_BLOCK)
        g0, g1 = h0 // hpg, (h1 - 1) // hpg + 1
        hs, gs = (slice(None), slice(None), slice(h0, h1)), (slice(None), slice(None), slice(g0, g1))
        # the head -> group map of the slice must stay that of the whole problem
        assert G == 1 or (h0 % hpg == 0 and (h1 - h0) % hpg == 0)
        init = d["h0"].values((slice(None), slice(h0, h1))) if d["h0"] is not None else None
        yr, hr = oracle.recurrent(d["x"].values(hs), d["dt"].values(hs), d["A"].value[h0:h1], d["B"].values(gs),
                                  d["C"].values(gs), d["D"].value[h0:h1], init)
        yg = y[:, :, h0:h1, :].float().cpu().double().numpy()
        hg = hf[:, h0:h1].cpu().double().numpy()
        assert np.all(np.isfinite(yg)) and np.all(np.isfinite(hg))
        ey[:, h0:h1] = np.max(np.abs(yg - yr), axis=(1, 3)) / np.maximum(np.max(np.abs(yr), axis=(1, 3)), 1e-30)
        eh[:, h0:h1] = np.max(np.abs(hg - hr), axis=(2, 3)) / np.maximum(np.max(np.abs(hr), axis=(2, 3)), 1e-30)
    return ey, eh


def assert_every_stream(d, chunk, device):
    y, hf = run_fwd(d, chunk, device)
    ey, eh = stream_errors(d, y, hf)
    bad = [(b, h, ey[b, h], eh[b, h]) for b in range(ey.shape[0]) for h in range(ey.shape[1])
           if not (ey[b, h] <= TOL["bf16"] and eh[b, h] <= TOL["bf16"])]
    assert not bad, bad[:8]
    return ey, eh


@pytest.mark.parametrize("name", ["mamba2_130m", "mamba2_2p7b", "long_n256", "mamba2_2p7b_softplus_dt"])
def test_every_stream_full_size(cuda_device, name):
    wl = inputs.WORKLOADS[name]
    d = inputs.draw(wl)
    assert plan_of(d, wl.chunk)["path"] == "tcgen05"
    ey, eh = assert_every_stream(d, wl.chunk, cuda_device)
    print(f"{name}: worst stream y {ey.max():.3e}, h_final {eh.max():.3e}")


def cut_streams(nstreams, nblocks, sms):
    """Streams split between two CTAs' shares, by the kernels' share rule: the stream-major
    (stream, block) tasks cut into min(sms, nstreams) near-equal contiguous shares, share i
    starting at task q i + (r i) // grid (q, r = divmod(total, grid))."""
    grid = max(1, min(sms, nstreams))
    total = nstreams * nblocks
    q, r = divmod(total, grid)
    starts = [q * i + (r * i) // grid for i in range(1, grid)]
    return sorted({st // nblocks for st in starts if st % nblocks != 0})


@pytest.mark.parametrize("dstate,nheads", [(128, 300), (256, 300), (128, 151), (256, 153)])
def test_cut_streams_every_stream(cuda_device, dstate, nheads):
    """150 to 300 streams of 16 blocks over 148 CTAs: head pairs (300 heads at N = 128, the
    head-pair kernel) or single heads (an odd head count, or N = 256: the one-head kernel).
    The shares are 16.2 to 32.4 blocks long, so nearly every stream is split between two
    CTAs at a different block, and its state crosses through the hand-over buffer."""
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_2p7b"], batch=1, seqlen=2048, nheads=nheads, dstate=dstate,
                             h0_std=0.2, seed=40 + dstate)
    d = inputs.draw(wl)
    assert plan_of(d, wl.chunk)["path"] == "tcgen05"
    ey, eh = assert_every_stream(d, wl.chunk, cuda_device)
    # the streams the share rule cuts, named explicitly (they are among those checked above)
    pair = dstate == 128 and nheads % 2 == 0
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    cut = cut_streams(wl.batch * (nheads // 2 if pair else nheads), wl.seqlen // 128, sms)
    assert len(cut) > 100, len(cut)
    heads = [h for c in cut for h in ((2 * c, 2 * c + 1) if pair else (c,))]
    assert max(ey[0, heads]) <= TOL["bf16"] and max(eh[0, heads]) <= TOL["bf16"]
