"""ssd_fwd_static_scratch: the forward pass for callers that cannot allocate
device memory (a server that reserves all of HBM itself, a real-time loop, a
plugin whose host owns every allocation). Its intermediates live in a built-in
device array instead of a caller-provided workspace. Two calls in a row -- a
larger problem, then a smaller one over the scratch the first left behind -- must
each match the fp64 oracle and ssd_fwd (the entry point with a workspace) on the
same inputs, without allocating device memory; a problem too large for the array
must be refused.

This file is collected last on purpose: it is the newest entry point, and a run
that stops at the first failure has already run every other test by then."""
import ctypes
import dataclasses

import pytest
import torch

import oracle
from ssd_cases import TOL, rel_err, to_np
from state_space_sequence_chunked_b200 import _binding as ssd
from state_space_sequence_chunked_b200 import inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def static_fwd():
    f = ssd.lib().ssd_fwd_static_scratch
    vp = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(ssd.ShapeT), ctypes.c_int] + [vp] * 7 + [ctypes.c_int64, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def call_static(g, h0, chunk, y, hf):
    Bsz, L, H, P = g["x"].shape
    G, N = g["B"].shape[2], g["B"].shape[3]
    shape = ssd.ShapeT(Bsz, L, H, P, G, N)
    code = ssd.SSD_BF16 if g["x"].dtype == torch.bfloat16 else ssd.SSD_F32
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return static_fwd()(ctypes.byref(shape), code, p(g["x"]), p(g["dt"]), p(g["A"]), p(g["B"]), p(g["C"]),
                        p(g["D"]), p(h0), chunk, p(y), p(hf), stream)


def draw_case(dtype, seed, h0_std, batch, seqlen, nheads):
    wl = dataclasses.replace(inputs.WORKLOADS["mamba2_130m"], batch=batch, seqlen=seqlen, nheads=nheads, ngroups=2,
                             dtype=dtype, seed=seed, h0_std=h0_std)
    return wl, inputs.draw(wl)


def device_bytes_in_use():
    free, total = torch.cuda.mem_get_info()
    return total - free


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_two_calls_match_oracle_and_ssd_fwd(cuda_device, dtype):
    # the first call fills more of the scratch (more chunks and heads) than the second reads
    cases = [(501, 0.1, 2, 1500, 8), (502, 0.0, 1, 700, 6)]
    # one call first, so that loading the module (its code and the built-in array) is not
    # counted as an allocation of the calls below
    wl, d = draw_case(dtype, 500, 0.0, 1, 300, 2)
    g = {k: d[k].torch(cuda_device) for k in ("x", "dt", "A", "B", "C", "D")}
    assert call_static(g, None, 256, torch.empty_like(g["x"]), None) == 0
    torch.cuda.synchronize()
    for call, (seed, std, Bsz, L, H) in enumerate(cases):
        wl, d = draw_case(dtype, seed, std, Bsz, L, H)
        g = {k: d[k].torch(cuda_device) for k in ("x", "dt", "A", "B", "C", "D")}
        h0 = d["h0"].torch(cuda_device) if d["h0"] is not None else None
        # the static path runs the fp32 CUDA-core kernels whatever the dtype: size it by their plan
        need = ssd.fwd_plan(wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.ngroups, wl.dstate, ssd.SSD_F32,
                            256)["workspace_bytes"]
        assert ssd.fwd_plan(wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.ngroups, wl.dstate, ssd.SSD_F32,
                            256)["path"] == "simt"
        assert 0 < need <= SCRATCH_BYTES
        y = torch.full_like(g["x"], float("nan"))
        hf = torch.full((wl.batch, wl.nheads, wl.headdim, wl.dstate), float("nan"), device=cuda_device)
        torch.cuda.synchronize()
        alloc0, used0 = torch.cuda.memory_allocated(cuda_device), device_bytes_in_use()
        assert call_static(g, h0, 256, y, hf) == 0, f"call {call}"
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated(cuda_device) == alloc0, f"call {call}"
        assert device_bytes_in_use() == used0, f"call {call}: device memory in use changed"
        yr, hr = oracle.recurrent(d["x"].value, d["dt"].value, d["A"].value, d["B"].value, d["C"].value,
                                  d["D"].value, d["h0"].value if d["h0"] is not None else None)
        assert rel_err(to_np(y), yr) <= TOL[dtype], f"call {call}"
        assert rel_err(to_np(hf), hr) <= TOL[dtype], f"call {call}"
        y_ref, hf_ref = ssd.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], h0, chunk=256)
        torch.cuda.synchronize()
        assert rel_err(to_np(y), to_np(y_ref)) <= TOL[dtype], f"call {call}"
        assert rel_err(to_np(hf), to_np(hf_ref)) <= TOL[dtype], f"call {call}"


def test_too_large_is_refused_without_launch(cuda_device):
    # B1 L65536 H8 P64 N128 chunk 256 needs 256 chunks x 8 heads x 32 KB of chunk states
    Bsz, L, H, P, N = 1, 65536, 8, 64, 128
    g = {"x": torch.zeros(Bsz, L, H, P, dtype=torch.bfloat16, device=cuda_device),
         "dt": torch.zeros(Bsz, L, H, dtype=torch.bfloat16, device=cuda_device),
         "A": torch.zeros(H, device=cuda_device), "D": None,
         "B": torch.zeros(Bsz, L, 1, N, dtype=torch.bfloat16, device=cuda_device)}
    g["C"] = g["B"]
    y = torch.full_like(g["x"], 7.0)
    assert call_static(g, None, 256, y, None) == 4  # SSD_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
