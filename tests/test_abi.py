"""The C ABI without a GPU: the library loads, exports every function that
include/*.h declares, sizes its workspace, and rejects bad arguments before it
launches anything."""
import ctypes
import glob
import os
import re

import pytest

from state_space_sequence_chunked_b200 import _binding as B
from state_space_sequence_chunked_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(ssd_[A-Za-z0-9_]+)\s*\(", text, re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("ssd_fwd", "ssd_verify", "ssd_select_state", "ssd_fwd_workspace_bytes", "ssd_strerror",
              "ssd_advance_state", "ssd_decode_step", "ssd_cp_decay", "ssd_cp_combine", "ssd_cp_correct",
              "ssd_bwd", "ssd_bwd_workspace_bytes", "ssd_conv_split", "ssd_gated_rmsnorm"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_strerror(lib):
    for code in range(7):
        assert lib.ssd_strerror(code)
    assert lib.ssd_strerror(99) == b"unknown status"


def ws(shape, dtype=B.SSD_BF16, chunk=256):
    out = ctypes.c_size_t(0)
    st = B.lib().ssd_fwd_workspace_bytes(ctypes.byref(B.ShapeT(*shape)), dtype, chunk, ctypes.byref(out))
    return st, out.value


def test_workspace_bytes(lib):
    st, n = ws((4, 8192, 80, 64, 1, 128))
    assert st == 0 and n > 0
    st0, n0 = ws((4, 0, 80, 64, 1, 128))
    assert st0 == 0 and n0 == 0
    assert ws((1, 10, 4, 16, 3, 16))[0] == 1    # H % G != 0
    assert ws((1, 10, 4, 16, 1, 16), chunk=0)[0] == 1
    assert ws((1, 10, 4, 16, 1, 16), chunk=512)[0] == 2
    assert ws((1, 10, 4, 512, 1, 16))[0] == 2
    assert ws((1, 10, 4, 16, 1, 16), dtype=7)[0] == 1
    assert lib.ssd_fwd_workspace_bytes(ctypes.byref(B.ShapeT(1, 1, 1, 1, 1, 1)), 0, 1, None) == 1


def test_plan_selects_path(lib):
    plan = B.fwd_plan(4, 8192, 80, 64, 1, 128, B.SSD_BF16, 256)
    assert plan["path"] == "tcgen05" and plan["kernels"] == 1
    assert B.fwd_plan(1, 65536, 80, 64, 1, 256, B.SSD_BF16, 256)["path"] == "tcgen05"
    assert B.fwd_plan(1, 256, 4, 16, 1, 16, B.SSD_F32, 64)["path"] == "simt"
    assert B.fwd_plan(4, 8192, 80, 64, 1, 128, B.SSD_F32, 256)["path"] == "simt"
    assert B.fwd_plan(4, 8192, 80, 64, 1, 128, B.SSD_BF16, 64)["path"] == "simt"
    assert B.fwd_plan(4, 8192, 80, 128, 1, 128, B.SSD_BF16, 256)["path"] == "simt"
    assert B.fwd_plan(4, 0, 80, 64, 1, 128, B.SSD_BF16, 256)["path"] == "none"


def fwd_call(shape, ptrs, chunk=64, ws_bytes=1 << 30, dtype=B.SSD_BF16):
    s = B.ShapeT(*shape)
    p = {k: ctypes.c_void_p(v) if v else None for k, v in ptrs.items()}
    return B.lib().ssd_fwd(ctypes.byref(s), dtype, p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["h0"],
                           chunk, p["y"], p["hf"], p["ws"], ws_bytes, None)


GOOD = dict(x=0x10000, dt=0x20000, A=0x30000, B=0x40000, C=0x50000, D=0x60000, h0=None, y=0x70000,
            hf=0x80000, ws=0x90000)


def test_fwd_rejects_before_launch(lib):
    shape = (2, 100, 4, 16, 2, 16)
    assert lib.ssd_fwd(None, 1, *([None] * 7), 64, None, None, None, 0, None) == 1
    for k in ("x", "dt", "A", "B", "C", "y"):
        assert fwd_call(shape, {**GOOD, k: None}) == 1, k
    for k in ("x", "dt", "A", "B", "C", "D", "y", "hf", "ws"):
        assert fwd_call(shape, {**GOOD, k: GOOD[k] + 4}) == 3, k
    assert fwd_call(shape, {**GOOD, "ws": None}) == 4
    assert fwd_call(shape, GOOD, ws_bytes=16) == 4
    assert fwd_call((2, 100, 4, 16, 3, 16), GOOD) == 1
    assert fwd_call((-1, 100, 4, 16, 1, 16), GOOD) == 1
    assert fwd_call((2, 100, 0, 16, 1, 16), GOOD) == 1
    assert fwd_call((2, 100, 4, 300, 1, 16), GOOD) == 2
    assert fwd_call((2, 100, 4, 16, 1, 300), GOOD) == 2
    assert fwd_call((70000, 100, 4, 16, 1, 16), GOOD) == 2
    assert fwd_call(shape, GOOD, chunk=0) == 1
    assert fwd_call(shape, GOOD, chunk=257) == 2
    assert fwd_call(shape, GOOD, dtype=3) == 1
    # batch == 0 is a valid empty problem: nothing to launch, nothing touched
    assert fwd_call((0, 100, 4, 16, 1, 16), {k: None for k in GOOD}) == 0


def static_call(shape, ptrs, chunk=64, dtype=B.SSD_BF16):
    s = B.ShapeT(*shape)
    p = {k: ctypes.c_void_p(v) if v else None for k, v in ptrs.items()}
    return B.lib().ssd_fwd_static_scratch(ctypes.byref(s), dtype, p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"],
                                          p["h0"], chunk, p["y"], p["hf"], None)


def test_static_scratch_rejects_like_fwd(lib):
    """The allocation-free entry point applies ssd_fwd's argument rules, before any launch."""
    shape = (2, 100, 4, 16, 2, 16)
    assert lib.ssd_fwd_static_scratch(None, 1, *([None] * 7), 64, None, None, None) == 1
    for k in ("x", "dt", "A", "B", "C", "y"):
        assert static_call(shape, {**GOOD, k: None}) == 1, k
    for k in ("x", "dt", "A", "B", "C", "D", "y", "hf"):
        assert static_call(shape, {**GOOD, k: GOOD[k] + 4}) == 3, k
    assert static_call((2, 100, 4, 16, 3, 16), GOOD) == 1
    assert static_call((-1, 100, 4, 16, 1, 16), GOOD) == 1
    assert static_call((2, 100, 4, 300, 1, 16), GOOD) == 2
    assert static_call((70000, 100, 4, 16, 1, 16), GOOD) == 2
    assert static_call(shape, GOOD, chunk=0) == 1
    assert static_call(shape, GOOD, chunk=257) == 2
    assert static_call(shape, GOOD, dtype=3) == 1
    assert static_call((0, 100, 4, 16, 1, 16), {k: None for k in GOOD}) == 0
    # intermediates larger than the built-in array are refused (SSD_ERR_WORKSPACE)
    assert static_call((64, 65536, 80, 64, 1, 128), GOOD, chunk=256) == 4


def test_status_and_wait_limit_args(lib):
    assert lib.ssd_set_wait_limit_us(-1) == 1
    assert lib.ssd_set_wait_limit_us(2000001) == 1
    assert lib.ssd_set_wait_limit_us(0) == 0
    assert lib.ssd_fwd_status(None, 1, 64, None, None) == 1
    assert lib.ssd_fwd_status(ctypes.byref(B.ShapeT(1, 10, 4, 16, 3, 16)), 1, 64, None, None) == 1
    assert lib.ssd_fwd_status(ctypes.byref(B.ShapeT(1, 10, 4, 16, 1, 16)), 1, 0, None, None) == 1


BWD_GOOD = dict(x=0x10000, dt=0x20000, A=0x30000, B=0x40000, C=0x50000, D=0x60000, h0=None, dy=0x70000,
                dhf=None, dx=0x80000, ddt=0x90000, dA=0xa0000, dB=0xb0000, dC=0xc0000, dD=0xd0000, dh0=None,
                ws=0xe0000)


def bwd_call(shape, ptrs, chunk=64, ws_bytes=1 << 34, dtype=B.SSD_BF16):
    s = B.ShapeT(*shape)
    p = {k: ctypes.c_void_p(v) if v else None for k, v in ptrs.items()}
    return B.lib().ssd_bwd(ctypes.byref(s), dtype, p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["h0"], chunk,
                           p["dy"], p["dhf"], p["dx"], p["ddt"], p["dA"], p["dB"], p["dC"], p["dD"], p["dh0"],
                           p["ws"], ws_bytes, None)


def test_bwd_workspace_bytes(lib):
    out = ctypes.c_size_t(0)
    shp = B.ShapeT(4, 8192, 80, 64, 1, 128)
    assert lib.ssd_bwd_workspace_bytes(ctypes.byref(shp), B.SSD_BF16, 256, ctypes.byref(out)) == 0
    # recomputed entering states and their gradients, [B,H,nc,P,N] fp32 each, dominate
    assert out.value >= 2 * 4 * 80 * 32 * 64 * 128 * 4
    assert lib.ssd_bwd_workspace_bytes(ctypes.byref(B.ShapeT(4, 0, 80, 64, 1, 128)), 1, 256, ctypes.byref(out)) == 0
    assert out.value == 0
    assert lib.ssd_bwd_workspace_bytes(ctypes.byref(shp), 1, 256, None) == 1
    assert lib.ssd_bwd_workspace_bytes(ctypes.byref(B.ShapeT(1, 10, 4, 16, 3, 16)), 1, 64, ctypes.byref(out)) == 1


def test_block_ops_reject_before_launch(lib):
    shp = B.ShapeT(2, 100, 4, 16, 1, 8)
    vp = ctypes.c_void_p
    good = dict(xbc=0x10000, dtr=0x20000, w=0x30000, b=None, dtb=None, x=0x40000, Bm=0x50000, Cm=0x60000, dt=0x70000)

    def conv(p=good, stride=96, dstride=100, width=4, shape=shp, dtype=B.SSD_BF16):
        q = {k: vp(v) if v else None for k, v in p.items()}
        return lib.ssd_conv_split(ctypes.byref(shape), dtype, q["xbc"], stride, q["dtr"], dstride, q["w"], q["b"],
                                  width, q["dtb"], q["x"], q["Bm"], q["Cm"], q["dt"], None)
    for k in ("xbc", "dtr", "w", "x", "Bm", "Cm", "dt"):
        assert conv({**good, k: None}) == 1, k
    assert conv(width=0) == 1 and conv(width=5) == 1
    assert conv(stride=79) == 1        # < H*P + 2*G*N = 80
    assert conv(stride=97) == 2        # odd row stride
    assert conv(dstride=3) == 1        # < H
    assert conv({**good, "xbc": 0x10002}) == 3 and conv({**good, "x": 0x40004}) == 3
    assert conv(shape=B.ShapeT(2, 100, 3, 5, 1, 8)) == 2  # H*P odd

    def norm(rows=10, dim=256, ng=4, y=0x10000, z=0x20000, zs=256, w=0x30000, eps=1e-5, out=0x40000):
        return lib.ssd_gated_rmsnorm(rows, dim, ng, B.SSD_BF16, vp(y) if y else None, vp(z) if z else None, zs,
                                     vp(w) if w else None, ctypes.c_float(eps), vp(out) if out else None, None)
    assert norm(y=None) == 1 and norm(w=None) == 1 and norm(out=None) == 1
    assert norm(dim=250, ng=5) == 2          # group of 50 channels
    assert norm(dim=256, ng=3) == 1          # groups do not divide dim
    assert norm(dim=8256, ng=1, zs=8256) == 2  # wider than the kernel's row
    assert norm(zs=128) == 1 and norm(eps=-1.0) == 1
    assert norm(z=0x20002) == 3 and norm(y=0x10004) == 3
    assert norm(zs=257) == 2                 # odd z row stride
    assert norm(rows=0, y=None, z=None, w=None, out=None) == 0


def test_bwd_plan_selects_path(lib):
    def plan(shape, dtype):
        out = B.PlanT()
        st = lib.ssd_bwd_plan(ctypes.byref(B.ShapeT(*shape)), dtype, 256, ctypes.byref(out))
        return st, out.path, out.kernels
    assert plan((4, 8192, 80, 64, 1, 128), B.SSD_BF16) == (0, 3, 11)   # tensor cores
    assert plan((4, 8192, 80, 64, 1, 128), B.SSD_F32) == (0, 1, 11)    # fp32 inputs: CUDA cores
    assert plan((1, 90, 2, 200, 1, 40), B.SSD_BF16) == (0, 1, 11)     # no compiled (P, N) instance
    assert plan((1, 0, 2, 64, 1, 128), B.SSD_BF16)[:2] == (0, 0)
    assert lib.ssd_bwd_plan(ctypes.byref(B.ShapeT(1, 1, 1, 1, 1, 1)), 0, 1, None) == 1


def test_bwd_rejects_before_launch(lib):
    shape = (2, 100, 4, 16, 2, 16)
    for k in ("x", "dt", "A", "B", "C", "dy", "dx", "ddt", "dA", "dB", "dC"):
        assert bwd_call(shape, {**BWD_GOOD, k: None}) == 1, k
    for k in ("x", "dt", "A", "B", "C", "D", "dy", "dx", "ddt", "dA", "dB", "dC", "dD", "ws"):
        assert bwd_call(shape, {**BWD_GOOD, k: BWD_GOOD[k] + 4}) == 3, k
    assert bwd_call(shape, {**BWD_GOOD, "h0": 0xf0004}) == 3
    assert bwd_call(shape, {**BWD_GOOD, "dhf": 0xf0008}) == 3
    assert bwd_call(shape, {**BWD_GOOD, "dh0": 0xf000c}) == 3
    assert bwd_call(shape, {**BWD_GOOD, "ws": None}) == 4
    assert bwd_call(shape, BWD_GOOD, ws_bytes=16) == 4
    assert bwd_call((2, 100, 4, 16, 3, 16), BWD_GOOD) == 1
    assert bwd_call((2, 100, 4, 300, 1, 16), BWD_GOOD) == 2
    assert bwd_call(shape, BWD_GOOD, chunk=0) == 1
    assert bwd_call(shape, BWD_GOOD, chunk=257) == 2
    assert bwd_call(shape, BWD_GOOD, dtype=3) == 1


def test_verify_and_select_reject_before_launch(lib):
    s = B.ShapeT(2, 8, 4, 16, 2, 16)
    v = lambda **kw: lib.ssd_verify(ctypes.byref(kw.get("shape", s)), 1, *[ctypes.c_void_p(a) if a else None for a in kw.get(
        "p", [0x1000] * 7)], kw.get("K", 8), ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000), None)
    assert v(K=7) == 1                       # seqlen != K
    assert v(K=0, shape=B.ShapeT(2, 0, 4, 16, 2, 16)) == 1
    assert v(K=65, shape=B.ShapeT(2, 65, 4, 16, 2, 16)) == 2
    assert v(shape=B.ShapeT(2, 8, 4, 16, 2, 18)) == 2   # dstate % 4
    assert v(p=[0x1000, None, 0x1000, 0x1000, 0x1000, 0x1000, None]) == 1
    assert v(p=[0x1008] + [0x1000] * 6) == 3
    sel = lambda K=8, acc=0x4000, shape=s: lib.ssd_select_state(ctypes.byref(shape), K, ctypes.c_void_p(0x1000),
                                                                 ctypes.c_void_p(0x2000), ctypes.c_void_p(acc) if acc else None,
                                                                 ctypes.c_void_p(0x3000), None)
    assert sel(K=0) == 1
    assert sel(acc=None) == 1
    assert sel(acc=0x4004) == 3
    assert sel(shape=B.ShapeT(2, 8, 4, 16, 2, 6)) == 2


def test_advance_and_decode_reject_before_launch(lib):
    s = B.ShapeT(2, 8, 4, 16, 2, 16)
    vp = lambda a: ctypes.c_void_p(a) if a else None

    def adv(shape=s, K=8, h0=0x1000, acc=0x4000, keep=0x100000, x=0x2000):
        return lib.ssd_advance_state(ctypes.byref(shape), 1, vp(h0), vp(x), vp(0x3000), vp(0x3100), vp(0x3200), K,
                                     vp(acc), vp(keep), None)

    assert adv(K=7) == 1                                   # seqlen != K
    assert adv(K=65, shape=B.ShapeT(2, 65, 4, 16, 2, 16)) == 2
    assert adv(shape=B.ShapeT(2, 8, 4, 16, 2, 18)) == 2     # dstate % 4
    assert adv(acc=None) == 1
    assert adv(x=0x2008) == 3
    assert adv(keep=0x1010) == 1                           # overlaps h0 without being it
    assert adv(shape=B.ShapeT(0, 8, 4, 16, 2, 16), h0=None, acc=None, keep=None) == 0   # empty batch

    def dec(shape=B.ShapeT(2, 1, 4, 16, 2, 16), state=0x1000, y=0x5000, D=None):
        return lib.ssd_decode_step(ctypes.byref(shape), 1, vp(state), vp(0x2000), vp(0x3000), vp(0x3100),
                                   vp(0x3200), vp(0x3300), vp(D), vp(y), None)

    assert dec(shape=B.ShapeT(2, 2, 4, 16, 2, 16)) == 1   # seqlen must be 1
    assert dec(shape=B.ShapeT(2, 1, 4, 16, 2, 6)) == 2
    assert dec(state=None) == 1
    assert dec(y=0x5002) == 3
    assert dec(D=0x6004) == 3


def test_context_parallel_steps_reject_before_launch(lib):
    vp = lambda a: ctypes.c_void_p(a) if a else None
    s = B.ShapeT(2, 300, 4, 64, 1, 128)

    def decay(shape=s, dtype=1, dt=0x1000, A=0x2000, bd=0x3000, tot=0x4000):
        return lib.ssd_cp_decay(ctypes.byref(shape), dtype, vp(dt), vp(A), vp(bd), vp(tot), None)

    assert decay(dtype=7) == 1
    assert decay(tot=None) == 1
    assert decay(dt=None) == 1                                   # L > 0 needs dt and block sums
    assert decay(A=0x2004) == 3
    assert decay(shape=B.ShapeT(2, 300, 4, 64, 3, 128)) == 1    # heads not a multiple of groups
    assert decay(shape=B.ShapeT(0, 300, 4, 64, 1, 128), dt=None, A=None, bd=None, tot=None) == 0

    def combine(shape=s, R=4, rank=1, states=0x1000, totals=0x2000, s_in=0x3000, hf=0x4000):
        return lib.ssd_cp_combine(ctypes.byref(shape), R, rank, vp(states), vp(totals), vp(s_in), vp(hf), None)

    assert combine(R=0) == 1 and combine(rank=4) == 1 and combine(rank=-1) == 1
    assert combine(R=70000, rank=0) == 2
    assert combine(s_in=None) == 1
    assert combine(hf=0x4008) == 3
    assert combine(shape=B.ShapeT(2, 300, 4, 1, 1, 3)) == 2       # headdim * dstate % 4

    def correct(shape=s, dt=0x1000, y=0x5000, status=None):
        return lib.ssd_cp_correct(ctypes.byref(shape), 1, vp(dt), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x6000),
                                  vp(y), vp(status), None)

    assert correct(dt=None) == 1
    assert correct(y=0x5008) == 3
    assert correct(status=0x7002) == 3                           # the status word is an int32
    assert correct(shape=B.ShapeT(2, 0, 4, 64, 1, 128), dt=None) == 0   # empty segment: nothing to do


def test_binding_requires_cuda_tensors():
    import torch

    x = torch.zeros(1, 4, 2, 8)
    with pytest.raises(ValueError):
        B.ssd_fwd(x, torch.zeros(1, 4, 2), torch.zeros(2), torch.zeros(1, 4, 1, 8), torch.zeros(1, 4, 1, 8), chunk=4)
    # every other entry point refuses host tensors too: there is no CPU path
    with pytest.raises(ValueError):
        B.ssd_bwd(x, torch.zeros(1, 4, 2), torch.zeros(2), torch.zeros(1, 4, 1, 8), torch.zeros(1, 4, 1, 8), None,
                  None, torch.zeros_like(x), chunk=4)
    row = torch.zeros(1, 4, 2 * 16 + 2 * 8 + 2)
    with pytest.raises(ValueError):
        B.ssd_conv_split(row[..., 16:48], row[..., 48:50], torch.zeros(32, 4), None, None, nheads=2, headdim=8,
                         ngroups=1, dstate=8)
    with pytest.raises(ValueError):
        B.ssd_gated_rmsnorm(torch.zeros(3, 64), torch.zeros(3, 64), torch.ones(64), ngroups=1)
    with pytest.raises(ValueError):
        B.ssd_verify(torch.zeros(1, 2, 8, 8), torch.zeros(1, 2, 2, 8), torch.zeros(1, 2, 2), torch.zeros(2),
                     torch.zeros(1, 2, 1, 8), torch.zeros(1, 2, 1, 8))


def test_mixer_config_sizes():
    """The input projection's row holds z, x, B, C (H*P, H*P, G*N, G*N) and dt_raw (H)."""
    from state_space_sequence_chunked_b200 import mamba2

    cfg = mamba2.MixerConfig(d_model=2560, nheads=80, headdim=64, ngroups=1, dstate=128)
    assert cfg.d_inner == 5120 and cfg.d_in_proj == 2 * 5120 + 2 * 128 + 80
