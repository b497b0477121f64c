"""ctypes binding of libssd (include/ssd.h): argument marshalling only.

Every step of the computation runs in the CUDA library. Torch tensors supply
device memory and the current CUDA stream. If the library is missing the calls
raise; there is no other implementation behind them.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd.so")

SSD_F32, SSD_BF16 = 0, 1
STATUS = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_ALIGNMENT",
          4: "SSD_ERR_WORKSPACE", 5: "SSD_ERR_CUDA", 6: "SSD_ERR_TIMEOUT"}


class SSDError(RuntimeError):
    def __init__(self, status: int, fn: str, text: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({text})")
        self.status = status
        self.name = STATUS.get(status, str(status))


class ShapeT(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate")]


class PlanT(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("kernels", ctypes.c_int32), ("workspace_bytes", ctypes.c_size_t)]


PATHS = {0: "none", 1: "simt", 2: "tcgen05", 3: "mma"}

_lib = None
_vp, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "ssd_strerror": ([ctypes.c_int], ctypes.c_char_p),
    "ssd_fwd_workspace_bytes": ([ctypes.POINTER(ShapeT), ctypes.c_int, _i64, ctypes.POINTER(_sz)], ctypes.c_int),
    "ssd_fwd_plan": ([ctypes.POINTER(ShapeT), ctypes.c_int, _i64, ctypes.POINTER(PlanT)], ctypes.c_int),
    "ssd_fwd": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 7 + [_i64, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "ssd_fwd_static_scratch": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 7 + [_i64, _vp, _vp, _vp], ctypes.c_int),
    "ssd_fwd_status": ([ctypes.POINTER(ShapeT), ctypes.c_int, _i64, _vp, _vp], ctypes.c_int),
    "ssd_set_wait_limit_us": ([ctypes.c_int32], ctypes.c_int),
    "ssd_verify": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 7 + [_i64, _vp, _vp, _vp], ctypes.c_int),
    "ssd_select_state": ([ctypes.POINTER(ShapeT), _i64] + [_vp] * 5, ctypes.c_int),
    "ssd_advance_state": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 5 + [_i64, _vp, _vp, _vp], ctypes.c_int),
    "ssd_decode_step": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 9, ctypes.c_int),
    "ssd_cp_decay": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 5, ctypes.c_int),
    "ssd_cp_combine": ([ctypes.POINTER(ShapeT), _i64, _i64] + [_vp] * 5, ctypes.c_int),
    "ssd_cp_correct": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 8, ctypes.c_int),
    "ssd_bwd_workspace_bytes": ([ctypes.POINTER(ShapeT), ctypes.c_int, _i64, ctypes.POINTER(_sz)], ctypes.c_int),
    "ssd_bwd_plan": ([ctypes.POINTER(ShapeT), ctypes.c_int, _i64, ctypes.POINTER(PlanT)], ctypes.c_int),
    "ssd_conv_split": ([ctypes.POINTER(ShapeT), ctypes.c_int, _vp, _i64, _vp, _i64, _vp, _vp, _i64] + [_vp] * 6,
                       ctypes.c_int),
    "ssd_gated_rmsnorm": ([_i64, _i64, _i64, ctypes.c_int, _vp, _vp, _i64, _vp, ctypes.c_float, _vp, _vp],
                          ctypes.c_int),
    "ssd_bwd": ([ctypes.POINTER(ShapeT), ctypes.c_int] + [_vp] * 7 + [_i64] + [_vp] * 9 + [_vp, _sz, _vp],
                ctypes.c_int),
}

CP_BLOCK = 128  # SSD_CP_BLOCK: tokens per decay block


def lib():
    """Load libssd.so (built in-tree by state_space_sequence_chunked_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libssd.so is not built ({LIB_PATH}); run state_space_sequence_chunked_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes, f.restype = args, res
        _lib = L
    return _lib


def _check(status: int, fn: str):
    if status != 0:
        raise SSDError(status, fn, lib().ssd_strerror(status).decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SSD_F32
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("libssd takes CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("libssd takes contiguous tensors")
        dev = t.device if dev is None else dev
    return dev


def _dev_rows(dev, *ts):
    """Row views (a column slice of wider rows): CUDA, on `dev`, unit column stride, rows at one
    stride (the C calls take that stride)."""
    for t in ts:
        if not t.is_cuda or (dev is not None and t.device != dev):
            raise ValueError("libssd takes CUDA tensors on one device")
        if t.stride(-1) != 1 or any(t.stride(i) != t.stride(i + 1) * t.shape[i + 1] for i in range(t.dim() - 2)):
            raise ValueError("row views need unit column stride and evenly spaced rows")


def _stream(dev, stream):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream)


def fwd_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate, dtype_code, chunk) -> int:
    shape = ShapeT(batch, seqlen, nheads, headdim, ngroups, dstate)
    out = _sz(0)
    _check(lib().ssd_fwd_workspace_bytes(ctypes.byref(shape), dtype_code, chunk, ctypes.byref(out)),
           "ssd_fwd_workspace_bytes")
    return out.value


def fwd_plan(batch, seqlen, nheads, headdim, ngroups, dstate, dtype_code, chunk) -> dict:
    """{'path': 'simt'|'tcgen05'|'none', 'kernels': launches per call, 'workspace_bytes': int}."""
    shape = ShapeT(batch, seqlen, nheads, headdim, ngroups, dstate)
    out = PlanT()
    _check(lib().ssd_fwd_plan(ctypes.byref(shape), dtype_code, chunk, ctypes.byref(out)), "ssd_fwd_plan")
    return {"path": PATHS.get(out.path, str(out.path)), "kernels": out.kernels,
            "workspace_bytes": out.workspace_bytes}


def ssd_fwd(x, dt, A, B, C, D=None, h0=None, *, chunk: int, y=None, h_final=None,
            return_final_state: bool = True, workspace=None, stream=None, check: bool = False):
    """y, h_final = ssd_fwd(x [B,L,H,P], dt [B,L,H], A [H] f32, B/C [B,L,G,N], D [H] f32?, h0 [B,H,P,N] f32?).

    check=True synchronizes the stream after the launch and raises SSDError (SSD_ERR_TIMEOUT)
    if a bounded device-side wait ran out, which leaves y and h_final incomplete."""
    dev = _dev(x, dt, A, B, C, D, h0, y, h_final, workspace)
    Bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    code = _dtype_code(x)
    shape = ShapeT(Bsz, L, H, P, G, N)
    if y is None:
        y = torch.empty_like(x)
    if h_final is None and return_final_state:
        h_final = torch.empty((Bsz, H, P, N), dtype=torch.float32, device=dev)
    need = fwd_workspace_bytes(Bsz, L, H, P, G, N, code, chunk)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().ssd_fwd(ctypes.byref(shape), code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                       _ptr(h0), chunk, _ptr(y), _ptr(h_final), _ptr(workspace), ws_bytes,
                       _stream(dev, stream))
    _check(st, "ssd_fwd")
    if check:
        _check(lib().ssd_fwd_status(ctypes.byref(shape), code, chunk, _ptr(workspace), _stream(dev, stream)),
               "ssd_fwd")
    return y, h_final


def fwd_status(shape_args, dtype_code, chunk, workspace, stream=None) -> int:
    """Raw ssd_fwd_status code for the last ssd_fwd on `workspace` (synchronizes the stream).

    shape_args = (batch, seqlen, nheads, headdim, ngroups, dstate)."""
    shape = ShapeT(*shape_args)
    dev = workspace.device if workspace is not None else torch.device("cuda", torch.cuda.current_device())
    return lib().ssd_fwd_status(ctypes.byref(shape), dtype_code, chunk, _ptr(workspace), _stream(dev, stream))


def set_wait_limit_us(us: int):
    """Test hook: limit of every bounded device-side wait in later launches (0: the built-in 2 s)."""
    _check(lib().ssd_set_wait_limit_us(int(us)), "ssd_set_wait_limit_us")


def ssd_verify(h0, x, dt, A, B, C, D=None, *, states_out=None, y=None, return_states: bool = True,
               stream=None):
    """y [B,K,H,P], states_out [B,K,H,P,N] = ssd_verify(h0 [B,H,P,N] f32, x [B,K,H,P], dt, A, B, C, D).

    return_states=False (and no states_out given) writes y only; states_out is then None."""
    dev = _dev(h0, x, dt, A, B, C, D, states_out, y)
    Bsz, K, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    shape = ShapeT(Bsz, K, H, P, G, N)
    if y is None:
        y = torch.empty_like(x)
    if states_out is None and return_states:
        states_out = torch.empty((Bsz, K, H, P, N), dtype=torch.float32, device=dev)
    st = lib().ssd_verify(ctypes.byref(shape), _dtype_code(x), _ptr(h0), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                          _ptr(C), _ptr(D), K, _ptr(states_out), _ptr(y), _stream(dev, stream))
    _check(st, "ssd_verify")
    return y, states_out


def ssd_select_state(h0, states_out, accepted, *, h_keep=None, stream=None):
    """h_keep[b] = h0[b] if accepted[b] == 0 else states_out[b, accepted[b] - 1] (bit-exact)."""
    dev = _dev(h0, states_out, accepted, h_keep)
    Bsz, K, H, P, N = states_out.shape
    if accepted.dtype != torch.int32:
        raise TypeError("accepted must be int32")
    shape = ShapeT(Bsz, K, H, P, 1, N)
    if h_keep is None:
        h_keep = torch.empty_like(h0)
    st = lib().ssd_select_state(ctypes.byref(shape), K, _ptr(h0), _ptr(states_out), _ptr(accepted),
                                _ptr(h_keep), _stream(dev, stream))
    _check(st, "ssd_select_state")
    return h_keep


def ssd_advance_state(h0, x, dt, A, B, accepted, *, h_keep=None, stream=None):
    """h_keep[b] = state after the first accepted[b] draft tokens from h0[b] (h_keep may be h0: in place)."""
    dev = _dev(h0, x, dt, A, B, accepted, h_keep)
    if accepted.dtype != torch.int32:
        raise TypeError("accepted must be int32")
    Bsz, K, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    shape = ShapeT(Bsz, K, H, P, G, N)
    if h_keep is None:
        h_keep = torch.empty_like(h0)
    st = lib().ssd_advance_state(ctypes.byref(shape), _dtype_code(x), _ptr(h0), _ptr(x), _ptr(dt), _ptr(A),
                                 _ptr(B), K, _ptr(accepted), _ptr(h_keep), _stream(dev, stream))
    _check(st, "ssd_advance_state")
    return h_keep


def ssd_decode_step(state, x, dt, A, B, C, D=None, *, y=None, stream=None):
    """One token in place: state [B,H,P,N] f32 <- exp(dt A) state + dt x B^T; returns y [B,H,P] = state C + D x.
    x [B,H,P], dt [B,H], B/C [B,G,N]."""
    dev = _dev(state, x, dt, A, B, C, D, y)
    Bsz, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    shape = ShapeT(Bsz, 1, H, P, G, N)
    if y is None:
        y = torch.empty_like(x)
    st = lib().ssd_decode_step(ctypes.byref(shape), _dtype_code(x), _ptr(state), _ptr(x), _ptr(dt), _ptr(A),
                               _ptr(B), _ptr(C), _ptr(D), _ptr(y), _stream(dev, stream))
    _check(st, "ssd_decode_step")
    return y


def ssd_cp_decay(dt, A, *, block_decay=None, total=None, stream=None):
    """block_decay [B,H,ceil(L/128)], total [B,H] = sums of dt*A over a segment's blocks and over the segment."""
    dev = _dev(dt, A, block_decay, total)
    Bsz, L, H = dt.shape
    nblk = (L + CP_BLOCK - 1) // CP_BLOCK
    if block_decay is None:
        block_decay = torch.empty((Bsz, H, max(nblk, 1)), dtype=torch.float32, device=dev)
    if total is None:
        total = torch.empty((Bsz, H), dtype=torch.float32, device=dev)
    shape = ShapeT(Bsz, L, H, 1, 1, 1)
    st = lib().ssd_cp_decay(ctypes.byref(shape), _dtype_code(dt), _ptr(dt), _ptr(A), _ptr(block_decay), _ptr(total),
                            _stream(dev, stream))
    _check(st, "ssd_cp_decay")
    return block_decay, total


def ssd_cp_combine(states, totals, rank, *, s_in=None, h_final=None, want_final=True, stream=None):
    """s_in (state entering segment `rank`), h_final (its true end state) from the gathered
    states [R,B,H,P,N] and totals [R,B,H]."""
    dev = _dev(states, totals, s_in, h_final)
    R, Bsz, H, P, N = states.shape
    if s_in is None:
        s_in = torch.empty((Bsz, H, P, N), dtype=torch.float32, device=dev)
    if h_final is None and want_final:
        h_final = torch.empty((Bsz, H, P, N), dtype=torch.float32, device=dev)
    shape = ShapeT(Bsz, 0, H, P, 1, N)
    st = lib().ssd_cp_combine(ctypes.byref(shape), R, rank, _ptr(states), _ptr(totals), _ptr(s_in), _ptr(h_final),
                              _stream(dev, stream))
    _check(st, "ssd_cp_combine")
    return s_in, h_final


def ssd_cp_correct(dt, A, C, block_decay, s_in, y, *, status=None, stream=None):
    """y += exp(cumulative dt*A from the segment start) * C S_in^T, in place; returns y.
    status: optional int32 device tensor (one element, zeroed by the caller); bit 0 is set if a
    bounded device-side wait ran out."""
    dev = _dev(dt, A, C, block_decay, s_in, y, status)
    Bsz, L, H, P = y.shape
    G, N = C.shape[2], C.shape[3]
    shape = ShapeT(Bsz, L, H, P, G, N)
    st = lib().ssd_cp_correct(ctypes.byref(shape), _dtype_code(y), _ptr(dt), _ptr(A), _ptr(C), _ptr(block_decay),
                              _ptr(s_in), _ptr(y), _ptr(status), _stream(dev, stream))
    _check(st, "ssd_cp_correct")
    return y


def bwd_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate, dtype_code, chunk) -> int:
    shape = ShapeT(batch, seqlen, nheads, headdim, ngroups, dstate)
    out = _sz(0)
    _check(lib().ssd_bwd_workspace_bytes(ctypes.byref(shape), dtype_code, chunk, ctypes.byref(out)),
           "ssd_bwd_workspace_bytes")
    return out.value


def bwd_plan(batch, seqlen, nheads, headdim, ngroups, dstate, dtype_code, chunk) -> dict:
    """{'path': 'simt'|'mma'|'none', 'kernels': launches per call, 'workspace_bytes': int}."""
    shape = ShapeT(batch, seqlen, nheads, headdim, ngroups, dstate)
    out = PlanT()
    _check(lib().ssd_bwd_plan(ctypes.byref(shape), dtype_code, chunk, ctypes.byref(out)), "ssd_bwd_plan")
    return {"path": PATHS.get(out.path, str(out.path)), "kernels": out.kernels,
            "workspace_bytes": out.workspace_bytes}


def ssd_bwd(x, dt, A, B, C, D, h0, dy, dh_final=None, *, chunk: int, want_dD: bool = True,
            want_dh0: bool = True, out=None, workspace=None, stream=None):
    """Gradients of sum(dy * y) + sum(dh_final * h_final) through ssd_fwd.

    Returns a dict dx, ddt, dA, dB, dC, dD (None unless want_dD), dh0 (None unless want_dh0);
    `out` may supply any of those tensors to write into."""
    dev = _dev(x, dt, A, B, C, D, h0, dy, dh_final, workspace)
    Bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    code = _dtype_code(x)
    shape = ShapeT(Bsz, L, H, P, G, N)
    o = dict(out or {})
    o.setdefault("dx", torch.empty_like(x))
    o.setdefault("ddt", torch.empty_like(dt))
    o.setdefault("dA", torch.empty(H, dtype=torch.float32, device=dev))
    o.setdefault("dB", torch.empty_like(B))
    o.setdefault("dC", torch.empty_like(C))
    o.setdefault("dD", torch.empty(H, dtype=torch.float32, device=dev) if want_dD else None)
    o.setdefault("dh0", torch.empty((Bsz, H, P, N), dtype=torch.float32, device=dev) if want_dh0 else None)
    need = bwd_workspace_bytes(Bsz, L, H, P, G, N, code, chunk)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().ssd_bwd(ctypes.byref(shape), code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                       _ptr(h0), chunk, _ptr(dy), _ptr(dh_final), _ptr(o["dx"]), _ptr(o["ddt"]), _ptr(o["dA"]),
                       _ptr(o["dB"]), _ptr(o["dC"]), _ptr(o["dD"]), _ptr(o["dh0"]), _ptr(workspace), ws_bytes,
                       _stream(dev, stream))
    _check(st, "ssd_bwd")
    return o


def ssd_conv_split(xbc, dt_raw, conv_w, conv_b, dt_bias, *, nheads, headdim, ngroups, dstate, out=None,
                   stream=None):
    """x [B,L,H,P], B, C [B,L,G,N], dt [B,L,H] from the convolution + SiLU of the x B C channels and
    softplus(dt_raw + dt_bias). xbc and dt_raw are [B, L, *] views with unit column stride (the
    input projection's columns can be passed in place)."""
    dev = _dev(conv_w, conv_b, dt_bias)
    _dev_rows(dev, xbc, dt_raw)
    Bsz, L = xbc.shape[0], xbc.shape[1]
    H, P, G, N = nheads, headdim, ngroups, dstate
    assert xbc.stride(2) == 1 and dt_raw.stride(2) == 1 and xbc.stride(0) == L * xbc.stride(1)
    assert dt_raw.stride(0) == L * dt_raw.stride(1)
    code = _dtype_code(xbc)
    o = dict(out or {})
    o.setdefault("x", torch.empty(Bsz, L, H, P, dtype=xbc.dtype, device=dev))
    o.setdefault("B", torch.empty(Bsz, L, G, N, dtype=xbc.dtype, device=dev))
    o.setdefault("C", torch.empty(Bsz, L, G, N, dtype=xbc.dtype, device=dev))
    o.setdefault("dt", torch.empty(Bsz, L, H, dtype=xbc.dtype, device=dev))
    shape = ShapeT(Bsz, L, H, P, G, N)
    st = lib().ssd_conv_split(ctypes.byref(shape), code, _ptr(xbc), xbc.stride(1), _ptr(dt_raw), dt_raw.stride(1),
                              _ptr(conv_w), _ptr(conv_b), conv_w.shape[1], _ptr(dt_bias), _ptr(o["x"]), _ptr(o["B"]),
                              _ptr(o["C"]), _ptr(o["dt"]), _stream(dev, stream))
    _check(st, "ssd_conv_split")
    return o


def ssd_gated_rmsnorm(y, z, weight, *, ngroups, eps=1e-5, out=None, stream=None):
    """out = weight * RMSNorm over `ngroups` groups of (y * silu(z)); y [..., dim] contiguous,
    z [..., dim] with unit column stride (a column slice of a wider row is fine)."""
    dev = _dev(y, weight, out)
    _dev_rows(dev, z)
    dim = y.shape[-1]
    rows = y.numel() // dim if dim else 0
    assert z.stride(-1) == 1
    zs = z.stride(-2) if z.dim() >= 2 else dim
    if out is None:
        out = torch.empty_like(y)
    st = lib().ssd_gated_rmsnorm(rows, dim, ngroups, _dtype_code(y), _ptr(y), _ptr(z), zs, _ptr(weight), float(eps),
                                 _ptr(out), _stream(dev, stream))
    _check(st, "ssd_gated_rmsnorm")
    return out

