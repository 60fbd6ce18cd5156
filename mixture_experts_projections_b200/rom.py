"""Python binding of librom.so (the C ABI in include/rom.h).

Argument marshalling only: every step of the RoM block runs in the CUDA
library. PyTorch supplies device memory and the current stream. The functions
keep the C names (rom_route, rom_dispatch, rom_expert_proj, rom_combine, ...);
``block_forward`` and ``inproj_forward`` chain them for one block.

Importing this module does not need a GPU; calling into the library does, and
a missing library raises at once (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librom.so")

ROM_OK, ROM_ERR_INVALID_ARG, ROM_ERR_UNSUPPORTED, ROM_ERR_WORKSPACE, ROM_ERR_CUDA, \
    ROM_ERR_TIMEOUT, ROM_ERR_ROUTING = range(7)
ROM_F32, ROM_BF16 = 0, 1
ROM_PROJ_CONV_GATE, ROM_PROJ_OUT, ROM_PROJ_INPROJ, ROM_PROJ_SLOTS, ROM_PROJ_CONV_GATE_SLOTS = \
    0, 1, 2, 3, 4
ROM_COMBINE_SUM, ROM_COMBINE_GATE, ROM_COMBINE_GATE_DENSE = 0, 1, 2
ROM_W_TILED = 0x100  # rom_expert_proj_dense: weights in the tile-major layout

# Every exported symbol of include/rom.h with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
SIGNATURES = {
    "rom_status_string": (ctypes.c_char_p, [_I]),
    "rom_version": (_I, []),
    "rom_workspace_size": (ctypes.c_size_t, [_L, _I]),
    "rom_route": (_I, [_P, _I, _L, _I, _P, _P, _I, _I, _I, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "rom_dispatch": (_I, [_P, _I, _L, _I, _I, _I, _P, _P, ctypes.c_size_t, _P, _P, _P, _P, _P]),
    "rom_expert_proj": (_I, [_I, _I, _P, _L, _I, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "rom_combine": (_I, [_I, _I, _P, _L, _I, _I, _P, _P, _P]),
    "rom_expert_proj_dense": (_I, [_I, _I, _P, _L, _I, _P, _I, _I, _I, _P, _P, _P, _P]),
    "rom_pack_expert_weights": (_I, [_I, _P, _I, _I, _I, _P, _P]),
    "rom_get_status": (_I, [_P, ctypes.POINTER(ctypes.c_int32)]),
    "rom_debug_wait_timeout": (_I, [ctypes.c_uint64, _P]),
    "rom_route_dispatch_noalloc": (_I, [_P, _I, _L, _I, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P,
                                        _P, _P, _P]),
    "rom_bwd_gather": (_I, [_P, _L, _I, _I, _P, _P, _P, _P]),
    "rom_bwd_dgrad_out": (_I, [_P, _L, _I, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "rom_bwd_gate": (_I, [_P, _P, _L, _I, _I, _P, _P, _P]),
    "rom_bwd_dgrad_in": (_I, [_P, _L, _I, _P, _P, _I, _I, _I, _P, _P, _P, _P]),
    "rom_route_bwd": (_I, [_L, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P]),
    "rom_route_probs": (_I, [_P, _I, _L, _I, _P, _P, _I, _P, _P]),
    "rom_route_wgrad": (_I, [_P, _I, _L, _I, _I, _P, _P, _P, _P]),
    "rom_bwd_wgrad": (_I, [_P, _I, _P, _I, _L, _I, _P, _I, _P, _P, _P]),
    "rom_ssm_core_workspace_size": (ctypes.c_size_t, [_L, _I, _I, _I, _I, _I]),
    "rom_ssm_core_routed_workspace_size": (ctypes.c_size_t, [_L, _I, _I, _I, _I, _I, _I, _I]),
    "rom_ssm_core_routed": (_I, [_P, _L, _I, _I, _P, _P, _I, _P, _I, _I, _I, _P, _P, _P, _P,
                                 _I, _I, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "rom_ssm_core": (_I, [_P, _L, _I, _I, _P, _P, _I, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                          ctypes.c_size_t, _P]),
}

_lib = None


class RomError(RuntimeError):
    pass


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librom.so (once) and declare the signatures of its entry points."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RomError(f"{path} is missing: build it with "
                           "`python -m mixture_experts_projections_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(code: int, what: str):
    if code != ROM_OK:
        msg = load_library().rom_status_string(code).decode()
        raise RomError(f"{what} failed: {msg} ({code})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ROM_BF16
    if t.dtype == torch.float32:
        return ROM_F32
    raise RomError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise RomError(f"{name} must be a contiguous CUDA tensor")


# ------------------------------------------------------------------ C entry points


def rom_workspace_size(T: int, E: int) -> int:
    return int(load_library().rom_workspace_size(T, E))


def rom_route(x, w_r, bias, k, renorm, topk_idx, topk_w, counts, ws, stream=None):
    for t, n in ((x, "x"), (w_r, "w_r"), (topk_idx, "topk_idx"), (topk_w, "topk_w")):
        _need(t, n)
    T, Dm = x.shape
    E = w_r.shape[1]
    _check(load_library().rom_route(
        _ptr(x), _dtype_code(x), T, Dm, _ptr(w_r), _ptr(bias), E, k, int(renorm),
        _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)), "rom_route")


def rom_dispatch(x, E, k, topk_idx, ws, offsets, sorted_slot, slot_pos, x_sorted, stream=None):
    T, Dm = x.shape
    _check(load_library().rom_dispatch(
        _ptr(x), _dtype_code(x), T, Dm, E, k, _ptr(topk_idx), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(offsets), _ptr(sorted_slot),
        _ptr(slot_pos), _ptr(x_sorted), _stream(stream)), "rom_dispatch")


def rom_expert_proj(proj, a_sorted, w0, w1, E, k, offsets, sorted_slot, topk_w, out,
                    stream=None):
    R, K = a_sorted.shape
    N = w0.shape[1]
    if not out.is_contiguous():
        raise RomError("out must be contiguous")
    _check(load_library().rom_expert_proj(
        proj, _dtype_code(a_sorted), _ptr(a_sorted), R, K, _ptr(w0), _ptr(w1), N, E, k,
        _ptr(offsets), _ptr(sorted_slot), _ptr(topk_w), _ptr(out), _stream(stream)),
        "rom_expert_proj")


def rom_expert_proj_dense(proj, x, w, E, k, topk_idx, topk_w, out, stream=None, tiled=False):
    """``tiled``: ``w`` holds the weights in the tile-major layout of
    pack_expert_weights (the same [E, N, K] shape and values, stored by tile)."""
    T, K = x.shape
    N = w.shape[1]
    _check(load_library().rom_expert_proj_dense(
        proj | (ROM_W_TILED if tiled else 0), _dtype_code(x), _ptr(x), T, K, _ptr(w), N, E, k,
        _ptr(topk_idx), _ptr(topk_w), _ptr(out), _stream(stream)), "rom_expert_proj_dense")


def pack_expert_weights(w, stream=None):
    """A copy of the expert weights w [E, N, K] (bf16) in the tile-major layout
    (each 128 x 64 weight tile one contiguous 16 KB block) that
    rom_expert_proj_dense reads with ``tiled=True``. Returned with the shape
    [E, N, K]; its elements are in tile order, not row order."""
    _need(w, "w")
    E, N, K = w.shape
    out = torch.empty_like(w)
    _check(load_library().rom_pack_expert_weights(_dtype_code(w), _ptr(w), E, N, K, _ptr(out),
                                                  _stream(stream)), "rom_pack_expert_weights")
    return out


# Few tokens: the routed projection reads x in token order and needs no
# dispatch (rom_expert_proj_dense).
DENSE_SMALL_MAX_TOKENS = 64


def rom_combine(mode, dtype_code, inp, T, k, N, slot_pos, out, stream=None):
    _check(load_library().rom_combine(mode, dtype_code, _ptr(inp), T, k, N, _ptr(slot_pos),
                                      _ptr(out), _stream(stream)), "rom_combine")


def rom_get_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(load_library().rom_get_status(_stream(stream), ctypes.byref(v)), "rom_get_status")
    return int(v.value)


def rom_debug_wait_timeout(limit_ns: int, stream=None):
    _check(load_library().rom_debug_wait_timeout(limit_ns, _stream(stream)),
           "rom_debug_wait_timeout")


def rom_route_dispatch_noalloc(x, w_r, bias, k, renorm, topk_idx, topk_w, counts, offsets,
                               sorted_slot, slot_pos, x_sorted, stream=None):
    """Routing + dispatch without a caller workspace (the library's own fixed
    device scratch; see include/rom.h)."""
    T, Dm = x.shape
    E = w_r.shape[1]
    _check(load_library().rom_route_dispatch_noalloc(
        _ptr(x), _dtype_code(x), T, Dm, _ptr(w_r), _ptr(bias), E, k, int(renorm),
        _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(offsets), _ptr(sorted_slot),
        _ptr(slot_pos), _ptr(x_sorted), _stream(stream)), "rom_route_dispatch_noalloc")


# ------------------------------------------------------------------ block helpers


def expert_weight_layout(w_pages: torch.Tensor) -> torch.Tensor:
    """[E, K, N] (the pages' x W notation) -> the library's [E, N, K] layout."""
    return w_pages.transpose(1, 2).contiguous()


class RoutingBuffers:
    """Device buffers of one routing + dispatch pass (allocated by torch)."""

    def __init__(self, T, Dm, E, k, dtype, device):
        R = T * k
        self.T, self.Dm, self.E, self.k = T, Dm, E, k
        self.topk_idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=device)
        self.counts = torch.empty((E,), dtype=torch.int32, device=device)
        nws = max(1, rom_workspace_size(T, E) // 4)
        self.ws = torch.empty((nws,), dtype=torch.int32, device=device)
        self.offsets = torch.empty((E + 1,), dtype=torch.int32, device=device)
        self.sorted_slot = torch.empty((max(R, 1),), dtype=torch.int32, device=device)
        self.slot_pos = torch.empty((max(R, 1),), dtype=torch.int32, device=device)
        self.x_sorted = torch.empty((max(R, 1), Dm), dtype=dtype, device=device)


def route_and_dispatch(x, w_r, bias, E, k, renorm, bufs=None, stream=None):
    T, Dm = x.shape
    if bufs is None:
        bufs = RoutingBuffers(T, Dm, E, k, x.dtype, x.device)
    rom_route(x, w_r, bias, k, renorm, bufs.topk_idx, bufs.topk_w, bufs.counts, bufs.ws, stream)
    rom_dispatch(x, E, k, bufs.topk_idx, bufs.ws, bufs.offsets, bufs.sorted_slot, bufs.slot_pos,
                 bufs.x_sorted, stream)
    return bufs


# ------------------------------------------------------------------ dense core


class CoreParams:
    """The dense core's parameters on the device in the library's layout
    (from float32 arrays in the pages' x W notation: conv_w [De, K],
    conv_b [De], w_x [De, R + 2N], w_dt [R, De], b_dt [De], a_log [De, N],
    d [De]; w_x and w_dt must hold bf16 values). With w_x [E, De, R + 2N]
    and w_dt [E, R, De] the x and dt projections are expertized
    (``self.E`` matrices, routed with the block's selection)."""

    def __init__(self, p, device="cuda"):
        import numpy as np
        De, K = p["conv_w"].shape
        wx_p = np.asarray(p["w_x"], np.float32)
        wdt_p = np.asarray(p["w_dt"], np.float32)
        self.routed = wx_p.ndim == 3
        if not self.routed:
            wx_p, wdt_p = wx_p[None], wdt_p[None]
        self.E = wx_p.shape[0]
        self.R = wdt_p.shape[1]
        self.De = De
        self.N = p["a_log"].shape[1]
        self.K = K
        self.Np = -(-(self.R + 2 * self.N) // 128) * 128

        def f32(a):
            return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)
        self.conv_w, self.conv_b = f32(p["conv_w"]), f32(p["conv_b"])
        self.b_dt, self.a_log, self.d = f32(p["b_dt"]), f32(p["a_log"]), f32(p["d"])
        wx = torch.zeros((self.E, self.Np, De), dtype=torch.float32)
        wx[:, :self.R + 2 * self.N] = torch.from_numpy(np.ascontiguousarray(wx_p)).transpose(1, 2)
        self.w_x = wx.to(torch.bfloat16).to(device).contiguous()  # exact: bf16 values
        self.w_dt = torch.from_numpy(np.ascontiguousarray(wdt_p)).transpose(1, 2).contiguous() \
            .to(torch.bfloat16).to(device)


def rom_ssm_core_workspace_size(T, De, seq_len, R, N, Np):
    return int(load_library().rom_ssm_core_workspace_size(T, De, seq_len, R, N, Np))


def rom_ssm_core(h, seq_len, core, y, ws, stream=None, routing=None):
    """Y = core(H) (h, y: float32 [T, De], may be the same tensor). An
    expertized core takes the block's RoutingBuffers as ``routing``."""
    T, De = h.shape
    common = (_ptr(h), T, De, seq_len, _ptr(core.conv_w), _ptr(core.conv_b), core.K,
              _ptr(core.w_x), core.R, core.N, core.Np, _ptr(core.w_dt), _ptr(core.b_dt),
              _ptr(core.a_log), _ptr(core.d))
    tail = (_ptr(y), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
            _stream(stream))
    if core.routed:
        _check(load_library().rom_ssm_core_routed(
            *common, core.E, routing.k, _ptr(routing.offsets), _ptr(routing.sorted_slot), *tail),
            "rom_ssm_core_routed")
    else:
        _check(load_library().rom_ssm_core(*common, *tail), "rom_ssm_core")


def core_workspace(T, De, seq_len, core, device, k=1):
    if core.routed:
        n = int(load_library().rom_ssm_core_routed_workspace_size(T, De, seq_len, core.R, core.N,
                                                                  core.Np, core.E, k))
    else:
        n = rom_ssm_core_workspace_size(T, De, seq_len, core.R, core.N, core.Np)
    return torch.empty((max(n, 256),), dtype=torch.uint8, device=device)


class BlockBuffers:
    """Intermediate and output buffers of one RoM block forward."""

    def __init__(self, T, Dm, De, E, k, dtype, device, core=None, seq_len=None, keep_uz=False):
        R = T * k
        self.routing = RoutingBuffers(T, Dm, E, k, dtype, device)
        self.h_sorted = torch.empty((max(R, 1), De), dtype=dtype, device=device)
        self.uz = (torch.empty((2, R, De), dtype=torch.float32, device=device)
                   if (k > 1 or core is not None or keep_uz) else None)
        self.core_ws = (core_workspace(T, De, seq_len or T, core, device, k)
                        if core is not None else None)
        self.hsum = (torch.empty((T, De), dtype=torch.float32, device=device)
                     if (core is not None and k > 1) else None)
        self.o_slots = (torch.empty((R, Dm), dtype=torch.float32, device=device)
                        if k > 1 else None)
        self.out = torch.empty((T, Dm), dtype=dtype, device=device)


def block_forward(x, w_r, bias, w_conv, w_gate, w_out, k, renorm=False, bufs=None, stream=None,
                  core=None, seq_len=None, keep_uz=False):
    """RoM block forward: route, dispatch, Conv+Gate, (gate combine), Out, (sum).

    x [T, Dm] (bf16 or float32), w_r [Dm, E] float32, bias [E] float32 or None,
    w_conv, w_gate [E, De, Dm] and w_out [E, Dm, De] in the library layout.
    ``core`` (CoreParams): the dense core runs between the projections, Y =
    core(H), over sequences of ``seq_len`` tokens (all T if None); without it
    Y = H. ``keep_uz`` (top-1): keep the float32 u and z of every token for a
    backward (the Conv+Gate projection then writes them and the gate combine
    forms h, instead of the fused u * SiLU(z) epilogue).
    Returns the BlockBuffers holding O (``.out``) and the intermediates.
    """
    T, Dm = x.shape
    E, De, _ = w_conv.shape
    if bufs is None:
        bufs = BlockBuffers(T, Dm, De, E, k, x.dtype, x.device, core, seq_len,
                            keep_uz=keep_uz)
    rb = route_and_dispatch(x, w_r, bias, E, k, renorm, bufs.routing, stream)
    R = T * k
    xs = rb.x_sorted[:R]
    if core is not None:
        # u and z per slot (float32); H in token order (the sum over the
        # slots for k > 1); Y = core(H) written just before the z rows, so
        # that [Y; z] feed the gate combine (Y per token, z per slot).
        rom_expert_proj(ROM_PROJ_CONV_GATE_SLOTS, xs, w_conv, w_gate, E, k, rb.offsets,
                        rb.sorted_slot, rb.topk_w, bufs.uz, stream)
        flat = bufs.uz.view(2 * R, De)
        y_rows = flat[R - T:R]
        if k > 1:
            rom_combine(ROM_COMBINE_SUM, ROM_F32, bufs.uz[0], T, k, De, None, bufs.hsum, stream)
            rom_ssm_core(bufs.hsum, seq_len or T, core, y_rows, bufs.core_ws, stream, rb)
        else:
            rom_ssm_core(flat[:T], seq_len or T, core, y_rows, bufs.core_ws, stream, rb)
        rom_combine(ROM_COMBINE_GATE_DENSE, _dtype_code(x), flat[R - T:], T, k, De, rb.slot_pos,
                    bufs.h_sorted, stream)
        if k == 1:
            rom_expert_proj(ROM_PROJ_OUT, bufs.h_sorted[:R], w_out, None, E, k, rb.offsets,
                            rb.sorted_slot, rb.topk_w, bufs.out, stream)
        else:
            rom_expert_proj(ROM_PROJ_OUT, bufs.h_sorted[:R], w_out, None, E, k, rb.offsets,
                            rb.sorted_slot, rb.topk_w, bufs.o_slots, stream)
            rom_combine(ROM_COMBINE_SUM, _dtype_code(x), bufs.o_slots, T, k, Dm, None, bufs.out,
                        stream)
        return bufs
    if k == 1 and keep_uz:
        if bufs.uz is None:
            raise RomError("keep_uz needs BlockBuffers made with keep_uz=True")
        rom_expert_proj(ROM_PROJ_CONV_GATE_SLOTS, xs, w_conv, w_gate, E, k, rb.offsets,
                        rb.sorted_slot, rb.topk_w, bufs.uz, stream)
        rom_combine(ROM_COMBINE_GATE, _dtype_code(x), bufs.uz, T, k, De, rb.slot_pos,
                    bufs.h_sorted, stream)
        rom_expert_proj(ROM_PROJ_OUT, bufs.h_sorted[:R], w_out, None, E, k, rb.offsets,
                        rb.sorted_slot, rb.topk_w, bufs.out, stream)
    elif k == 1:
        rom_expert_proj(ROM_PROJ_CONV_GATE, xs, w_conv, w_gate, E, k, rb.offsets, rb.sorted_slot,
                        rb.topk_w, bufs.h_sorted, stream)
        rom_expert_proj(ROM_PROJ_OUT, bufs.h_sorted[:R], w_out, None, E, k, rb.offsets,
                        rb.sorted_slot, rb.topk_w, bufs.out, stream)
    else:
        rom_expert_proj(ROM_PROJ_CONV_GATE, xs, w_conv, w_gate, E, k, rb.offsets, rb.sorted_slot,
                        rb.topk_w, bufs.uz, stream)
        rom_combine(ROM_COMBINE_GATE, _dtype_code(x), bufs.uz, T, k, De, rb.slot_pos,
                    bufs.h_sorted, stream)
        rom_expert_proj(ROM_PROJ_OUT, bufs.h_sorted[:R], w_out, None, E, k, rb.offsets,
                        rb.sorted_slot, rb.topk_w, bufs.o_slots, stream)
        rom_combine(ROM_COMBINE_SUM, _dtype_code(x), bufs.o_slots, T, k, Dm, None, bufs.out,
                    stream)
    return bufs


def inproj_forward(x, w_r, w, k=1, renorm=False, bias=None, bufs=None, out=None, slots=None,
                   stream=None, dense_small=True, w_tiled=None):
    """Swimba routed in-projection: s_t = sum_j r_{t,j} x_t W_{S_j} (W as [E, N, Dm]).

    A bf16 batch of at most DENSE_SMALL_MAX_TOKENS tokens (a decode step)
    takes the projection without a dispatch (rom_expert_proj_dense) unless
    ``dense_small`` is False; the router then forms neither the per-expert
    counts nor the per-chunk histograms (``bufs.counts`` is left as it was),
    which only a dispatch needs. ``w_tiled`` (pack_expert_weights(w)), when
    given, is what that path reads instead of ``w``."""
    T, Dm = x.shape
    E, N, _ = w.shape
    R = T * k
    if out is None:
        out = torch.empty((T, N), dtype=x.dtype, device=x.device)
    if dense_small and x.dtype == torch.bfloat16 and 0 < T <= DENSE_SMALL_MAX_TOKENS:
        if bufs is None:
            bufs = RoutingBuffers(T, Dm, E, k, x.dtype, x.device)
        rom_route(x, w_r, bias, k, renorm, bufs.topk_idx, bufs.topk_w, None, None, stream)
        wd = w if w_tiled is None else w_tiled
        tiled = w_tiled is not None
        if k == 1:
            rom_expert_proj_dense(ROM_PROJ_INPROJ, x, wd, E, k, bufs.topk_idx, bufs.topk_w, out,
                                  stream, tiled)
        else:
            if slots is None:
                slots = torch.empty((R, N), dtype=torch.float32, device=x.device)
            rom_expert_proj_dense(ROM_PROJ_INPROJ, x, wd, E, k, bufs.topk_idx, bufs.topk_w, slots,
                                  stream, tiled)
            rom_combine(ROM_COMBINE_SUM, _dtype_code(x), slots, T, k, N, None, out, stream)
        return out, bufs
    rb = route_and_dispatch(x, w_r, bias, E, k, renorm, bufs, stream)
    if k == 1:
        rom_expert_proj(ROM_PROJ_INPROJ, rb.x_sorted[:R], w, None, E, k, rb.offsets,
                        rb.sorted_slot, rb.topk_w, out, stream)
    else:
        if slots is None:
            slots = torch.empty((R, N), dtype=torch.float32, device=x.device)
        rom_expert_proj(ROM_PROJ_INPROJ, rb.x_sorted[:R], w, None, E, k, rb.offsets,
                        rb.sorted_slot, rb.topk_w, slots, stream)
        rom_combine(ROM_COMBINE_SUM, _dtype_code(x), slots, T, k, N, None, out, stream)
    return out, rb


# ------------------------------------------------------------------ projection variants

PROJECTIONS = ("conv", "gate", "out")


class VariantBuffers:
    """Buffers of one forward of a projection variant (allocated by torch)."""

    def __init__(self, T, Dm, De, k, dtype, device):
        R = T * k
        self.routings = {}  # id(router weight) -> RoutingBuffers, made on first use
        self.uz = torch.empty((2 * R, De), dtype=torch.float32, device=device)
        self.h = torch.empty((R, De), dtype=dtype, device=device)
        self.o_slots = torch.empty((R, Dm), dtype=torch.float32, device=device)
        self.out = torch.empty((T, Dm), dtype=dtype, device=device)


def variant_block_forward(x, routers, weighted, w_conv, w_gate, w_out, k, renorm=False,
                          bias=None, bufs=None, stream=None,
                          phases=("route", "project", "output")):
    """Projection block with each of Conv, Gate and Out dense or routed.

    routers: {"conv", "gate", "out"} -> router weight [Dm, E] float32, or None
    for a dense projection (its weight stack then holds one matrix). The same
    tensor passed for several projections is one shared routing decision
    (routed and dispatched once). weighted: the same keys -> True when that
    projection's expert outputs are scaled by its routing weights (Out must
    be weighted when routed). Weights in the library layout [E, N, K].

    Independently routed MoE-Mamba (RoM page, Knowl 4) passes three routers
    and weights all three; RoM (Gate, Out) (Knowl 3) passes None for Conv and
    one router for Gate and Out. Returns the VariantBuffers (O in ``.out``).

    ``phases`` runs a subset of the three steps, in order, on ``bufs`` from
    an earlier call: "route" (route and dispatch every distinct router),
    "project" (the Conv and Gate projections to float32 rows) and "output"
    (the gate combine and the Out projection).
    """
    T, Dm = x.shape
    De = w_conv.shape[1]
    R = T * k
    if routers["out"] is not None and not weighted["out"]:
        raise RomError("a routed Out projection is weighted by its routing weights")
    if routers["gate"] is None and routers["conv"] is not None and k > 1:
        raise RomError("a dense Gate projection with routed Conv needs k == 1")
    if bufs is None:
        bufs = VariantBuffers(T, Dm, De, k, x.dtype, x.device)
    wts = {"conv": w_conv, "gate": w_gate, "out": w_out}
    rbs = {}
    for n in PROJECTIONS:
        w_r = routers[n]
        if w_r is None:
            rbs[n] = None
            continue
        key = id(w_r)
        if key not in bufs.routings:
            bufs.routings[key] = RoutingBuffers(T, Dm, w_r.shape[1], k, x.dtype, x.device)
        rb = bufs.routings[key]
        # route each distinct router once
        if "route" in phases and not any(rbs.get(m) is rb for m in rbs):
            route_and_dispatch(x, w_r, bias, w_r.shape[1], k, renorm, rb, stream)
        rbs[n] = rb

    def project_slots(name, dst):
        rb = rbs[name]
        if rb is None:  # dense: one matrix over the tokens in order
            rom_expert_proj(ROM_PROJ_SLOTS, x, wts[name], None, 1, 1, None, None, None, dst,
                            stream)
        else:
            rom_expert_proj(ROM_PROJ_SLOTS, rb.x_sorted[:R], wts[name], None, wts[name].shape[0],
                            k, rb.offsets, rb.sorted_slot, rb.topk_w if weighted[name] else None,
                            dst, stream)

    conv_rows = T if rbs["conv"] is None else R
    gate_rows = T if rbs["gate"] is None else R
    if "project" in phases:
        project_slots("conv", bufs.uz[:conv_rows])
        project_slots("gate", bufs.uz[conv_rows:conv_rows + gate_rows])
    if "output" not in phases:
        return bufs
    rb_o = rbs["out"]
    dt = _dtype_code(x)
    h_pos = None if rb_o is None else rb_o.slot_pos
    h_rows = T if rb_o is None else R
    if rbs["conv"] is None and k > 1:
        rom_combine(ROM_COMBINE_GATE_DENSE, dt, bufs.uz[:T + R], T, k, De, h_pos, bufs.h, stream)
    else:
        # both Conv and Gate routed (u and z per slot), or k == 1 (a dense one
        # has one row per token, which is also its slot)
        rom_combine(ROM_COMBINE_GATE, dt, bufs.uz[:2 * R], T, k, De, h_pos, bufs.h, stream)
    if rb_o is None:
        rom_expert_proj(ROM_PROJ_SLOTS, bufs.h[:T], w_out, None, 1, 1, None, None, None,
                        bufs.o_slots[:T], stream)
        rom_combine(ROM_COMBINE_SUM, dt, bufs.o_slots[:T], T, 1, Dm, None, bufs.out, stream)
    elif k == 1:
        rom_expert_proj(ROM_PROJ_OUT, bufs.h[:h_rows], w_out, None, w_out.shape[0], k,
                        rb_o.offsets, rb_o.sorted_slot, rb_o.topk_w, bufs.out, stream)
    else:
        rom_expert_proj(ROM_PROJ_OUT, bufs.h[:h_rows], w_out, None, w_out.shape[0], k,
                        rb_o.offsets, rb_o.sorted_slot, rb_o.topk_w, bufs.o_slots, stream)
        rom_combine(ROM_COMBINE_SUM, dt, bufs.o_slots, T, k, Dm, None, bufs.out, stream)
    return bufs


# ------------------------------------------------------------------ backward


def rom_bwd_gather(dout, k, sorted_slot, topk_w, rdo_sorted, stream=None):
    T, N = dout.shape
    _check(load_library().rom_bwd_gather(_ptr(dout), T, k, N, _ptr(sorted_slot), _ptr(topk_w),
                                         _ptr(rdo_sorted), _stream(stream)), "rom_bwd_gather")


def rom_bwd_dgrad_out(rdo_sorted, w_out, E, k, offsets, sorted_slot, h_sorted, g_slots, dr_part,
                      stream=None):
    R, Dm = rdo_sorted.shape
    De = w_out.shape[2]
    _check(load_library().rom_bwd_dgrad_out(
        _ptr(rdo_sorted), R, Dm, _ptr(w_out), De, E, k, _ptr(offsets), _ptr(sorted_slot),
        _ptr(h_sorted), _ptr(g_slots), _ptr(dr_part), _stream(stream)), "rom_bwd_dgrad_out")


def rom_bwd_gate(uz, g_slots, T, k, De, slot_pos, dhz_sorted, stream=None):
    _check(load_library().rom_bwd_gate(_ptr(uz), _ptr(g_slots), T, k, De, _ptr(slot_pos),
                                       _ptr(dhz_sorted), _stream(stream)), "rom_bwd_gate")


def rom_bwd_dgrad_in(dhz_sorted, w_in, w_g, E, k, offsets, sorted_slot, dx_slots, stream=None):
    R = dhz_sorted.shape[0]
    De = dhz_sorted.shape[1] // 2
    Dm = w_in.shape[2]
    _check(load_library().rom_bwd_dgrad_in(
        _ptr(dhz_sorted), R, De, _ptr(w_in), _ptr(w_g), Dm, E, k, _ptr(offsets),
        _ptr(sorted_slot), _ptr(dx_slots), _stream(stream)), "rom_bwd_dgrad_in")


def rom_route_bwd(T, k, E, Dm, renorm, topk_idx, topk_w, dr_part, dx_slots, w_r, dlogits, dx,
                  stream=None, probs=None):
    _check(load_library().rom_route_bwd(
        T, k, E, Dm, int(renorm), _ptr(topk_idx), _ptr(topk_w), _ptr(probs), _ptr(dr_part),
        dr_part.shape[1], _ptr(dx_slots), _ptr(w_r), _ptr(dlogits), _ptr(dx), _stream(stream)),
        "rom_route_bwd")


def rom_route_probs(x, w_r, bias, probs, stream=None):
    T, Dm = x.shape
    _check(load_library().rom_route_probs(_ptr(x), _dtype_code(x), T, Dm, _ptr(w_r), _ptr(bias),
                                          w_r.shape[1], _ptr(probs), _stream(stream)),
           "rom_route_probs")


def rom_route_wgrad(x, dlogits, dw_r, dbias, stream=None):
    T, Dm = x.shape
    _check(load_library().rom_route_wgrad(_ptr(x), _dtype_code(x), T, Dm, dlogits.shape[1],
                                          _ptr(dlogits), _ptr(dw_r), _ptr(dbias),
                                          _stream(stream)), "rom_route_wgrad")


def rom_bwd_wgrad(a_sorted, b_sorted, E, offsets, m_split, out0, out1, stream=None):
    R, M = a_sorted.shape
    N = b_sorted.shape[1]
    _check(load_library().rom_bwd_wgrad(
        _ptr(a_sorted), M, _ptr(b_sorted), N, R, E, _ptr(offsets), m_split, _ptr(out0),
        _ptr(out1), _stream(stream)), "rom_bwd_wgrad")


class GradientAllReduce:
    """Data-parallel exchange of the weight gradients: every rank holds the
    gradients of its own tokens, and each tensor handed to ``start`` is summed
    over the ranks of ``group`` (torch.distributed all-reduce: NCCL over
    NVLink between GPUs, gloo between CPU processes). A transfer is started
    as soon as the kernel that produces its tensor is enqueued, so it overlaps
    the rest of the backward; ``finish`` makes the current stream wait for
    all of them. Every rank must start the same tensors in the same order.
    The token batch is split across ranks and the expert and router weights
    are replicated; the tokens themselves are never exchanged."""

    def __init__(self, group=None):
        self.group = group
        self.pending = []

    def start(self, *tensors):
        import torch.distributed as dist
        for t in tensors:
            self.pending.append(dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group,
                                                async_op=True))

    def finish(self):
        for w in self.pending:
            w.wait()
        self.pending = []


class BackwardBuffers:
    """Device buffers of one backward pass (allocated by torch)."""

    def __init__(self, T, Dm, De, E, k, device):
        R = T * k
        bf = torch.bfloat16
        self.rdo_sorted = torch.empty((R, Dm), dtype=bf, device=device)
        self.g_slots = torch.empty((R, De), dtype=torch.float32, device=device)
        self.dr_part = torch.empty((R, De // 256), dtype=torch.float32, device=device)
        self.dhz_sorted = torch.empty((R, 2 * De), dtype=bf, device=device)
        self.dx_slots = torch.empty((R, Dm), dtype=torch.float32, device=device)
        self.dx = torch.empty((T, Dm), dtype=bf, device=device)
        self.dlogits = torch.empty((T, E), dtype=torch.float32, device=device)
        self.dw_out = torch.empty((E, Dm, De), dtype=torch.float32, device=device)
        self.dw_conv = torch.empty((E, De, Dm), dtype=torch.float32, device=device)
        self.dw_gate = torch.empty((E, De, Dm), dtype=torch.float32, device=device)
        self.dw_r = torch.empty((Dm, E), dtype=torch.float32, device=device)
        self.dbias = torch.empty((E,), dtype=torch.float32, device=device)
        self.probs = torch.empty((T, E), dtype=torch.float32, device=device)


def block_backward(fwd, dout, w_r, w_conv, w_gate, w_out, renorm=True, bufs=None, stream=None,
                   x=None, bias=None, grad_sync=None):
    """Backward of the RoM block (renormalised weights, or r = p with ``x``).

    fwd: the BlockBuffers of the forward (routing, h_sorted, u/z slot
    partials: for k == 1 the forward must have run with keep_uz=True);
    dout [T, Dm] bf16; weights in the library layout. With ``x`` (the
    forward's input) the router weight gradients dw_r [Dm, E] and dbias [E]
    are computed too; r = p (renorm=False) needs ``x`` (and the forward's
    ``bias``) for the softmax over all experts. Returns BackwardBuffers with
    dx [T, Dm] bf16, dlogits [T, E] and dw_conv / dw_gate [E, De, Dm],
    dw_out [E, Dm, De] (float32, the weights' layout).
    ``grad_sync`` (a GradientAllReduce): data-parallel training; the weight
    gradients are summed over its ranks, dW_out while the rest of the
    backward runs.
    """
    rb = fwd.routing
    T, Dm = dout.shape
    E, De, _ = w_conv.shape
    k = rb.k
    if fwd.uz is None:
        raise RomError("block_backward needs the forward's u/z slot partials "
                       "(top-k > 1, or block_forward(..., keep_uz=True))")
    if not renorm and x is None:
        raise RomError("the backward of r = p needs the forward's input x")
    R = T * k
    if bufs is None:
        bufs = BackwardBuffers(T, Dm, De, E, k, dout.device)
    rom_bwd_gather(dout, k, rb.sorted_slot, rb.topk_w, bufs.rdo_sorted, stream)
    rom_bwd_dgrad_out(bufs.rdo_sorted, w_out, E, k, rb.offsets, rb.sorted_slot,
                      fwd.h_sorted[:R], bufs.g_slots, bufs.dr_part, stream)
    if grad_sync is not None:
        # dW_out first, so that its exchange overlaps the rest of the backward
        rom_bwd_wgrad(bufs.rdo_sorted, fwd.h_sorted[:R], E, rb.offsets, Dm, bufs.dw_out, None,
                      stream)
        grad_sync.start(bufs.dw_out)
    rom_bwd_gate(fwd.uz, bufs.g_slots, T, k, De, rb.slot_pos, bufs.dhz_sorted, stream)
    rom_bwd_dgrad_in(bufs.dhz_sorted, w_conv, w_gate, E, k, rb.offsets, rb.sorted_slot,
                     bufs.dx_slots, stream)
    if not renorm:
        rom_route_probs(x, w_r, bias, bufs.probs, stream)
    rom_route_bwd(T, k, E, Dm, renorm, rb.topk_idx, rb.topk_w, bufs.dr_part, bufs.dx_slots, w_r,
                  bufs.dlogits, bufs.dx, stream, probs=None if renorm else bufs.probs)
    if x is not None:
        rom_route_wgrad(x, bufs.dlogits, bufs.dw_r, bufs.dbias, stream)
        if grad_sync is not None:
            grad_sync.start(bufs.dw_r, bufs.dbias)
    if grad_sync is None:
        rom_bwd_wgrad(bufs.rdo_sorted, fwd.h_sorted[:R], E, rb.offsets, Dm, bufs.dw_out, None,
                      stream)
    rom_bwd_wgrad(bufs.dhz_sorted, rb.x_sorted[:R], E, rb.offsets, De, bufs.dw_conv, bufs.dw_gate,
                  stream)
    if grad_sync is not None:
        grad_sync.start(bufs.dw_conv, bufs.dw_gate)
        grad_sync.finish()
    return bufs


# ------------------------------------------------------------------ host buffers, pipelined


class HostPipeline:
    """Forward of the block (or the Swimba in-projection) on HOST tensors.

    Tokens are independent, so the batch is cut into chunks (multiples of the
    128-token routing chunk) that go through three stages, each on streams of
    its own: the host-to-device copies on one stream, the kernels on two
    (a chunk of a few thousand tokens leaves the GPU room for a second one),
    the device-to-host copies on one, chained by events. The input copy of one
    chunk, the kernels of the previous ones and the output copy of an earlier
    one run at the same time, and the two copy directions overlap on the
    link. `nstreams` device buffer sets rotate over the chunks; a set takes a
    new chunk once its last chunk's output copy has completed. Each token's
    routing is the one a single call on the whole batch gives, and so is its
    output when the chunk and the batch take the same projection kernels
    (more than 1024 routed rows each); a short last chunk may take the
    swap-AB Out GEMM, whose output agrees within the forward's tolerance.
    Chunks of 2048 tokens and four buffer sets measured best for the prefill
    batch (smaller chunks cost more GEMM efficiency than the shorter first
    and last copies save). Device buffers are allocated once (torch); the
    kernels are the library's.

    With ``graph=True`` the second call with the same host buffers, weights
    and size captures the whole multi-stream sequence (copies and kernels)
    into a CUDA graph, and later such calls replay it: the host then issues
    one launch per call instead of some ten per chunk. The first call runs
    eagerly (it also initialises the library's per-device state).
    """

    def __init__(self, T, Dm, N_out, E, k, dtype, device="cuda", chunks=8, nstreams=4,
                 De=None, graph=True, min_chunk=2048):
        self.T, self.Dm, self.E, self.k = T, Dm, E, k
        self.graph = graph
        self._graphs, self._seen, self._tail = {}, set(), {}
        per = -(-T // chunks)
        # Chunks of at least min_chunk tokens (smaller ones lose more GEMM
        # efficiency and launch time than their shorter first and last copies
        # save), at most the batch.
        self.chunk = min(max(min_chunk, -(-per // 128) * 128), max(128, -(-T // 128) * 128))
        self.nbuf = nstreams
        self.s_in = torch.cuda.Stream(device=device)
        self.s_out = torch.cuda.Stream(device=device)
        self.s_comp = [torch.cuda.Stream(device=device) for _ in range(2)]
        self.x = [torch.empty((self.chunk, Dm), dtype=dtype, device=device) for _ in range(nstreams)]
        if De is not None:  # RoM block
            self.bufs = [BlockBuffers(self.chunk, Dm, De, E, k, dtype, device) for _ in range(nstreams)]
        else:  # in-projection
            self.bufs = [RoutingBuffers(self.chunk, Dm, E, k, dtype, device) for _ in range(nstreams)]
            self.out = [torch.empty((self.chunk, N_out), dtype=dtype, device=device)
                        for _ in range(nstreams)]
            self.slots = ([torch.empty((self.chunk * k, N_out), dtype=torch.float32, device=device)
                           for _ in range(nstreams)] if k > 1 else [None] * nstreams)

    def _chunks(self, T):
        return [(i, min(T, i + self.chunk)) for i in range(0, T, self.chunk)]

    def _run(self, T, body):
        """body = (copy_in, compute, copy_out), each called (j, a, b, stream)
        for every chunk [a, b) with buffer set j: one chunk runs on the
        current stream, several go through the staged streams."""
        copy_in, compute, copy_out = body
        cur = torch.cuda.current_stream()
        chunks = self._chunks(T)
        if len(chunks) == 1:
            for f in body:
                f(0, 0, T, cur)
            return
        start = torch.cuda.Event()
        start.record(cur)
        streams = [self.s_in, self.s_out] + self.s_comp
        for s in streams:
            s.wait_event(start)
        free = [None] * self.nbuf  # buffer set j: its last output copy
        for n, (a, b) in enumerate(chunks):
            j = n % self.nbuf
            with torch.cuda.stream(self.s_in):
                if free[j] is not None:
                    self.s_in.wait_event(free[j])
                copy_in(j, a, b, self.s_in)
                e_in = torch.cuda.Event()
                e_in.record(self.s_in)
            sc = self.s_comp[n % len(self.s_comp)]
            with torch.cuda.stream(sc):
                sc.wait_event(e_in)
                compute(j, a, b, sc)
                e_c = torch.cuda.Event()
                e_c.record(sc)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(e_c)
                copy_out(j, a, b, self.s_out)
                free[j] = torch.cuda.Event()
                free[j].record(self.s_out)
        for s in streams:
            ev = torch.cuda.Event()
            ev.record(s)
            cur.wait_event(ev)

    def _launch(self, key, T, body):
        """Eager on the first call for `key`, captured into a CUDA graph on
        the second, replayed afterwards."""
        if not self.graph:
            self._run(T, body)
            return
        g = self._graphs.get(key)
        if g is None and key in self._seen:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._run(T, body)
            self._graphs[key] = g
        if g is None:
            self._seen.add(key)
            self._run(T, body)
        else:
            g.replay()

    def _tail_bufs(self, n, make):
        """Buffers of a shorter last chunk, made once per size (outside any capture)."""
        if n not in self._tail:
            self._tail[n] = make(n)
        return self._tail[n]

    def block_forward(self, x_host, w_r, bias, w_conv, w_gate, w_out, out_host, renorm=False):
        """x_host [T, Dm] and out_host [T, Dm]: pinned host tensors."""
        T = x_host.shape[0]
        De = w_conv.shape[1]
        for a, b in self._chunks(T):
            if b - a != self.chunk:
                self._tail_bufs(b - a, lambda n: BlockBuffers(n, self.Dm, De, self.E, self.k,
                                                              self.x[0].dtype, self.x[0].device))

        def bufs_of(j, a, b):
            return self.bufs[j] if b - a == self.chunk else self._tail[b - a]

        def copy_in(j, a, b, s):
            self.x[j][: b - a].copy_(x_host[a:b], non_blocking=True)

        def compute(j, a, b, s):
            block_forward(self.x[j][: b - a], w_r, bias, w_conv, w_gate, w_out, self.k, renorm,
                          bufs_of(j, a, b), stream=s)

        def copy_out(j, a, b, s):
            out_host[a:b].copy_(bufs_of(j, a, b).out, non_blocking=True)

        body = (copy_in, compute, copy_out)

        key = ("block", T, x_host.data_ptr(), out_host.data_ptr(), w_r.data_ptr(),
               0 if bias is None else bias.data_ptr(), w_conv.data_ptr(), w_gate.data_ptr(),
               w_out.data_ptr(), bool(renorm))
        self._launch(key, T, body)
        return out_host

    def inproj_forward(self, x_host, w_r, w, out_host, renorm=False, bias=None, w_tiled=None):
        """x_host [T, Dm], out_host [T, N_out]: pinned host tensors."""
        T = x_host.shape[0]
        for a, b in self._chunks(T):
            if b - a != self.chunk:
                self._tail_bufs(b - a, lambda n: RoutingBuffers(n, self.Dm, self.E, self.k,
                                                                self.x[0].dtype, self.x[0].device))

        def copy_in(j, a, b, s):
            self.x[j][: b - a].copy_(x_host[a:b], non_blocking=True)

        def compute(j, a, b, s):
            bufs = self.bufs[j] if b - a == self.chunk else self._tail[b - a]
            sl = None if self.slots[j] is None else self.slots[j][: (b - a) * self.k]
            inproj_forward(self.x[j][: b - a], w_r, w, self.k, renorm, bias, bufs,
                           self.out[j][: b - a], sl, stream=s, w_tiled=w_tiled)

        def copy_out(j, a, b, s):
            out_host[a:b].copy_(self.out[j][: b - a], non_blocking=True)

        body = (copy_in, compute, copy_out)

        key = ("inproj", T, x_host.data_ptr(), out_host.data_ptr(), w_r.data_ptr(), w.data_ptr(),
               0 if bias is None else bias.data_ptr(), bool(renorm),
               0 if w_tiled is None else w_tiled.data_ptr())
        self._launch(key, T, body)
        return out_host
