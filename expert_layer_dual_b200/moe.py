"""ctypes binding of libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: every function here hands device pointers, sizes
and the current CUDA stream to the entry point of the same name and raises
``MoEError`` on a non-zero status.  All arithmetic runs in the library's
CUDA kernels; there is no CPU path.  PyTorch supplies device memory and
streams.

Loading fails loudly: importing this module raises ``ImportError`` when the
shared library has not been built (``python -m expert_layer_dual_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .configs import MoEConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m expert_layer_dual_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

OK, INVALID_ARG, UNSUPPORTED, CUDA_ERROR, WORKSPACE_TOO_SMALL, DEVICE_TIMEOUT, DEVICE_BAD_INDEX = range(7)
WDTYPE_BF16, WDTYPE_FP8_BLOCK128, WDTYPE_MXFP8, WDTYPE_FP8_TENSOR = 0, 1, 2, 3

EXPORTS = ["moe_status_string", "moe_workspace_bytes", "moe_permute_workspace_bytes",
           "moe_router_split", "moe_quantize_weights_fp8", "moe_quantize_act_fp8",
           "moe_quantize_act_fp8_permuted", "moe_quantize_weights_mxfp8", "moe_quantize_act_mxfp8",
           "moe_quantize_act_mxfp8_permuted", "moe_quantize_weights_fp8_tensor",
           "moe_quantize_act_fp8_static", "moe_quantize_act_fp8_static_permuted",
           "moe_router_logits", "moe_route_topk", "moe_permute", "moe_permute_noalloc",
           "moe_gemm_gateup",
           "moe_gemm_down", "moe_combine", "moe_forward", "moe_forward_profiled", "moe_forward_host",
           "moe_forward_host_async",
           "moe_read_device_status", "moe_selftest_timeout", "moe_workspace_offsets",
           "moe_calibrate_fp8_static", "moe_route", "moe_ep_dispatch", "moe_gather_rows",
           "moe_lamport_buffer_bytes", "moe_lamport_init", "moe_allreduce_rmsnorm",
           "moe_allreduce_rmsnorm_emulated", "moe_peer_buffer_alloc", "moe_peer_buffer_open",
           "moe_peer_buffer_close", "moe_peer_buffer_free"]


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("I", ctypes.c_int32), ("I_shared", ctypes.c_int32),
                ("wdtype", ctypes.c_int32), ("renormalize", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_gu", "w_d", "w_gu_scale", "w_d_scale", "ws_gu", "ws_d", "ws_gu_scale",
                 "ws_d_scale", "router_hi", "router_lo", "router_bias")] + \
               [("act_scale_x", ctypes.c_float), ("act_scale_h", ctypes.c_float)]


class moe_workspace_map(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("logits", "ids", "w", "counts", "offsets", "perm", "inv", "xq", "xs", "h", "total")]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_S, _W = ctypes.POINTER(moe_shape), ctypes.POINTER(moe_weights)
_sig = {
    "moe_status_string": (ctypes.c_char_p, [_i32]),
    "moe_workspace_bytes": (_sz, [_S]),
    "moe_permute_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "moe_router_split": (_i32, [_vp, _vp, _vp, _i64, _vp]),
    "moe_quantize_weights_fp8": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp]),
    "moe_quantize_act_fp8": (_i32, [_vp, _i64, _i32, _vp, _vp, _vp]),
    "moe_quantize_act_fp8_permuted": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_quantize_weights_mxfp8": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp]),
    "moe_quantize_weights_fp8_tensor": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _vp]),
    "moe_quantize_act_fp8_static": (_i32, [_vp, _i64, _i32, ctypes.c_float, _vp, _vp]),
    "moe_quantize_act_fp8_static_permuted": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, ctypes.c_float,
                                                    _vp, _vp]),
    "moe_quantize_act_mxfp8": (_i32, [_vp, _i64, _i32, _vp, _vp, _vp]),
    "moe_quantize_act_mxfp8_permuted": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_router_logits": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp]),
    "moe_route_topk": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_permute": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "moe_gemm_gateup": (_i32, [_S, _W, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_gemm_down": (_i32, [_S, _W, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_combine": (_i32, [_S, _vp, _vp, _vp, _vp, _vp]),
    "moe_forward": (_i32, [_S, _W, _vp, _vp, _vp, _sz, _vp]),
    "moe_forward_profiled": (_i32, [_S, _W, _vp, _vp, _vp, _sz, _vp, ctypes.POINTER(_vp), _i32]),
    "moe_forward_host": (_i32, [_S, _W, _vp, _vp, _vp, _sz, _vp]),
    "moe_forward_host_async": (_i32, [_S, _W, _vp, _vp, _vp, _sz, _vp]),
    "moe_read_device_status": (_i32, [_vp, _vp]),
    "moe_selftest_timeout": (_i32, [_vp, _i32, _vp]),
    "moe_workspace_offsets": (_i32, [_S, ctypes.POINTER(moe_workspace_map)]),
    "moe_calibrate_fp8_static": (_i32, [_S, _W, _vp, _vp, _vp, _sz, _vp]),
    "moe_route": (_i32, [_S, _W, _vp, _vp, _sz, _vp]),
    "moe_ep_dispatch": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_gather_rows": (_i32, [_vp, _vp, _i64, _i32, _vp, _vp]),
    "moe_lamport_buffer_bytes": (_sz, [_i32, _i32, _i32]),
    "moe_lamport_init": (_i32, [_vp, _sz, _vp]),
    "moe_allreduce_rmsnorm": (_i32, [ctypes.POINTER(_vp), _i32, _i32, ctypes.c_uint32, _i32, _vp, _vp,
                                     _vp, ctypes.c_float, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "moe_allreduce_rmsnorm_emulated": (_i32, [ctypes.POINTER(_vp), _i32, _i32, ctypes.c_uint32, _i32,
                                              ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp,
                                              ctypes.c_float, _i32, _i32, ctypes.POINTER(_vp),
                                              ctypes.POINTER(_vp), _i32, _vp, _sz, _vp]),
    "moe_peer_buffer_alloc": (_i32, [_sz, ctypes.POINTER(_vp), _vp]),
    "moe_peer_buffer_open": (_i32, [_vp, ctypes.POINTER(_vp)]),
    "moe_peer_buffer_close": (_i32, [_vp]),
    "moe_peer_buffer_free": (_i32, [_vp]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def status_string(code: int) -> str:
    return _lib.moe_status_string(code).decode()


def _check(code: int, where: str) -> None:
    if code != OK:
        raise MoEError(code, where)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if t.numel() and not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return ctypes.c_void_p(t.data_ptr()) if t.numel() else None


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def shape_of(cfg: MoEConfig, T: Optional[int] = None) -> moe_shape:
    return moe_shape(cfg.T if T is None else T, cfg.d, cfg.E, cfg.k, cfg.I, cfg.Is, cfg.wdtype,
                     int(cfg.renorm))


# ------------------------------------------------------------------ entry points
def workspace_bytes(shape: moe_shape) -> int:
    return int(_lib.moe_workspace_bytes(ctypes.byref(shape)))


def workspace_offsets(shape: moe_shape) -> moe_workspace_map:
    m = moe_workspace_map()
    _check(_lib.moe_workspace_offsets(ctypes.byref(shape), ctypes.byref(m)), "moe_workspace_offsets")
    return m


def workspace_view(ws: torch.Tensor, shape: moe_shape) -> dict:
    """Views (no copies) of the routing intermediates, the quantised
    activations (FP8 formats) and h (BF16) that moe_forward leaves in `ws`,
    at the offsets moe_workspace_offsets reports."""
    m = workspace_offsets(shape)
    T, E, k = shape.T, shape.E, shape.k
    R = T * k + (T if shape.I_shared else 0)

    def region(off, n, dtype):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return ws[off: off + nbytes].view(dtype)

    out = {"logits": region(m.logits, T * E, torch.float32).view(T, E),
           "ids": region(m.ids, T * k, torch.int32).view(T, k),
           "w": region(m.w, T * k, torch.float32).view(T, k),
           "counts": region(m.counts, E, torch.int32),
           "offsets": region(m.offsets, E + 1, torch.int32),
           "perm": region(m.perm, T * k, torch.int32),
           "inv": region(m.inv, T * k, torch.int32)}
    if shape.wdtype == WDTYPE_BF16:
        out["h"] = region(m.h, R * shape.I, torch.bfloat16).view(R, shape.I)
        if m.xq:   # the routed rows of x in permuted order (the CTA-pair gate-up's A)
            out["xq"] = region(m.xq, T * k * shape.d, torch.bfloat16).view(T * k, shape.d)
    else:
        d = shape.d
        out["xq"] = region(m.xq, R * d, torch.uint8).view(R, d)
        if shape.wdtype == WDTYPE_FP8_BLOCK128:
            out["xs"] = region(m.xs, R * (d // 128), torch.float32).view(R, d // 128)
        elif shape.wdtype == WDTYPE_MXFP8:
            out["xs"] = region(m.xs, R * (d // 32), torch.uint8)
    return out


def calibrate_fp8_static(shape, weights, x, scales, ws, stream=None):
    """moe_calibrate_fp8_static: scales (float32 [2], device) <- the static
    activation scales of x and of the BF16 gate-up output h."""
    _check(_lib.moe_calibrate_fp8_static(ctypes.byref(shape), ctypes.byref(weights), _p(x), _p(scales),
                                         _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_calibrate_fp8_static")


def route(shape, weights, x, ws, stream=None):
    """moe_route: router logits, fused top-k and permute into `ws`."""
    _check(_lib.moe_route(ctypes.byref(shape), ctypes.byref(weights), _p(x), _p(ws),
                          ws.numel() * ws.element_size(), _stream(stream)), "moe_route")


def ep_dispatch(x, ids, perm, E_local, send_rows, send_ids, stream=None):
    T, d = x.shape
    k = ids.shape[1]
    _check(_lib.moe_ep_dispatch(_p(x), _p(ids), _p(perm), T, d, k, E_local, _p(send_rows),
                                _p(send_ids), _stream(stream)), "moe_ep_dispatch")


def gather_rows(src, index, dst, stream=None):
    n = index.numel()
    row_bytes = dst.numel() * dst.element_size() // max(n, 1) if n else 16
    _check(_lib.moe_gather_rows(_p(src), _p(index), n, row_bytes, _p(dst), _stream(stream)),
           "moe_gather_rows")


def _ptrs(items) -> "ctypes.Array":
    """HOST array of device pointers (ints or tensors; None -> NULL)."""
    vals = [None if v is None else (v if isinstance(v, int) else v.data_ptr()) for v in items]
    return (_vp * len(vals))(*vals)


def lamport_buffer_bytes(G: int, T_max: int, d: int) -> int:
    return int(_lib.moe_lamport_buffer_bytes(G, T_max, d))


def lamport_init(buf, nbytes: int, stream=None):
    ptr = buf if isinstance(buf, int) else buf.data_ptr()
    _check(_lib.moe_lamport_init(ctypes.c_void_p(ptr), nbytes, _stream(stream)), "moe_lamport_init")


def allreduce_rmsnorm(bufs, rank, call, T_max, x, residual, gamma, eps, out, residual_out, ws,
                      stream=None):
    """One rank's moe_allreduce_rmsnorm; `bufs`: every rank's Lamport buffer
    (device pointers as ints, or tensors) in rank order."""
    T, d = x.shape
    _check(_lib.moe_allreduce_rmsnorm(_ptrs(bufs), len(bufs), rank, call & 0xffffffff, T_max, _p(x),
                                      _p(residual), _p(gamma), float(eps), T, d, _p(out),
                                      _p(residual_out), _p(ws), ws.numel() * ws.element_size(),
                                      _stream(stream)), "moe_allreduce_rmsnorm")


def allreduce_rmsnorm_emulated(bufs, call, T_max, xs, residuals, gamma, eps, outs, residual_outs,
                               ws, ranks=None, timeout_us=2_000_000, stream=None):
    """moe_allreduce_rmsnorm_emulated: every rank of the group in one launch
    on this GPU (lists indexed by rank; `ranks` < len(bufs) leaves the last
    ranks out)."""
    G = len(bufs)
    n = G if ranks is None else ranks
    T, d = xs[0].shape
    _check(_lib.moe_allreduce_rmsnorm_emulated(
        _ptrs(bufs), G, n, call & 0xffffffff, T_max, _ptrs(xs[:n]),
        None if residuals is None else _ptrs(residuals[:n]), _p(gamma), float(eps), T, d,
        _ptrs(outs[:n]), None if residual_outs is None else _ptrs(residual_outs[:n]), int(timeout_us),
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_allreduce_rmsnorm_emulated")


def peer_buffer_alloc(nbytes: int):
    """(device pointer, 64-byte IPC handle) of a new cudaMalloc'd buffer."""
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(64)
    _check(_lib.moe_peer_buffer_alloc(nbytes, ctypes.byref(ptr), handle), "moe_peer_buffer_alloc")
    return int(ptr.value), handle.raw


def peer_buffer_open(handle: bytes) -> int:
    ptr = ctypes.c_void_p()
    buf = ctypes.create_string_buffer(bytes(handle), 64)
    _check(_lib.moe_peer_buffer_open(buf, ctypes.byref(ptr)), "moe_peer_buffer_open")
    return int(ptr.value)


def peer_buffer_close(ptr: int):
    _check(_lib.moe_peer_buffer_close(ctypes.c_void_p(ptr)), "moe_peer_buffer_close")


def peer_buffer_free(ptr: int):
    _check(_lib.moe_peer_buffer_free(ctypes.c_void_p(ptr)), "moe_peer_buffer_free")


def permute_workspace_bytes(T: int, E: int, k: int) -> int:
    return int(_lib.moe_permute_workspace_bytes(T, E, k))


def router_split(W, hi, lo, stream=None):
    _check(_lib.moe_router_split(_p(W), _p(hi), _p(lo), W.numel(), _stream(stream)), "moe_router_split")


def quantize_weights_fp8(W, q, scale, stream=None):
    rows, cols = W.shape[-2:]
    batch = W.numel() // (rows * cols) if W.numel() else 0
    _check(_lib.moe_quantize_weights_fp8(_p(W), batch, rows, cols, _p(q), _p(scale), _stream(stream)),
           "moe_quantize_weights_fp8")


def quantize_act_fp8(x, q, scale, stream=None):
    rows, cols = x.shape
    _check(_lib.moe_quantize_act_fp8(_p(x), rows, cols, _p(q), _p(scale), _stream(stream)),
           "moe_quantize_act_fp8")


def quantize_weights_mxfp8(W, q, scale, stream=None):
    """W bf16 bits [..., rows, cols] -> q e4m3 codes (same shape), scale E8M0 bytes [..., rows, cols/32]."""
    rows, cols = W.shape[-2:]
    batch = W.numel() // (rows * cols)
    _check(_lib.moe_quantize_weights_mxfp8(_p(W), batch, rows, cols, _p(q), _p(scale), _stream(stream)),
           "moe_quantize_weights_mxfp8")


def quantize_weights_fp8_tensor(W, q, scale, stream=None):
    """W bf16 bits [..., rows, cols] -> q e4m3 (same shape), scale float32 [...] (one per matrix)."""
    rows, cols = W.shape[-2:]
    batch = W.numel() // (rows * cols)
    _check(_lib.moe_quantize_weights_fp8_tensor(_p(W), batch, rows, cols, _p(q), _p(scale),
                                                _stream(stream)), "moe_quantize_weights_fp8_tensor")


def quantize_act_fp8_static(x, scale, q, stream=None):
    rows, cols = x.shape
    _check(_lib.moe_quantize_act_fp8_static(_p(x), rows, cols, float(scale), _p(q), _stream(stream)),
           "moe_quantize_act_fp8_static")


def quantize_act_fp8_static_permuted(x, perm, k, with_shared, scale, q, stream=None):
    T, d = x.shape
    _check(_lib.moe_quantize_act_fp8_static_permuted(_p(x), _p(perm), T, k, int(with_shared), d,
                                                     float(scale), _p(q), _stream(stream)),
           "moe_quantize_act_fp8_static_permuted")


def quantize_act_mxfp8(x, q, scale, stream=None):
    rows, cols = x.shape
    _check(_lib.moe_quantize_act_mxfp8(_p(x), rows, cols, _p(q), _p(scale), _stream(stream)),
           "moe_quantize_act_mxfp8")


def quantize_act_mxfp8_permuted(x, perm, k, with_shared, q, scale, stream=None):
    T, d = x.shape
    _check(_lib.moe_quantize_act_mxfp8_permuted(_p(x), _p(perm), T, k, int(with_shared), d, _p(q),
                                                _p(scale), _stream(stream)),
           "moe_quantize_act_mxfp8_permuted")


def quantize_act_fp8_permuted(x, perm, k, with_shared, q, scale, stream=None):
    T, d = x.shape
    _check(_lib.moe_quantize_act_fp8_permuted(_p(x), _p(perm), T, k, int(with_shared), d, _p(q), _p(scale),
                                              _stream(stream)), "moe_quantize_act_fp8_permuted")


def router_logits(x, hi, lo, bias, logits, stream=None):
    T, d = x.shape
    _check(_lib.moe_router_logits(_p(x), _p(hi), _p(lo), _p(bias), _p(logits), T, d, hi.shape[0],
                                  _stream(stream)), "moe_router_logits")


def route_topk(logits, k, renormalize, ids, w, stream=None):
    T, E = logits.shape
    _check(_lib.moe_route_topk(_p(logits), T, E, k, int(renormalize), _p(ids), _p(w), _stream(stream)),
           "moe_route_topk")


def permute(ids, E, counts, offsets, perm, inv, ws, stream=None):
    T, k = ids.shape
    _check(_lib.moe_permute(_p(ids), T, E, k, _p(counts), _p(offsets), _p(perm), _p(inv), _p(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "moe_permute")


def permute_noalloc(ids, E, counts, offsets, perm, inv, stream=None):
    """moe_permute without a workspace, for callers that cannot allocate:
    the library's own fixed device scratch is used (see include/moe.h)."""
    T, k = ids.shape
    _check(_lib.moe_permute_noalloc(_p(ids), T, E, k, _p(counts), _p(offsets), _p(perm), _p(inv),
                                    _stream(stream)), "moe_permute_noalloc")


def gemm_gateup(shape, weights, x, x_scale, perm, offsets, h, h_scale, ws, stream=None):
    _check(_lib.moe_gemm_gateup(ctypes.byref(shape), ctypes.byref(weights), _p(x), _p(x_scale),
                                _p(perm), _p(offsets), _p(h), _p(h_scale), _p(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "moe_gemm_gateup")


def gemm_down(shape, weights, h, h_scale, offsets, o, ws, stream=None):
    _check(_lib.moe_gemm_down(ctypes.byref(shape), ctypes.byref(weights), _p(h), _p(h_scale),
                              _p(offsets), _p(o), _p(ws), ws.numel() * ws.element_size(),
                              _stream(stream)), "moe_gemm_down")


def combine(shape, o, inv, w, y, stream=None):
    _check(_lib.moe_combine(ctypes.byref(shape), _p(o), _p(inv), _p(w), _p(y), _stream(stream)),
           "moe_combine")


def forward(shape, weights, x, y, ws, stream=None):
    _check(_lib.moe_forward(ctypes.byref(shape), ctypes.byref(weights), _p(x), _p(y), _p(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "moe_forward")


PROFILE_EVENTS = 8
STAGES = ["router_logits", "route_topk", "permute", "quant_act", "gemm_gateup", "gemm_down", "combine"]


def forward_profiled(shape, weights, x, y, ws, events, stream=None):
    """moe_forward recording `events` (8 torch.cuda.Event(enable_timing=True),
    already recorded once so their handles exist) at the stage boundaries."""
    arr = (_vp * PROFILE_EVENTS)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(_lib.moe_forward_profiled(ctypes.byref(shape), ctypes.byref(weights), _p(x), _p(y), _p(ws),
                                     ws.numel() * ws.element_size(), _stream(stream), arr,
                                     PROFILE_EVENTS), "moe_forward_profiled")


def forward_host(shape, weights, x_host, y_host, ws, stream=None):
    _check(_lib.moe_forward_host(ctypes.byref(shape), ctypes.byref(weights), _p(x_host), _p(y_host),
                                 _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_forward_host")


def forward_host_async(shape, weights, x_host, y_host, ws, stream=None):
    _check(_lib.moe_forward_host_async(ctypes.byref(shape), ctypes.byref(weights), _p(x_host),
                                       _p(y_host), _p(ws), ws.numel() * ws.element_size(),
                                       _stream(stream)), "moe_forward_host_async")


def read_device_status(ws, stream=None) -> int:
    return int(_lib.moe_read_device_status(_p(ws), _stream(stream)))


def selftest_timeout(ws, limit_us: int, stream=None):
    _check(_lib.moe_selftest_timeout(_p(ws), int(limit_us), _stream(stream)), "moe_selftest_timeout")


# ------------------------------------------------------------------ layer object
class MoELayer:
    """One MoE layer resident on the GPU: weights in the library's layout,
    a workspace, and `forward(x) -> y` through moe_forward.

    `inputs` holds the BF16 expert weights and the FP32 router weight (as
    drawn by expert_layer_dual_b200.inputs.make_layer).  Preparation runs the
    library's offline kernels: the dual-BF16 router split and, for FP8
    layers, the 128x128 block quantisation of every expert matrix.  `act_scales`:
    the static activation scales of a per-tensor FP8 layer when they are known
    already (otherwise calibrated here on the input's first tokens)."""

    def __init__(self, cfg: MoEConfig, inputs: dict, device="cuda", max_tokens: Optional[int] = None,
                 act_scales=None):
        self.cfg = cfg
        dev = torch.device(device)
        self.max_tokens = cfg.T if max_tokens is None else max_tokens
        E, d = cfg.E, cfg.d
        rw = inputs["router_w"].to(dev, torch.float32).contiguous()
        self.router_hi = torch.empty((E, d), dtype=torch.uint16, device=dev)
        self.router_lo = torch.empty((E, d), dtype=torch.uint16, device=dev)
        router_split(rw, self.router_hi, self.router_lo)
        self.router_bias = None if inputs.get("router_bias") is None else \
            inputs["router_bias"].to(dev, torch.float32).contiguous()
        self.scales = {}
        self.mats = {}
        for name in ("w_gu", "w_d", "ws_gu", "ws_d"):
            t = inputs.get(name)
            if t is None:
                self.mats[name] = None
                self.scales[name] = None
                continue
            t = t.to(dev, torch.bfloat16).contiguous()
            if cfg.wdtype == WDTYPE_FP8_BLOCK128:
                q = torch.empty(t.shape, dtype=torch.uint8, device=dev)
                s = torch.empty(t.shape[:-2] + (t.shape[-2] // 128, t.shape[-1] // 128),
                                dtype=torch.float32, device=dev)
                quantize_weights_fp8(t.view(torch.uint16), q, s)
                self.mats[name], self.scales[name] = q, s
            elif cfg.wdtype == WDTYPE_FP8_TENSOR:
                q = torch.empty(t.shape, dtype=torch.uint8, device=dev)
                s = torch.empty(t.shape[:-2] if t.dim() > 2 else (1,), dtype=torch.float32, device=dev)
                quantize_weights_fp8_tensor(t.view(torch.uint16), q, s)
                self.mats[name], self.scales[name] = q, s
            elif cfg.wdtype == WDTYPE_MXFP8:
                q = torch.empty(t.shape, dtype=torch.uint8, device=dev)
                s = torch.empty(t.shape[:-1] + (t.shape[-1] // 32,), dtype=torch.uint8, device=dev)
                quantize_weights_mxfp8(t.view(torch.uint16), q, s)
                self.mats[name], self.scales[name] = q, s
            else:
                self.mats[name], self.scales[name] = t.view(torch.uint16), None
        self.act_scales = (1.0, 1.0)
        if cfg.wdtype == WDTYPE_FP8_TENSOR:
            self.act_scales = (tuple(act_scales) if act_scales is not None
                               else self._calibrate_static_scales(cfg, inputs, dev))
        self.weights = moe_weights(*[_p(v) for v in (
            self.mats["w_gu"], self.mats["w_d"], self.scales["w_gu"], self.scales["w_d"],
            self.mats["ws_gu"], self.mats["ws_d"], self.scales["ws_gu"], self.scales["ws_d"],
            self.router_hi, self.router_lo, self.router_bias)], *self.act_scales)
        nbytes = workspace_bytes(shape_of(cfg, self.max_tokens))
        if nbytes == 0:
            raise MoEError(UNSUPPORTED, "moe_workspace_bytes")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    CALIBRATION_TOKENS = 64

    def _calibrate_static_scales(self, cfg: MoEConfig, inputs: dict, dev):
        """Static activation scales of the per-tensor FP8 layer, calibrated by
        moe_calibrate_fp8_static on the first CALIBRATION_TOKENS tokens of the
        input with the BF16 weights; the two device floats are copied to the
        host, where moe_weights carries them."""
        x = inputs["x"][: self.CALIBRATION_TOKENS].to(dev, torch.bfloat16).contiguous()
        bf = {n: (None if inputs.get(n) is None else inputs[n].to(dev, torch.bfloat16).contiguous())
              for n in ("w_gu", "w_d", "ws_gu", "ws_d")}
        w16 = moe_weights(_p(bf["w_gu"]), _p(bf["w_d"]), None, None, _p(bf["ws_gu"]), _p(bf["ws_d"]),
                          None, None, _p(self.router_hi), _p(self.router_lo), _p(self.router_bias),
                          1.0, 1.0)
        shape16 = moe_shape(x.shape[0], cfg.d, cfg.E, cfg.k, cfg.I, cfg.Is, WDTYPE_BF16,
                            int(cfg.renorm))
        ws = torch.empty(workspace_bytes(shape16), dtype=torch.uint8, device=dev)
        scales = torch.empty(2, dtype=torch.float32, device=dev)
        calibrate_fp8_static(shape16, w16, x.view(torch.uint16), scales, ws)
        sx, sh = scales.cpu().tolist()
        return (sx, sh)

    def shape(self, T: int) -> moe_shape:
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds the layer's max_tokens={self.max_tokens}")
        return shape_of(self.cfg, T)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        if y is None:
            y = torch.empty_like(x)
        forward(self.shape(x.shape[0]), self.weights, x.view(torch.uint16), y.view(torch.uint16),
                self.ws, stream)
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None) -> torch.Tensor:
        forward_host(self.shape(x_host.shape[0]), self.weights, x_host.view(torch.uint16),
                     y_host.view(torch.uint16), self.ws, stream)
        return y_host

    def forward_host_async(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None,
                           ws: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Enqueue only (no synchronisation); `ws`: a workspace of this layer's
        size for a second stream in flight (default: the layer's own)."""
        forward_host_async(self.shape(x_host.shape[0]), self.weights, x_host.view(torch.uint16),
                           y_host.view(torch.uint16), self.ws if ws is None else ws, stream)
        return y_host

    def device_status(self, stream=None) -> int:
        return read_device_status(self.ws, stream)
