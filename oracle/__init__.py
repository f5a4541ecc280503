"""Plain FP64 CPU oracle of the fused MoE layer forward (ctypes wrapper).

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test suite,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg
may import this package.  It shares no code with the CUDA library in
``expert_layer_dual_b200``; neither imports the other.  The arithmetic lives
in ``moe_oracle.c`` (sources and readings in ``moe_oracle.h``); this module
only builds it with gcc and marshals numpy arrays.

Every function takes and returns host numpy arrays.  BF16 values travel as
``uint16`` bit patterns, FP8 e4m3 values as ``uint8`` codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_HDR = os.path.join(_HERE, "moe_oracle.h")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no fast-math) if it is stale."""
    stale = force or not os.path.exists(_LIB) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d", ctypes.c_int), ("E", ctypes.c_int),
                ("k", ctypes.c_int), ("I", ctypes.c_int), ("Is", ctypes.c_int),
                ("wdtype", ctypes.c_int), ("renorm", ctypes.c_int),
                ("w_gu", ctypes.c_void_p), ("w_d", ctypes.c_void_p),
                ("ws_gu", ctypes.c_void_p), ("ws_d", ctypes.c_void_p),
                ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("act_sx", ctypes.c_float), ("act_sh", ctypes.c_float)]


class _Out(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("logits", "ids", "w", "counts", "offsets", "perm", "inv", "y")]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.orc_bf16_decode.restype = ctypes.c_double
        L.orc_bf16_decode.argtypes = [ctypes.c_uint16]
        L.orc_bf16_round.restype = ctypes.c_uint16
        L.orc_bf16_round.argtypes = [ctypes.c_double]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_round.restype = ctypes.c_uint8
        L.orc_e4m3_round.argtypes = [ctypes.c_double]
        L.orc_bf16_round_array.argtypes = [vp, i64, vp]
        L.orc_router_split.argtypes = [vp, i64, vp, vp]
        L.orc_router_logits.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp]
        L.orc_route_topk.argtypes = [vp, i32, i32, i32, i32, vp, vp]
        L.orc_permute.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
        L.orc_quant_fp8_blocks.argtypes = [vp, i64, i32, i32, vp, vp]
        L.orc_quant_fp8_rows.argtypes = [vp, i64, i32, vp, vp]
        L.orc_e8m0_decode.restype = ctypes.c_double
        L.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.orc_mx_scale_byte.restype = ctypes.c_uint8
        L.orc_mx_scale_byte.argtypes = [ctypes.c_float]
        L.orc_quant_mx_rows.argtypes = [vp, i64, i32, vp, vp]
        L.orc_quant_mx_bf16.argtypes = [vp, i64, i32, i32, vp, vp]
        L.orc_quant_fp8_tensor.argtypes = [vp, i64, i32, i32, vp, vp]
        L.orc_quant_fp8_static.argtypes = [vp, i64, ctypes.c_float, vp]
        L.orc_gateup.argtypes = [ctypes.POINTER(_Layer), vp, vp, vp, vp]
        L.orc_down.argtypes = [ctypes.POINTER(_Layer), vp, vp, vp]
        L.orc_combine.argtypes = [ctypes.POINTER(_Layer), vp, vp, vp, vp]
        L.orc_forward.argtypes = [ctypes.POINTER(_Layer), vp, ctypes.POINTER(_Out)]
        L.orc_forward.restype = i32
        L.orc_num_threads.restype = i32
        L.orc_allreduce_rmsnorm.argtypes = [vp, i32, i32, i32, vp, vp, ctypes.c_double, vp, vp]
        _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ----------------------------------------------------------------- formats
def bf16_decode(bits: np.ndarray) -> np.ndarray:
    f = lib().orc_bf16_decode
    b = _c(bits, np.uint16)
    return np.array([f(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def bf16_round(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().orc_bf16_round_array(_p(v), v.size, _p(out))
    return out


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    f = lib().orc_e4m3_decode
    c = _c(codes, np.uint8)
    return np.array([f(int(v)) for v in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_round(v: np.ndarray) -> np.ndarray:
    f = lib().orc_e4m3_round
    v = _c(v, np.float64)
    return np.array([f(float(a)) for a in v.ravel()], dtype=np.uint8).reshape(v.shape)


# ----------------------------------------------------------------- stages
def router_split(W: np.ndarray):
    W = _c(W, np.float32)
    hi = np.empty(W.shape, np.uint16)
    lo = np.empty(W.shape, np.uint16)
    lib().orc_router_split(_p(W), W.size, _p(hi), _p(lo))
    return hi, lo


def router_logits(x, hi, lo, bias=None) -> np.ndarray:
    x, hi, lo = _c(x, np.uint16), _c(hi, np.uint16), _c(lo, np.uint16)
    T, d = x.shape
    E = hi.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), np.float64)
    lib().orc_router_logits(_p(x), _p(hi), _p(lo), _p(b), T, d, E, _p(out))
    return out


def route_topk(logits32: np.ndarray, k: int, renorm: bool = True):
    l = _c(logits32, np.float32)
    T, E = l.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().orc_route_topk(_p(l), T, E, k, int(renorm), _p(ids), _p(w))
    return ids, w


def permute(ids: np.ndarray, E: int):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    lib().orc_permute(_p(ids), T, E, k, _p(counts), _p(offsets), _p(perm), _p(inv))
    return counts, offsets, perm, inv


def quant_fp8_blocks(W: np.ndarray):
    """W: bf16 bits [..., rows, cols] -> (q uint8, s float32 [..., rows/128, cols/128])."""
    W = _c(W, np.uint16)
    rows, cols = W.shape[-2:]
    batch = int(np.prod(W.shape[:-2])) if W.ndim > 2 else 1
    q = np.empty(W.shape, np.uint8)
    s = np.empty(W.shape[:-2] + (rows // 128, cols // 128), np.float32)
    lib().orc_quant_fp8_blocks(_p(W), batch, rows, cols, _p(q), _p(s))
    return q, s


def quant_fp8_rows(v: np.ndarray):
    """v: float32 [rows, cols] -> (q uint8 [rows, cols], s float32 [rows, cols/128])."""
    v = _c(v, np.float32)
    rows, cols = v.shape
    q = np.empty(v.shape, np.uint8)
    s = np.empty((rows, cols // 128), np.float32)
    lib().orc_quant_fp8_rows(_p(v), rows, cols, _p(q), _p(s))
    return q, s


def quant_fp8_tensor(W: np.ndarray):
    """W: bf16 bits [..., rows, cols] -> (q uint8, s float32 [...]): one scale per matrix."""
    W = _c(W, np.uint16)
    rows, cols = W.shape[-2:]
    batch = int(np.prod(W.shape[:-2])) if W.ndim > 2 else 1
    q = np.empty(W.shape, np.uint8)
    s = np.empty(W.shape[:-2] if W.ndim > 2 else (1,), np.float32)
    lib().orc_quant_fp8_tensor(_p(W), batch, rows, cols, _p(q), _p(s))
    return q, s


def quant_fp8_static(v: np.ndarray, s: float) -> np.ndarray:
    """v: float32 array, static scale s -> e4m3 codes of fp32(v / s), saturating."""
    v = _c(v, np.float32)
    q = np.empty(v.shape, np.uint8)
    lib().orc_quant_fp8_static(_p(v), v.size, float(s), _p(q))
    return q


def e8m0_decode(b: int) -> float:
    return lib().orc_e8m0_decode(int(b))


def mx_scale_byte(amax: float) -> int:
    return int(lib().orc_mx_scale_byte(float(amax)))


def quant_mx_rows(v: np.ndarray):
    """v: float32 [rows, cols] -> (q uint8 [rows, cols], s uint8 E8M0 [rows, cols/32])."""
    v = _c(v, np.float32)
    rows, cols = v.shape
    q = np.empty(v.shape, np.uint8)
    s = np.empty((rows, cols // 32), np.uint8)
    lib().orc_quant_mx_rows(_p(v), rows, cols, _p(q), _p(s))
    return q, s


def quant_mx_bf16(W: np.ndarray):
    """W: bf16 bits [..., rows, cols] -> (q uint8, s uint8 E8M0 [..., rows, cols/32])."""
    W = _c(W, np.uint16)
    rows, cols = W.shape[-2:]
    batch = int(np.prod(W.shape[:-2])) if W.ndim > 2 else 1
    q = np.empty(W.shape, np.uint8)
    s = np.empty(W.shape[:-1] + (cols // 32,), np.uint8)
    lib().orc_quant_mx_bf16(_p(W), batch, rows, cols, _p(q), _p(s))
    return q, s


@dataclass
class Layer:
    """Host copy of one MoE layer's weights, as the oracle consumes them."""
    T: int
    d: int
    E: int
    k: int
    I: int
    Is: int
    w_gu: np.ndarray            # bf16 bits [E, 2I, d]
    w_d: np.ndarray             # bf16 bits [E, d, I]
    router_w: np.ndarray        # float32 [E, d]
    ws_gu: Optional[np.ndarray] = None   # bf16 bits [2Is, d]
    ws_d: Optional[np.ndarray] = None    # bf16 bits [d, Is]
    router_bias: Optional[np.ndarray] = None
    wdtype: int = 0             # 0 bf16, 1 fp8 e4m3 with 128x128 block scales, 2 mxfp8,
                                # 3 fp8 per tensor (static activation scales act_sx, act_sh)
    act_sx: float = 1.0
    act_sh: float = 1.0
    renorm: bool = True

    def _struct(self, T: Optional[int] = None):
        self._keep = [_c(self.w_gu, np.uint16), _c(self.w_d, np.uint16),
                      None if self.ws_gu is None else _c(self.ws_gu, np.uint16),
                      None if self.ws_d is None else _c(self.ws_d, np.uint16),
                      _c(self.router_w, np.float32),
                      None if self.router_bias is None else _c(self.router_bias, np.float32)]
        k = self._keep
        return _Layer(self.T if T is None else T, self.d, self.E, self.k, self.I,
                      self.Is, self.wdtype, int(self.renorm),
                      _p(k[0]), _p(k[1]), _p(k[2]), _p(k[3]), _p(k[4]), _p(k[5]),
                      float(self.act_sx), float(self.act_sh))

    def rows(self, T: Optional[int] = None) -> int:
        T = self.T if T is None else T
        return T * self.k + (T if self.Is > 0 else 0)


def gateup(L: Layer, x: np.ndarray, perm: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    x = _c(x, np.uint16)
    T = x.shape[0]
    st = L._struct(T)
    hs = max(L.I, L.Is)
    h = np.zeros((L.rows(T), hs), np.float64)
    perm, offsets = _c(perm, np.int32), _c(offsets, np.int32)
    lib().orc_gateup(ctypes.byref(st), _p(x), _p(perm), _p(offsets), _p(h))
    return h


def down(L: Layer, h: np.ndarray, offsets: np.ndarray, T: int) -> np.ndarray:
    st = L._struct(T)
    h = _c(h, np.float64)
    o = np.zeros((L.rows(T), L.d), np.float64)
    offsets = _c(offsets, np.int32)
    lib().orc_down(ctypes.byref(st), _p(h), _p(offsets), _p(o))
    return o


def combine(L: Layer, o: np.ndarray, inv: np.ndarray, w: np.ndarray, T: int) -> np.ndarray:
    st = L._struct(T)
    o, inv, w = _c(o, np.float64), _c(inv, np.int32), _c(w, np.float64)
    y = np.empty((T, L.d), np.float64)
    lib().orc_combine(ctypes.byref(st), _p(o), _p(inv), _p(w), _p(y))
    return y


def forward(L: Layer, x: np.ndarray) -> dict:
    """The whole layer on the tokens of x (bf16 bits [T, d]); returns every
    intermediate the oracle exposes plus y (float64 [T, d])."""
    x = _c(x, np.uint16)
    T = x.shape[0]
    st = L._struct(T)
    r = dict(logits=np.empty((T, L.E), np.float64), ids=np.empty((T, L.k), np.int32),
             w=np.empty((T, L.k), np.float64), counts=np.empty(L.E, np.int32),
             offsets=np.empty(L.E + 1, np.int32), perm=np.empty(T * L.k, np.int32),
             inv=np.empty(T * L.k, np.int32), y=np.empty((T, L.d), np.float64))
    out = _Out(*[_p(r[n]) for n in ("logits", "ids", "w", "counts", "offsets", "perm", "inv", "y")])
    rc = lib().orc_forward(ctypes.byref(st), _p(x), ctypes.byref(out))
    if rc != 0:
        raise MemoryError("oracle forward could not allocate its buffers")
    return r


def allreduce_rmsnorm(x: np.ndarray, residual: Optional[np.ndarray], gamma: np.ndarray,
                      eps: float):
    """x: bf16 bits [G, T, d]; residual: bf16 bits [T, d] or None; gamma: bf16
    bits [d] -> (res, out), both float64 [T, d]: the summed residual stream and
    its RMSNorm times gamma."""
    x = _c(x, np.uint16)
    G, T, d = x.shape
    r = None if residual is None else _c(residual, np.uint16)
    g = _c(gamma, np.uint16)
    res = np.empty((T, d), np.float64)
    out = np.empty((T, d), np.float64)
    lib().orc_allreduce_rmsnorm(_p(x), G, T, d, _p(r), _p(g), float(eps), _p(res), _p(out))
    return res, out
