"""Helpers of the GPU parity tests: move seeded inputs between the CUDA path
(through the C-ABI binding) and the oracle (host numpy), and compare.

Nothing here computes the layer: the CUDA side calls the library, the
expected side calls ``oracle``."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from expert_layer_dual_b200.configs import MoEConfig


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 / uint16 tensor -> numpy uint16 bit patterns on the host."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    elif t.dtype == torch.uint16:
        t = t.view(torch.int16)
    return t.numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def oracle_layer(cfg: MoEConfig, inp: dict, T: int = None, act=(1.0, 1.0)) -> oracle.Layer:
    """`act`: the static activation scales of a per-tensor FP8 layer (the GPU
    layer's calibrated MoELayer.act_scales)."""
    def host(name):
        t = inp.get(name)
        return None if t is None else bits(t)
    return oracle.Layer(
        T=cfg.T if T is None else T, d=cfg.d, E=cfg.E, k=cfg.k, I=cfg.I, Is=cfg.Is,
        w_gu=host("w_gu"), w_d=host("w_d"), ws_gu=host("ws_gu"), ws_d=host("ws_d"),
        router_w=inp["router_w"].detach().cpu().numpy(),
        router_bias=None if inp.get("router_bias") is None else inp["router_bias"].cpu().numpy(),
        wdtype=cfg.wdtype, renorm=cfg.renorm, act_sx=act[0], act_sh=act[1])


def rms(a: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.square(a, dtype=np.float64))))


# Expert-output rows o are stored FP16 (round to nearest even): one rounding
# of at most 2^-11 relative on top of the FP32 accumulation (1e-4).
O_RTOL = 2.0 ** -11 + 1e-4


def assert_close_rel(got, ref, rtol, atol, what=""):
    """|got - ref| <= atol + rtol * |ref| elementwise, with a useful message."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} (atol {atol:.3g}, rtol {rtol:.3g})")


def row_scale(logits64: np.ndarray) -> np.ndarray:
    """Per-row logit scale: rms over the entries that can be selected (a
    masking bias of -1e4 on some experts would otherwise dominate it)."""
    med = np.median(np.abs(logits64), axis=1, keepdims=True)
    live = np.abs(logits64) <= 100.0 * np.maximum(med, 1e-30)
    sq = np.where(live, logits64 ** 2, 0.0)
    return np.sqrt(sq.sum(axis=1, keepdims=True) / np.maximum(live.sum(axis=1, keepdims=True), 1))


def logit_rel_error(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """|g - o| / max(|o|, row scale): the router-logit error measure."""
    return np.abs(got - ref) / np.maximum(np.abs(ref), row_scale(ref))


def ambiguous_tokens(logits64: np.ndarray, k: int, rel: float = 1e-4) -> np.ndarray:
    """Tokens whose top-(k+1) oracle logits contain two values closer than
    rel * the row scale: there the FP32 kernel and the FP64 oracle may
    legitimately order or select differently (both are correct within the
    logits tolerance), so only validity is checked for them."""
    s = -np.sort(-logits64, axis=1)[:, : min(k + 1, logits64.shape[1])]
    gaps = -np.diff(s, axis=1)
    return np.any(gaps < rel * np.maximum(row_scale(logits64), 1e-30), axis=1)
