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


# ------------------------------------------------------------------ layer parity
def oracle_routed(L: oracle.Layer, x: np.ndarray, ids: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The oracle's layer output on a GIVEN routing (ids [T, k], weights w
    [T, k] FP64): its own permute, gate-up, down and combine on the tokens of
    x (bf16 bits [T, d]).  The layer's expert ids must index L.w_gu / L.w_d."""
    T = x.shape[0]
    _, offsets, perm, inv = oracle.permute(ids, L.E)
    h = oracle.gateup(L, x, perm, offsets)
    o = oracle.down(L, h, offsets, T)
    return oracle.combine(L, o, inv, w, T)


def oracle_routed_sampled(cfg: MoEConfig, inp: dict, x_rows: np.ndarray, ids: np.ndarray,
                          w: np.ndarray, act=(1.0, 1.0), chunk: int = 8) -> np.ndarray:
    """oracle_routed for a sample of tokens of a full-size layer whose weights
    live on the GPU: in chunks of `chunk` tokens, the experts the chunk's
    routing selects are copied to the host and renumbered 0..n-1 (in
    ascending id order), so the oracle sees a compact layer holding only
    them.  Every expert's FFN is evaluated independently, so renumbering
    changes nothing in the arithmetic."""
    out = np.empty((x_rows.shape[0], cfg.d), np.float64)
    for c0 in range(0, x_rows.shape[0], chunk):
        sl = slice(c0, min(c0 + chunk, x_rows.shape[0]))
        need = np.unique(ids[sl])
        remap = {int(e): i for i, e in enumerate(need)}
        w_gu = np.stack([bits(inp["w_gu"][int(e)]) for e in need])
        w_d = np.stack([bits(inp["w_d"][int(e)]) for e in need])
        L = oracle.Layer(T=sl.stop - sl.start, d=cfg.d, E=len(need), k=cfg.k, I=cfg.I, Is=cfg.Is,
                         w_gu=w_gu, w_d=w_d,
                         ws_gu=None if inp.get("ws_gu") is None else bits(inp["ws_gu"]),
                         ws_d=None if inp.get("ws_d") is None else bits(inp["ws_d"]),
                         router_w=np.zeros((len(need), cfg.d), np.float32), wdtype=cfg.wdtype,
                         renorm=cfg.renorm, act_sx=act[0], act_sh=act[1])
        ids_c = np.vectorize(remap.get)(ids[sl]).astype(np.int32)
        out[sl] = oracle_routed(L, x_rows[sl], ids_c, w[sl])
        del w_gu, w_d, L
    return out


def bf16_allowance(y64: np.ndarray) -> np.ndarray:
    """2^-8 |y|: at least half a bf16 ulp of any value within a small
    distance of y (half an ulp of v is 2^(e-8) <= 2^-8 |v| for 2^e <= |v|)."""
    return 2.0 ** -8 * np.abs(y64)


def layer_errors(y: np.ndarray, y64: np.ndarray) -> dict:
    """Error measures of a layer output y (bf16 values as FP64) against the
    oracle's FP64 y64, in units of rms(y64):
      raw   max |y - y64|
      comp  max (|y - y64| - 2^-8 |y64|): the error left once the output's own
            bf16 rounding is allowed for (the computation before that rounding)
      floor max |RNE_bf16(y64) - y64|: the error of the correctly rounded bf16
            output, which no bf16 result can beat."""
    s = rms(y64)
    err = np.abs(y - y64)
    rounded = oracle.bf16_decode(oracle.bf16_round(y64))
    return {"raw": float(err.max() / s), "comp": float((err - bf16_allowance(y64)).max() / s),
            "floor": float(np.abs(rounded - y64).max() / s), "rms": s}


def report(record: dict) -> None:
    """Append one JSON line to $MOE_PARITY_REPORT (when set): the measured
    error distribution the design notes quote."""
    import json
    import os
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(record) + "\n")


def pick_tokens(offsets: np.ndarray, perm: np.ndarray, k: int, T: int, n: int,
                seed: int = 99) -> np.ndarray:
    """About n distinct tokens of a routed batch (all of them when T <= n),
    chosen to reach the grouped GEMMs' edge rows: the largest expert's first
    and last rows and the rows on both sides of each of its first four
    128-row tile boundaries, the last row of other experts (a partly filled
    last tile), then random tokens.  Sorted."""
    if T <= n:
        return np.arange(T)
    counts = np.diff(offsets)
    big = int(np.argmax(counts))
    lo, hi = int(offsets[big]), int(offsets[big + 1])
    rows = {lo, hi - 1}
    for b in range(1, 5):
        rows |= {r for r in (lo + 128 * b - 1, lo + 128 * b) if r < hi}
    rng = np.random.default_rng(seed)
    live = np.nonzero(counts)[0]
    rows |= {int(offsets[e + 1]) - 1 for e in rng.choice(live, min(len(live), n // 4), replace=False)}
    pick = {int(perm[r]) // k for r in rows}
    for t in rng.permutation(T):
        if len(pick) >= n:
            break
        pick.add(int(t))
    return np.array(sorted(pick))
