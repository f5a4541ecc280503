"""Pins of the oracle's expert FFN stages and whole-layer forward.

y = sum_k w_k * E_{e_k}(x) + S(x) with SiLU-gated experts.  Sources:
"HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的主要功能
(FusedMoE: Gate-Up GEMM, activation quantisation, Down GEMM, Top-K weighted
aggregation) and "PR #54160 完整报告", section 功能与动机 (routed experts plus
one shared expert)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from expert_layer_dual_b200.configs import MoEConfig
from expert_layer_dual_b200.inputs import make_layer


def _np_bits(t):
    return None if t is None else t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _layer(cfg, inp, wdtype=0):
    return oracle.Layer(
        T=cfg.T, d=cfg.d, E=cfg.E, k=cfg.k, I=cfg.I, Is=cfg.Is,
        w_gu=_np_bits(inp["w_gu"]), w_d=_np_bits(inp["w_d"]),
        ws_gu=_np_bits(inp["ws_gu"]), ws_d=_np_bits(inp["ws_d"]),
        router_w=inp["router_w"].numpy(),
        router_bias=None if inp["router_bias"] is None else inp["router_bias"].numpy(),
        wdtype=wdtype)


def _swiglu(x, wgu, wd):
    """Textbook SiLU-gated FFN in float64 torch: (silu(x Wg^T) * (x Wu^T)) Wd^T."""
    I = wd.shape[1]
    return (F.silu(x @ wgu[:I].T) * (x @ wgu[I:].T)) @ wd.T


def _f64(t):
    return t.to(torch.float64)


def test_single_expert_is_a_dense_swiglu_ffn():
    cfg = MoEConfig("one", T=13, d=256, E=1, k=1, I=128, Is=0, seed=7)
    inp = make_layer(cfg)
    r = oracle.forward(_layer(cfg, inp), _np_bits(inp["x"]))
    assert np.all(r["ids"] == 0) and np.all(r["w"] == 1.0)
    ref = _swiglu(_f64(inp["x"]), _f64(inp["w_gu"][0]), _f64(inp["w_d"][0])).numpy()
    np.testing.assert_allclose(r["y"], ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


def test_identical_experts_make_routing_irrelevant():
    cfg = MoEConfig("same", T=21, d=256, E=6, k=3, I=128, Is=128, seed=8)
    inp = make_layer(cfg)
    inp["w_gu"][:] = inp["w_gu"][0]
    inp["w_d"][:] = inp["w_d"][0]
    r = oracle.forward(_layer(cfg, inp), _np_bits(inp["x"]))
    x = _f64(inp["x"])
    ref = (_swiglu(x, _f64(inp["w_gu"][0]), _f64(inp["w_d"][0])) +
           _swiglu(x, _f64(inp["ws_gu"]), _f64(inp["ws_d"]))).numpy()
    np.testing.assert_allclose(r["y"], ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


@pytest.mark.parametrize("shared", [0, 128])
def test_forward_equals_per_token_evaluation(shared):
    cfg = MoEConfig("bf", T=40, d=256, E=8, k=3, I=128, Is=shared, seed=9)
    inp = make_layer(cfg)
    r = oracle.forward(_layer(cfg, inp), _np_bits(inp["x"]))
    x = _f64(inp["x"])
    for t in range(cfg.T):
        y = torch.zeros(cfg.d, dtype=torch.float64)
        for j in range(cfg.k):
            e = int(r["ids"][t, j])
            y += float(r["w"][t, j]) * _swiglu(x[t:t + 1], _f64(inp["w_gu"][e]), _f64(inp["w_d"][e]))[0]
        if shared:
            y += _swiglu(x[t:t + 1], _f64(inp["ws_gu"]), _f64(inp["ws_d"]))[0]
        np.testing.assert_allclose(r["y"][t], y.numpy(), rtol=1e-11, atol=1e-12)
    # routing inside the forward is the top-k of the router logits' FP32 rounding
    ids, _ = oracle.route_topk(r["logits"].astype(np.float32), cfg.k)
    assert np.array_equal(ids, r["ids"])


def _grid_matrix(rng, rows, cols, group_rows):
    """bf16 bits of a matrix whose every (group_rows x 128) block is e4m3 values
    times its own power of two, with the block maximum at 448 * 2^n."""
    out = np.zeros((rows, cols))
    for i in range(0, rows, group_rows):
        for j in range(0, cols, 128):
            codes = rng.integers(0, 256, group_rows * 128).astype(np.uint8)
            codes[(codes & 0x7F) == 0x7F] = 0x7E
            v = oracle.e4m3_decode(codes)
            v[rng.integers(v.size)] = 448.0
            out[i:i + group_rows, j:j + 128] = v.reshape(group_rows, 128) * 2.0 ** int(rng.integers(-14, -8))
    return oracle.bf16_round(out)


def test_fp8_stages_equal_bf16_stages_on_grid_values():
    # Weights and activations that block/group quantisation reproduces exactly:
    # the FP8 path must then equal the BF16 path (pins every scale index).
    rng = np.random.default_rng(10)
    T, d, E, k, I = 12, 256, 3, 2, 256
    w_gu = np.stack([_grid_matrix(rng, 2 * I, d, 128) for _ in range(E)])
    w_d = np.stack([_grid_matrix(rng, d, I, 128) for _ in range(E)])
    ws_gu, ws_d = _grid_matrix(rng, 2 * I, d, 128), _grid_matrix(rng, d, I, 128)
    x = _grid_matrix(rng, T, d, 1)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    layers = [oracle.Layer(T=T, d=d, E=E, k=k, I=I, Is=I, w_gu=w_gu, w_d=w_d, ws_gu=ws_gu,
                           ws_d=ws_d, router_w=np.zeros((E, d), np.float32), wdtype=wd)
              for wd in (0, 1)]
    h0 = oracle.gateup(layers[0], x, perm, offsets)
    h1 = oracle.gateup(layers[1], x, perm, offsets)
    np.testing.assert_allclose(h1, h0, rtol=1e-13, atol=0)
    hg = oracle.bf16_decode(_grid_matrix(rng, T * k + T, I, 1))
    o0 = oracle.down(layers[0], hg, offsets, T)
    o1 = oracle.down(layers[1], hg, offsets, T)
    np.testing.assert_allclose(o1, o0, rtol=1e-13, atol=0)
    # and off the grid the FP8 path does differ (the quantisation is really applied)
    hn = rng.standard_normal((T * k + T, I))
    assert np.max(np.abs(oracle.down(layers[1], hn, offsets, T) - oracle.down(layers[0], hn, offsets, T))) > 0


def test_combine_weights_and_shared_row():
    cfg = MoEConfig("c", T=3, d=128, E=4, k=2, I=128, Is=128)
    L = oracle.Layer(T=3, d=128, E=4, k=2, I=128, Is=128, w_gu=np.zeros((4, 256, 128), np.uint16),
                     w_d=np.zeros((4, 128, 128), np.uint16), router_w=np.zeros((4, 128), np.float32))
    rng = np.random.default_rng(11)
    o = rng.standard_normal((cfg.rows(), 128))
    ids = np.array([[0, 2], [3, 0], [1, 2]], np.int32)
    _, _, perm, inv = oracle.permute(ids, 4)
    w = rng.random((3, 2))
    y = oracle.combine(L, o, inv, w, 3)
    for t in range(3):
        ref = w[t, 0] * o[inv[2 * t]] + w[t, 1] * o[inv[2 * t + 1]] + o[6 + t]
        np.testing.assert_allclose(y[t], ref, rtol=1e-15)
