"""GPU parity of each stage entry point of the C ABI against the oracle, on
seeded synthetic inputs at sizes the oracle finishes in seconds (several
tiles, ragged tails).

Tolerances (derived from the arithmetic):
  - router split, top-k ids, counts / offsets / perm / inv, FP8 codes: exact;
  - router logits: |g - o| <= 1e-5 * max(|o|, rms(row)) (FP32 accumulation of
    exact bf16 products against the FP64 sum);
  - top-k weights: 2e-6 absolute (FP32 exp and division of values <= 1);
  - bf16 outputs of one FP32-accumulated GEMM or sum: one bf16 rounding
    (8 significant bits: at most 2^-8 relative, reached just above a power of
    two) plus FP32 noise (~1e-6 relative, inside the atol): rtol 2^-8,
    atol 1e-3 * rms(ref).
"""
import numpy as np
import pytest
import torch

import oracle
from expert_layer_dual_b200.configs import MoEConfig
from expert_layer_dual_b200.inputs import (make_layer, random_bf16, random_ids, random_logits,
                                           random_weights)
from gpu_util import O_RTOL, assert_close_rel, bf16_to_f64, bits, logit_rel_error, oracle_layer, rms

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import expert_layer_dual_b200.moe as M

DEV = "cuda"

SMALL = [
    MoEConfig("tiny", T=16, d=256, E=8, k=2, I=128, Is=0, seed=0),
    MoEConfig("ragged", T=300, d=512, E=16, k=4, I=256, Is=256, seed=21),
    MoEConfig("odd", T=203, d=384, E=40, k=8, I=128, Is=128, seed=22),
    MoEConfig("wide", T=130, d=256, E=256, k=8, I=128, Is=128, seed=23),
    # >= 256 rows per expert on average: the down GEMM runs on CTA pairs
    MoEConfig("pair", T=1100, d=512, E=8, k=4, I=256, Is=256, seed=27),
    MoEConfig("pairodd", T=1100, d=384, E=6, k=3, I=128, Is=128, seed=28),
]
IDS = [c.name for c in SMALL]


def _u16(t):
    return t.view(torch.uint16)


@pytest.mark.parametrize("n", [1, 1000, 256 * 4096 + 3])
def test_router_split_bit_exact(n):
    g = torch.Generator().manual_seed(n)
    W = torch.randn(n, generator=g) * torch.exp2(torch.randint(-20, 20, (n,), generator=g).float())
    hi = torch.empty(n, dtype=torch.uint16, device=DEV)
    lo = torch.empty(n, dtype=torch.uint16, device=DEV)
    M.router_split(W.to(DEV), hi, lo)
    ohi, olo = oracle.router_split(W.numpy())
    assert np.array_equal(bits(hi), ohi) and np.array_equal(bits(lo), olo)


@pytest.mark.parametrize("cfg", SMALL + [MoEConfig("d4096", T=257, d=4096, E=256, k=8, I=128, seed=24)],
                         ids=IDS + ["d4096"])
def test_router_logits(cfg):
    inp = make_layer(cfg)
    W = inp["router_w"]
    hi = torch.empty(W.shape, dtype=torch.uint16, device=DEV)
    lo = torch.empty_like(hi)
    M.router_split(W.to(DEV), hi, lo)
    bias = torch.randn(cfg.E, generator=torch.Generator().manual_seed(5)) if cfg.T % 2 else None
    x = inp["x"].to(DEV)
    logits = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=DEV)
    M.router_logits(_u16(x), hi, lo, None if bias is None else bias.to(DEV), logits)
    ref = oracle.router_logits(bits(inp["x"]), bits(hi), bits(lo), None if bias is None else bias.numpy())
    rel = logit_rel_error(logits.cpu().double().numpy(), ref)
    assert rel.max() <= 1e-5, f"max relative logit error {rel.max():.3g}"


@pytest.mark.parametrize("T,E,k,renorm", [(16, 8, 2, 1), (999, 256, 8, 1), (77, 40, 8, 1),
                                          (64, 256, 8, 0), (5, 3, 3, 1), (33, 256, 1, 1)])
def test_route_topk(T, E, k, renorm):
    l = random_logits(T, E, seed=T * 7 + E)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    M.route_topk(l.to(DEV), k, renorm, ids, w)
    oids, ow = oracle.route_topk(l.numpy(), k, renorm=bool(renorm))
    assert np.array_equal(ids.cpu().numpy(), oids)
    assert np.max(np.abs(w.cpu().double().numpy() - ow)) <= 2e-6


def test_route_topk_all_equal_logits():
    T, E, k = 40, 256, 8
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    M.route_topk(torch.zeros((T, E), device=DEV), k, 1, ids, w)
    assert np.array_equal(ids.cpu().numpy(), np.tile(np.arange(k), (T, 1)))
    assert torch.all(w == 1.0 / k)


@pytest.mark.parametrize("T,E,k", [(16, 8, 2), (4097, 256, 8), (300, 16, 4), (1, 1, 1), (16384, 256, 8)])
def test_permute_bit_exact(T, E, k):
    ids = random_ids(T, E, k, seed=T + E)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    ws = torch.empty(M.permute_workspace_bytes(T, E, k), dtype=torch.uint8, device=DEV)
    M.permute(ids.to(DEV), E, counts, offsets, perm, inv, ws)
    oc, oo, op, oi = oracle.permute(ids.numpy(), E)
    for g, o in ((counts, oc), (offsets, oo), (perm, op), (inv, oi)):
        assert np.array_equal(g.cpu().numpy(), o)
    assert M.read_device_status(ws) == M.OK


def test_permute_skewed_and_empty_experts():
    T, E, k = 2000, 256, 8
    g = torch.Generator().manual_seed(3)
    hot = torch.randperm(E, generator=g)[:12]          # only 12 experts receive tokens
    ids = torch.stack([hot[torch.randperm(12, generator=g)[:k]] for _ in range(T)]).to(torch.int32)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    ws = torch.empty(M.permute_workspace_bytes(T, E, k), dtype=torch.uint8, device=DEV)
    M.permute(ids.to(DEV), E, counts, offsets, perm, inv, ws)
    oc, oo, op, oi = oracle.permute(ids.numpy(), E)
    assert np.array_equal(perm.cpu().numpy(), op) and np.array_equal(offsets.cpu().numpy(), oo)
    assert (oc == 0).sum() == E - 12


def _gpu_permute(ids_dev, E):
    T, k = ids_dev.shape
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    ws = torch.empty(M.permute_workspace_bytes(T, E, k), dtype=torch.uint8, device=DEV)
    M.permute(ids_dev, E, counts, offsets, perm, inv, ws)
    return counts, offsets, perm, inv


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_gemm_gateup_bf16(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 100)
    _, offsets, perm, _ = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    h = torch.empty((R, cfg.I), dtype=torch.bfloat16, device=DEV)
    M.gemm_gateup(layer.shape(cfg.T), layer.weights, _u16(inp["x"].to(DEV)), None, perm, offsets,
                  _u16(h), None, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, operm, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.gateup(oracle_layer(cfg, inp), bits(inp["x"]), operm, ooff)
    assert_close_rel(bf16_to_f64(h), ref, rtol=2.0 ** -8, atol=1e-3 * rms(ref), what="h")


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_gemm_down_bf16(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 200)
    _, offsets, _, _ = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    hin = random_bf16((R, cfg.I), seed=cfg.seed, idx=1, std=0.5)
    o = torch.empty((R, cfg.d), dtype=torch.float16, device=DEV)
    M.gemm_down(layer.shape(cfg.T), layer.weights, _u16(hin.to(DEV)), None, offsets, o, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, _, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.down(oracle_layer(cfg, inp), bf16_to_f64(hin), ooff, cfg.T)
    # FP16 rows: the tensor core's FP32 accumulation over I terms, one FP16 rounding
    assert_close_rel(o.cpu().double().numpy(), ref, rtol=O_RTOL, atol=1e-4 * rms(ref), what="o")


def test_gemm_down_saturates_fp16_rows():
    """Sums past the FP16 range are stored as +-65504 (never inf); the rest as usual."""
    cfg = SMALL[0]
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 210)
    _, offsets, _, _ = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    hin = random_bf16((R, cfg.I), seed=cfg.seed, idx=12, std=2.0e6)
    o = torch.empty((R, cfg.d), dtype=torch.float16, device=DEV)
    M.gemm_down(layer.shape(cfg.T), layer.weights, _u16(hin.to(DEV)), None, offsets, o, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, _, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.down(oracle_layer(cfg, inp), bf16_to_f64(hin), ooff, cfg.T)
    got = o.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    big = np.abs(ref) > 65504.0 * (1 + 1e-3)
    assert big.mean() > 0.1 and (~big).mean() > 0.01          # both regimes are exercised
    assert np.array_equal(got[big], np.sign(ref[big]) * 65504.0)
    small = np.abs(ref) < 65504.0 * (1 - 1e-3)
    assert_close_rel(got[small], ref[small], rtol=O_RTOL, atol=1e-4 * rms(ref), what="o")


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_combine(cfg):
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 300)
    _, _, _, inv = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    o = torch.randn((R, cfg.d), generator=torch.Generator().manual_seed(cfg.seed)).half()
    w = random_weights(cfg.T, cfg.k, seed=cfg.seed)
    y = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=DEV)
    M.combine(M.shape_of(cfg), o.to(DEV), inv, w.to(DEV), _u16(y))
    _, _, _, oinv = oracle.permute(ids.numpy(), cfg.E)
    L = oracle_layer(cfg, {"router_w": torch.zeros(1), "w_gu": torch.zeros(1, dtype=torch.bfloat16),
                           "w_d": torch.zeros(1, dtype=torch.bfloat16)})
    ref = oracle.combine(L, o.double().numpy(), oinv, w.double().numpy(), cfg.T)
    assert_close_rel(bf16_to_f64(y), ref, rtol=2.0 ** -8, atol=1e-5 * rms(ref), what="y")


@pytest.mark.parametrize("rows,cols", [(1, 128), (300, 512), (4096, 6144)])
def test_quantize_act_fp8_bit_exact(rows, cols):
    x = random_bf16((rows, cols), seed=rows, idx=3, std=3.0)
    x[0, :128] = 0                                             # an all-zero group
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    s = torch.empty((rows, cols // 128), dtype=torch.float32, device=DEV)
    M.quantize_act_fp8(_u16(x.to(DEV)), q, s)
    oq, os_ = oracle.quant_fp8_rows(x.float().numpy())
    assert np.array_equal(q.cpu().numpy(), oq) and np.array_equal(s.cpu().numpy(), os_)


@pytest.mark.parametrize("batch,rows,cols", [(1, 128, 128), (3, 256, 384), (2, 4096, 1024)])
def test_quantize_weights_fp8_bit_exact(batch, rows, cols):
    W = random_bf16((batch, rows, cols), seed=rows + cols, idx=4, std=0.02)
    q = torch.empty(W.shape, dtype=torch.uint8, device=DEV)
    s = torch.empty((batch, rows // 128, cols // 128), dtype=torch.float32, device=DEV)
    M.quantize_weights_fp8(_u16(W.to(DEV)), q, s)
    oq, os_ = oracle.quant_fp8_blocks(bits(W))
    assert np.array_equal(q.cpu().numpy(), oq) and np.array_equal(s.cpu().numpy(), os_)


# ---------------------------------------------------------------- FP8 path
FP8 = [
    MoEConfig("fp8small", T=200, d=512, E=16, k=4, I=256, Is=256, wdtype=1, seed=31),
    MoEConfig("fp8odd", T=77, d=384, E=8, k=2, I=128, Is=0, wdtype=1, seed=32),
]
FP8_IDS = [c.name for c in FP8]


def _permuted_quant(x_dev, perm, cfg):
    R = cfg.rows()
    q = torch.empty((R, cfg.d), dtype=torch.uint8, device=DEV)
    s = torch.empty((R, cfg.d // 128), dtype=torch.float32, device=DEV)
    M.quantize_act_fp8_permuted(_u16(x_dev), perm, cfg.k, cfg.Is > 0, q, s)
    return q, s


@pytest.mark.parametrize("cfg", FP8, ids=FP8_IDS)
def test_quantize_act_fp8_permuted_bit_exact(cfg):
    x = make_layer(cfg)["x"]
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 400)
    _, _, perm, _ = _gpu_permute(ids.to(DEV), cfg.E)
    q, s = _permuted_quant(x.to(DEV), perm, cfg)
    _, _, operm, _ = oracle.permute(ids.numpy(), cfg.E)
    tok = np.concatenate([operm // cfg.k, np.arange(cfg.T) if cfg.Is else np.zeros(0, np.int64)])
    oq, os_ = oracle.quant_fp8_rows(x.float().numpy()[tok])
    assert np.array_equal(q.cpu().numpy(), oq) and np.array_equal(s.cpu().numpy(), os_)


@pytest.mark.parametrize("cfg", FP8, ids=FP8_IDS)
def test_weights_fp8_match_oracle_quantisation(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    q, s = oracle.quant_fp8_blocks(bits(inp["w_gu"]))
    assert np.array_equal(layer.mats["w_gu"].cpu().numpy(), q)
    assert np.array_equal(layer.scales["w_gu"].cpu().numpy(), s)


@pytest.mark.parametrize("cfg", FP8, ids=FP8_IDS)
def test_gemm_gateup_fp8(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 100)
    _, offsets, perm, _ = _gpu_permute(ids.to(DEV), cfg.E)
    xq, xs = _permuted_quant(inp["x"].to(DEV), perm, cfg)
    R = cfg.rows()
    hq = torch.empty((R, cfg.I), dtype=torch.uint8, device=DEV)
    hs = torch.empty((R, cfg.I // 128), dtype=torch.float32, device=DEV)
    M.gemm_gateup(layer.shape(cfg.T), layer.weights, xq, xs, None, offsets, hq, hs, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, operm, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.gateup(oracle_layer(cfg, inp), bits(inp["x"]), operm, ooff)   # FP64 h, pre-quantisation
    gq, gs = hq.cpu().numpy(), hs.cpu().numpy()
    deq = oracle.e4m3_decode(gq) * np.repeat(gs.astype(np.float64), 128, axis=1)
    sfull = np.repeat(gs.astype(np.float64), 128, axis=1)
    # one e4m3 rounding of the row group (relative 2^-4, or 2^-10 s near zero) plus FP32 noise
    bound = 2.0 ** -4 * np.abs(ref) + 2.0 ** -10 * sfull + 1e-5 * rms(ref)
    assert np.all(np.abs(deq - ref) <= bound * (1 + 1e-6))
    # codes and scales against the oracle's own quantisation of its h
    oq, os_ = oracle.quant_fp8_rows(ref.astype(np.float32))
    assert np.mean(gq == oq) >= 0.99
    np.testing.assert_allclose(gs, os_, rtol=1e-5)


@pytest.mark.parametrize("cfg", FP8, ids=FP8_IDS)
def test_gemm_down_fp8(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 200)
    _, offsets, _, _ = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    hin = random_bf16((R, cfg.I), seed=cfg.seed, idx=5, std=0.5)
    hq = torch.empty((R, cfg.I), dtype=torch.uint8, device=DEV)
    hs = torch.empty((R, cfg.I // 128), dtype=torch.float32, device=DEV)
    M.quantize_act_fp8(_u16(hin.to(DEV)), hq, hs)
    o = torch.empty((R, cfg.d), dtype=torch.float16, device=DEV)
    M.gemm_down(layer.shape(cfg.T), layer.weights, hq, hs, offsets, o, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, _, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.down(oracle_layer(cfg, inp), bf16_to_f64(hin), ooff, cfg.T)
    assert_close_rel(o.cpu().double().numpy(), ref, rtol=O_RTOL, atol=1e-4 * rms(ref), what="o")
