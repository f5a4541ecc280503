"""GPU parity of the MXFP8 path (e4m3 with an E8M0 scale per 1x32 along K,
native block-scaled MMA) against the FP64 oracle: quantisation codes and
scales bit-exact, the grouped GEMMs within one e4m3 rounding of h (gate-up)
or FP32 accumulation noise (down).  The format is the MXFP8 weight format of
"PR #54160 完整报告", section 实现拆解 item 4."""
import numpy as np
import pytest
import torch

import oracle
from expert_layer_dual_b200.configs import MoEConfig
from expert_layer_dual_b200.inputs import make_layer, random_bf16, random_ids
from gpu_util import O_RTOL, assert_close_rel, bf16_to_f64, bits, oracle_layer, rms

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import expert_layer_dual_b200.moe as M

DEV = "cuda"

MX = [
    MoEConfig("mxsmall", T=200, d=512, E=16, k=4, I=256, Is=256, wdtype=2, seed=41),
    MoEConfig("mxodd", T=77, d=384, E=8, k=2, I=128, Is=0, wdtype=2, seed=42),
    MoEConfig("mxwide", T=300, d=1024, E=4, k=2, I=384, Is=384, wdtype=2, seed=43),
]
MX_IDS = [c.name for c in MX]


def _u16(t):
    return t.view(torch.uint16)


def _e8m0(b):
    return np.ldexp(1.0, b.astype(np.int64) - 127)


def _kbm_to_rows(s, rows, cols):
    """Activation scales, k-block-major [cols/128][rows][4] -> [rows][cols/32]."""
    return s.reshape(cols // 128, rows, 4).transpose(1, 0, 2).reshape(rows, cols // 32)


def _image_to_rows(s, batch, rows, cols):
    """Weight scales in the block-scaled MMA's copy image -> [batch][rows][cols/32]:
    per matrix, [k-block][128-row block][row % 32][row / 32 % 4][4]."""
    a = s.reshape(batch, cols // 128, rows // 128, 32, 4, 4)      # b, kb, rb, l, g, kk
    return a.transpose(0, 2, 4, 3, 1, 5).reshape(batch, rows, cols // 32)


def _gpu_permute(ids_dev, E):
    T, k = ids_dev.shape
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    ws = torch.empty(M.permute_workspace_bytes(T, E, k), dtype=torch.uint8, device=DEV)
    M.permute(ids_dev, E, counts, offsets, perm, inv, ws)
    return counts, offsets, perm, inv


@pytest.mark.parametrize("rows,cols", [(1, 128), (300, 384), (4096, 6144)])
def test_quantize_act_mxfp8_bit_exact(rows, cols):
    x = random_bf16((rows, cols), seed=rows, idx=6, std=3.0)
    x[0, :32] = 0                                              # an all-zero block
    if rows > 2:
        x[1, 32:64] *= 1e-30                                   # tiny values: clamped scale
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    s = torch.empty((rows, cols // 32), dtype=torch.uint8, device=DEV)
    M.quantize_act_mxfp8(_u16(x.to(DEV)), q, s)
    oq, os_ = oracle.quant_mx_rows(x.float().numpy())
    assert np.array_equal(_kbm_to_rows(s.cpu().numpy(), rows, cols), os_)
    assert np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("batch,rows,cols", [(1, 128, 128), (3, 256, 384), (2, 2048, 1024)])
def test_quantize_weights_mxfp8_bit_exact(batch, rows, cols):
    W = random_bf16((batch, rows, cols), seed=rows + cols, idx=7, std=0.02)
    q = torch.empty(W.shape, dtype=torch.uint8, device=DEV)
    s = torch.empty((batch, rows, cols // 32), dtype=torch.uint8, device=DEV)
    M.quantize_weights_mxfp8(_u16(W.to(DEV)), q, s)
    oq, os_ = oracle.quant_mx_bf16(bits(W))
    assert np.array_equal(_image_to_rows(s.cpu().numpy(), batch, rows, cols), os_)
    assert np.array_equal(q.cpu().numpy(), oq)


def _permuted_quant(x_dev, perm, cfg):
    R = cfg.rows()
    q = torch.empty((R, cfg.d), dtype=torch.uint8, device=DEV)
    s = torch.empty((R, cfg.d // 32), dtype=torch.uint8, device=DEV)
    M.quantize_act_mxfp8_permuted(_u16(x_dev), perm, cfg.k, cfg.Is > 0, q, s)
    return q, s


@pytest.mark.parametrize("cfg", MX, ids=MX_IDS)
def test_quantize_act_mxfp8_permuted_bit_exact(cfg):
    x = make_layer(cfg)["x"]
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 400)
    _, _, perm, _ = _gpu_permute(ids.to(DEV), cfg.E)
    q, s = _permuted_quant(x.to(DEV), perm, cfg)
    _, _, operm, _ = oracle.permute(ids.numpy(), cfg.E)
    tok = np.concatenate([operm // cfg.k, np.arange(cfg.T) if cfg.Is else np.zeros(0, np.int64)])
    oq, os_ = oracle.quant_mx_rows(x.float().numpy()[tok])
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(_kbm_to_rows(s.cpu().numpy(), cfg.rows(), cfg.d), os_)


@pytest.mark.parametrize("cfg", MX, ids=MX_IDS)
def test_weights_mxfp8_match_oracle_quantisation(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    q, s = oracle.quant_mx_bf16(bits(inp["w_d"]))
    assert np.array_equal(layer.mats["w_d"].cpu().numpy(), q)
    assert np.array_equal(_image_to_rows(layer.scales["w_d"].cpu().numpy(), cfg.E, cfg.d, cfg.I), s)


@pytest.mark.parametrize("cfg", MX, ids=MX_IDS)
def test_gemm_gateup_mx(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 100)
    _, offsets, perm, _ = _gpu_permute(ids.to(DEV), cfg.E)
    xq, xs = _permuted_quant(inp["x"].to(DEV), perm, cfg)
    R = cfg.rows()
    hq = torch.empty((R, cfg.I), dtype=torch.uint8, device=DEV)
    hs = torch.empty((R, cfg.I // 32), dtype=torch.uint8, device=DEV)
    M.gemm_gateup(layer.shape(cfg.T), layer.weights, xq, xs, None, offsets, hq, hs, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, operm, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.gateup(oracle_layer(cfg, inp), bits(inp["x"]), operm, ooff)  # FP64 h, pre-quantisation
    gq, gs = hq.cpu().numpy(), _kbm_to_rows(hs.cpu().numpy(), R, cfg.I)
    X = np.repeat(_e8m0(gs), 32, axis=1)
    deq = oracle.e4m3_decode(gq) * X
    # one e4m3 rounding of the block (relative 2^-4, or 2^-10 X near zero) plus
    # FP32 noise; a block maximum whose scaled value lies in (464, 512) saturates
    # at 448 X (the MX format's own clamp): up to 64 X there
    sat = np.abs(deq) == 448.0 * X
    bound = 2.0 ** -4 * np.abs(ref) + 2.0 ** -10 * X + 64.0 * X * sat + 1e-5 * rms(ref)
    assert np.all(np.abs(deq - ref) <= bound * (1 + 1e-6))
    oq, os_ = oracle.quant_mx_rows(ref.astype(np.float32))
    assert np.mean(gs == os_) >= 0.99 and np.mean(gq == oq) >= 0.99


@pytest.mark.parametrize("cfg", MX, ids=MX_IDS)
def test_gemm_down_mx(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 200)
    _, offsets, _, _ = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    hin = random_bf16((R, cfg.I), seed=cfg.seed, idx=8, std=0.5)
    hq = torch.empty((R, cfg.I), dtype=torch.uint8, device=DEV)
    hs = torch.empty((R, cfg.I // 32), dtype=torch.uint8, device=DEV)
    M.quantize_act_mxfp8(_u16(hin.to(DEV)), hq, hs)
    o = torch.empty((R, cfg.d), dtype=torch.float16, device=DEV)
    M.gemm_down(layer.shape(cfg.T), layer.weights, hq, hs, offsets, o, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, _, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.down(oracle_layer(cfg, inp), bf16_to_f64(hin), ooff, cfg.T)
    assert_close_rel(o.cpu().double().numpy(), ref, rtol=O_RTOL, atol=1e-4 * rms(ref), what="o")
