"""GPU: the preparation of the gate-up's A operand inside moe_forward is
token-major -- each token's row is read (and, for the FP8 formats, quantised)
once and stored to each permuted row that holds it (the rows inv[t*k + j],
and T*k + t with the shared expert).  FP8 formats: the output, read from the
forward's workspace, must equal
bit for bit both the stage entry point that quantises each permuted row on
its own (moe_quantize_act_*_permuted, given the forward's perm) and the
oracle's quantisation of the rows x[perm / k] (plus x for the shared rows):
 - 128x128 block FP8: e4m3 codes and FP32 1x128 scales (oracle.quant_fp8_rows);
 - MXFP8: e4m3 codes and E8M0 bytes per 1x32 (oracle.quant_mx_rows);
 - per-tensor FP8: e4m3 codes of v / s_x (oracle.quant_fp8_static).
Configurations cover k = 2, 4, 8 (every copy slot), with and without the
shared expert, and ragged token counts.  BF16 with >= 256 rows per expert on
average (the CTA-pair gate-up): the bf16 routed rows of x in that order, bit for bit,
and the pair gate-up's h equal to the gathering gate-up's on the same routing."""
import numpy as np
import pytest
import torch

import oracle
from expert_layer_dual_b200.configs import MoEConfig
from expert_layer_dual_b200.inputs import make_layer

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import expert_layer_dual_b200.moe as M

DEV = "cuda"

CFGS = [
    MoEConfig("qsmall", T=200, d=512, E=16, k=4, I=256, Is=256, seed=61),
    MoEConfig("qodd", T=77, d=384, E=8, k=2, I=128, Is=0, seed=62),
    MoEConfig("qk8", T=130, d=256, E=64, k=8, I=128, Is=128, seed=63),
]


def _cases():
    for c in CFGS:
        for wd in (1, 2, 3):
            yield pytest.param(MoEConfig(c.name, T=c.T, d=c.d, E=c.E, k=c.k, I=c.I, Is=c.Is,
                                         wdtype=wd, seed=c.seed), id=f"{c.name}-w{wd}")


def _kbm_to_rows(s, rows, cols):
    """MX activation scales, k-block-major [cols/128][rows][4] -> [rows][cols/32]."""
    return s.reshape(cols // 128, rows, 4).transpose(1, 0, 2).reshape(rows, cols // 32)


@pytest.mark.parametrize("cfg", list(_cases()))
def test_forward_quantisation_is_bit_exact(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    x_dev = inp["x"].to(DEV)
    layer.forward(x_dev)
    torch.cuda.synchronize()
    assert layer.device_status() == M.OK
    view = M.workspace_view(layer.ws, layer.shape(cfg.T))
    perm = view["perm"].clone()
    xq = view["xq"].clone()
    R = cfg.rows()
    u16 = x_dev.view(torch.uint16)
    # the per-row stage entry point on the same permutation
    q = torch.empty((R, cfg.d), dtype=torch.uint8, device=DEV)
    if cfg.wdtype == 1:
        s = torch.empty((R, cfg.d // 128), dtype=torch.float32, device=DEV)
        M.quantize_act_fp8_permuted(u16, perm, cfg.k, cfg.Is > 0, q, s)
        assert torch.equal(view["xs"], s)
    elif cfg.wdtype == 2:
        s = torch.empty(R * (cfg.d // 32), dtype=torch.uint8, device=DEV)
        M.quantize_act_mxfp8_permuted(u16, perm, cfg.k, cfg.Is > 0, q, s)
        assert torch.equal(view["xs"], s)
    else:
        M.quantize_act_fp8_static_permuted(u16, perm, cfg.k, cfg.Is > 0, layer.act_scales[0], q)
    assert torch.equal(xq, q)
    # and the oracle on the rows the permutation names
    p = perm.cpu().numpy().astype(np.int64)
    tok = np.concatenate([p // cfg.k, np.arange(cfg.T) if cfg.Is else np.zeros(0, np.int64)])
    rows = inp["x"].float().numpy()[tok]
    if cfg.wdtype == 1:
        oq, os_ = oracle.quant_fp8_rows(rows)
        assert np.array_equal(view["xs"].cpu().numpy(), os_)
    elif cfg.wdtype == 2:
        oq, os_ = oracle.quant_mx_rows(rows)
        assert np.array_equal(_kbm_to_rows(view["xs"].cpu().numpy(), R, cfg.d), os_)
    else:
        oq = oracle.quant_fp8_static(rows, np.float32(layer.act_scales[0]))
    assert np.array_equal(xq.cpu().numpy(), oq)


@pytest.mark.parametrize("cfg", [
    MoEConfig("pair", T=1100, d=512, E=8, k=4, I=256, Is=256, seed=64),
    MoEConfig("pairodd", T=1100, d=384, E=6, k=3, I=128, Is=0, seed=65),
], ids=lambda c: c.name)
def test_forward_permuted_x_bf16(cfg):
    # BF16 with >= 256 rows per expert on average: the forward copies x's routed
    # rows into the permuted row order (token-major) for the CTA-pair gate-up (which
    # reads the shared expert's rows from x itself); row p must be x[perm[p] / k],
    # bit for bit
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    x_dev = inp["x"].to(DEV)
    layer.forward(x_dev)
    torch.cuda.synchronize()
    assert layer.device_status() == M.OK
    view = M.workspace_view(layer.ws, layer.shape(cfg.T))
    assert "xq" in view
    p = view["perm"].cpu().numpy().astype(np.int64)
    want = inp["x"].view(torch.int16).numpy()[p // cfg.k]
    assert np.array_equal(view["xq"].cpu().view(torch.int16).numpy(), want)


@pytest.mark.parametrize("cfg", [
    MoEConfig("pair", T=1100, d=512, E=8, k=4, I=256, Is=256, seed=66),
    MoEConfig("pairodd", T=1100, d=384, E=6, k=3, I=128, Is=0, seed=67),
], ids=lambda c: c.name)
def test_pair_gateup_equals_gathering_gateup(cfg):
    # the forward's gate-up on CTA pairs (A rows from the permuted copy of x) and
    # the stage entry point's gate-up (x gathered through perm, one-CTA tiles) on
    # the same routing give the same h, bit for bit
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    x_dev = inp["x"].to(DEV)
    layer.forward(x_dev)
    torch.cuda.synchronize()
    assert layer.device_status() == M.OK
    shape = layer.shape(cfg.T)
    view = M.workspace_view(layer.ws, shape)
    h_pair = view["h"].clone()
    perm, offsets = view["perm"].clone(), view["offsets"].clone()
    h = torch.empty_like(h_pair)
    ws = torch.zeros(M.workspace_bytes(shape), dtype=torch.uint8, device=DEV)
    M.gemm_gateup(shape, layer.weights, x_dev.view(torch.uint16), None, perm, offsets, h.view(torch.uint16),
                  None, ws)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), h_pair.view(torch.int16))
