"""GPU parity of the per-tensor FP8 path (one scale per weight matrix, static
calibrated activation scales) against the FP64 oracle: codes and scales
bit-exact, gate-up within one e4m3 rounding of h (values past the static range
clamp at 448 s_h), down within FP32 accumulation noise.  Sources: "HPC-Ops",
section HPC-Ops的主要功能 (GroupGEMM FP8, per-tensor); "腾讯混元大模型：从多场景适配到
高效部署的全栈技术解析", section 量化压缩技术实践 / FP8量化方案 (static FP8)."""
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

F8T = [
    MoEConfig("f8tsmall", T=200, d=512, E=16, k=4, I=256, Is=256, wdtype=3, seed=51),
    MoEConfig("f8todd", T=77, d=384, E=8, k=2, I=128, Is=0, wdtype=3, seed=52),
]
IDS = [c.name for c in F8T]


def _u16(t):
    return t.view(torch.uint16)


def _gpu_permute(ids_dev, E):
    T, k = ids_dev.shape
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    ws = torch.empty(M.permute_workspace_bytes(T, E, k), dtype=torch.uint8, device=DEV)
    M.permute(ids_dev, E, counts, offsets, perm, inv, ws)
    return counts, offsets, perm, inv


@pytest.mark.parametrize("batch,rows,cols", [(1, 8, 128), (3, 256, 384), (2, 2048, 1024)])
def test_quantize_weights_fp8_tensor_bit_exact(batch, rows, cols):
    W = random_bf16((batch, rows, cols), seed=rows + cols, idx=9, std=0.02)
    W[0] *= 7.0                                                # matrices with different scales
    q = torch.empty(W.shape, dtype=torch.uint8, device=DEV)
    s = torch.empty(batch, dtype=torch.float32, device=DEV)
    M.quantize_weights_fp8_tensor(_u16(W.to(DEV)), q, s)
    oq, os_ = oracle.quant_fp8_tensor(bits(W))
    assert np.array_equal(s.cpu().numpy(), os_) and np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("scale", [0.001, 0.02, 1.0])
def test_quantize_act_fp8_static_bit_exact(scale):
    x = random_bf16((300, 384), seed=5, idx=10, std=3.0)
    q = torch.empty(x.shape, dtype=torch.uint8, device=DEV)
    M.quantize_act_fp8_static(_u16(x.to(DEV)), scale, q)
    oq = oracle.quant_fp8_static(x.float().numpy(), np.float32(scale))
    assert np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("scale", [2.0 ** -26, 3.1e-7, 1.7e-3, 0.0123, 5.1 / 448, 0.25, 1.0, 3.0,
                                   777.7, 2.0 ** 26, 2.0 ** -27, 2.0 ** 27, 1.0e-30, 1.0e30])
def test_quantize_act_fp8_static_every_bf16_value(scale):
    # all 65536 bf16 bit patterns (zeros, subnormals, infinities and NaNs included):
    # the static quantiser divides by its fixed scale through the reciprocal with two
    # FMA corrections inside 2^-26 <= s <= 2^26 and 2^-100 <= |v| <= 2^100 (IEEE
    # division elsewhere); its codes must equal the oracle's e4m3(fp32(v / s)) for all
    bits16 = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    x = bits16.reshape(512, 128).contiguous()
    q = torch.empty((512, 128), dtype=torch.uint8, device=DEV)
    M.quantize_act_fp8_static(_u16(x.to(DEV)), scale, q)
    oq = oracle.quant_fp8_static(x.float().numpy(), np.float32(scale))
    assert np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("cfg", F8T, ids=IDS)
def test_quantize_act_fp8_static_permuted_bit_exact(cfg):
    x = make_layer(cfg)["x"]
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 400)
    _, _, perm, _ = _gpu_permute(ids.to(DEV), cfg.E)
    q = torch.empty((cfg.rows(), cfg.d), dtype=torch.uint8, device=DEV)
    M.quantize_act_fp8_static_permuted(_u16(x.to(DEV)), perm, cfg.k, cfg.Is > 0, 0.01, q)
    _, _, operm, _ = oracle.permute(ids.numpy(), cfg.E)
    tok = np.concatenate([operm // cfg.k, np.arange(cfg.T) if cfg.Is else np.zeros(0, np.int64)])
    assert np.array_equal(q.cpu().numpy(), oracle.quant_fp8_static(x.float().numpy()[tok], np.float32(0.01)))


@pytest.mark.parametrize("cfg", F8T, ids=IDS)
@pytest.mark.parametrize("n_tokens", [64, 1, 77])
def test_calibrate_fp8_static_bit_exact(cfg, n_tokens):
    # moe_calibrate_fp8_static computes, on the GPU, the static scales of x and of the
    # BF16 gate-up output h of the calibration tokens.  Both must equal the oracle's
    # per-tensor quantiser rule s = fp32(amax) / 448 (FP32 division) applied to the same
    # values: x itself, and the h the library's BF16 gate-up left in the workspace (whose
    # own parity is checked against the oracle here, and by the gate-up stage tests).
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    n = min(n_tokens, cfg.T)
    x = inp["x"][:n].contiguous()
    bf = {k: inp[k].to(DEV) if inp.get(k) is not None else None for k in ("w_gu", "w_d", "ws_gu", "ws_d")}
    p = M._p
    w16 = M.moe_weights(p(bf["w_gu"]), p(bf["w_d"]), None, None, p(bf["ws_gu"]), p(bf["ws_d"]), None, None,
                        p(layer.router_hi), p(layer.router_lo), p(layer.router_bias), 1.0, 1.0)
    shape16 = M.moe_shape(n, cfg.d, cfg.E, cfg.k, cfg.I, cfg.Is, M.WDTYPE_BF16, int(cfg.renorm))
    ws = torch.empty(M.workspace_bytes(shape16), dtype=torch.uint8, device=DEV)
    scales = torch.empty(2, dtype=torch.float32, device=DEV)
    M.calibrate_fp8_static(shape16, w16, _u16(x.to(DEV)), scales, ws)
    st = M.workspace_view(ws, shape16)
    h = st["h"].clone()
    torch.cuda.synchronize()
    assert M.read_device_status(ws) == M.OK
    sx, sh = scales.cpu().numpy()
    _, osx = oracle.quant_fp8_tensor(bits(x)[None])
    _, osh = oracle.quant_fp8_tensor(bits(h)[None])
    assert sx.tobytes() == osx[0].tobytes() and sh.tobytes() == osh[0].tobytes()
    # the h the scale was taken over is the layer's gate-up output of these tokens
    ids = st["ids"].cpu().numpy()
    _, ooff, operm, _ = oracle.permute(ids, cfg.E)
    L = oracle_layer(MoEConfig(**{**cfg.__dict__, "wdtype": 0}), inp, T=n)
    ref = oracle.gateup(L, bits(x), operm, ooff)[:, : cfg.I]
    assert_close_rel(bf16_to_f64(h), ref, rtol=2.0 ** -8, atol=1e-3 * rms(ref), what="h")
    # the layer object calibrates with the same entry point on its first 64 tokens
    if n == min(layer.CALIBRATION_TOKENS, cfg.T):
        assert layer.act_scales == (float(sx), float(sh))


def test_calibrate_fp8_static_rejects_bad_arguments():
    cfg = F8T[0]
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    scales = torch.empty(2, dtype=torch.float32, device=DEV)
    x = inp["x"][:8].to(DEV)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(M.MoEError) as e:              # the weights must be the BF16 originals
        M.calibrate_fp8_static(layer.shape(8), layer.weights, _u16(x), scales, ws)
    assert e.value.code == M.UNSUPPORTED
    shape0 = M.moe_shape(0, cfg.d, cfg.E, cfg.k, cfg.I, cfg.Is, M.WDTYPE_BF16, 1)
    with pytest.raises(M.MoEError) as e:              # nothing to calibrate on
        M.calibrate_fp8_static(shape0, layer.weights, _u16(x), scales, ws)
    assert e.value.code == M.INVALID_ARG


@pytest.mark.parametrize("cfg", F8T, ids=IDS)
def test_gemm_gateup_f8t(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    sx, sh = (float(np.float32(v)) for v in layer.act_scales)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 100)
    _, offsets, perm, _ = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    xq = torch.empty((R, cfg.d), dtype=torch.uint8, device=DEV)
    M.quantize_act_fp8_static_permuted(_u16(inp["x"].to(DEV)), perm, cfg.k, cfg.Is > 0, sx, xq)
    hq = torch.empty((R, cfg.I), dtype=torch.uint8, device=DEV)
    M.gemm_gateup(layer.shape(cfg.T), layer.weights, xq, None, None, offsets, hq, None, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, operm, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.gateup(oracle_layer(cfg, inp, act=(sx, sh)), bits(inp["x"]), operm, ooff)
    gq = hq.cpu().numpy()
    deq = oracle.e4m3_decode(gq) * sh
    sat = np.abs(ref) > 448.0 * sh
    want = np.where(sat, np.sign(ref) * 448.0 * sh, ref)
    bound = 2.0 ** -4 * np.abs(want) + 2.0 ** -10 * sh + 1e-5 * rms(ref)
    assert np.all(np.abs(deq - want) <= bound * (1 + 1e-6))
    oq = oracle.quant_fp8_static(ref.astype(np.float32), np.float32(sh))
    assert np.mean(gq == oq) >= 0.99


@pytest.mark.parametrize("cfg", F8T, ids=IDS)
def test_gemm_down_f8t(cfg):
    inp = make_layer(cfg)
    layer = M.MoELayer(cfg, inp)
    sx, sh = (float(np.float32(v)) for v in layer.act_scales)
    ids = random_ids(cfg.T, cfg.E, cfg.k, seed=cfg.seed + 200)
    _, offsets, _, _ = _gpu_permute(ids.to(DEV), cfg.E)
    R = cfg.rows()
    hin = random_bf16((R, cfg.I), seed=cfg.seed, idx=11, std=0.5)
    hq = torch.empty((R, cfg.I), dtype=torch.uint8, device=DEV)
    M.quantize_act_fp8_static(_u16(hin.to(DEV)), sh, hq)
    o = torch.empty((R, cfg.d), dtype=torch.float16, device=DEV)
    M.gemm_down(layer.shape(cfg.T), layer.weights, hq, None, offsets, o, layer.ws)
    assert M.read_device_status(layer.ws) == M.OK
    _, ooff, _, _ = oracle.permute(ids.numpy(), cfg.E)
    ref = oracle.down(oracle_layer(cfg, inp, act=(sx, sh)), bf16_to_f64(hin), ooff, cfg.T)
    assert_close_rel(o.cpu().double().numpy(), ref, rtol=O_RTOL, atol=1e-4 * rms(ref), what="o")
