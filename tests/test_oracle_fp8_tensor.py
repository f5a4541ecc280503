"""Pins of the oracle's per-tensor FP8: one FP32 scale per weight matrix
(fp32(amax) / 448) and static activation scales.  Sources: "HPC-Ops -
騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的主要功能 (GroupGEMM FP8:
per-tensor and block-wise FP8), and "腾讯混元大模型：从多场景适配到高效部署的全栈技术解析",
section 量化压缩技术实践 / FP8量化方案 (static FP8 quantisation of weights and
activations, scales precomputed from calibration data)."""
import numpy as np
import torch

import oracle


def _e4m3_torch(v):
    return torch.from_numpy(np.clip(v, -448.0, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_tensor_scale_maps_the_amax_to_448_and_codes_match_torch():
    rng = np.random.default_rng(0)
    W = oracle.bf16_round(rng.standard_normal((3, 128, 256)) * np.array([0.01, 1.0, 30.0])[:, None, None])
    q, s = oracle.quant_fp8_tensor(W)
    assert s.shape == (3,)
    Wf = oracle.bf16_decode(W).astype(np.float32)
    amax = np.abs(Wf).reshape(3, -1).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(448.0)).astype(np.float32))
    for b in range(3):
        scaled = (Wf[b] / s[b]).astype(np.float32).astype(np.float64)
        assert np.array_equal(q[b], _e4m3_torch(scaled))
        assert np.max(np.abs(oracle.e4m3_decode(q[b]))) == 448.0


def test_tensor_scale_is_per_matrix_and_zero_matrix_is_lossless():
    rng = np.random.default_rng(1)
    W = oracle.bf16_round(rng.standard_normal((2, 128, 128)) * 0.1)
    q, s = oracle.quant_fp8_tensor(W)
    W2 = W.copy()
    W2[1] = oracle.bf16_round(oracle.bf16_decode(W[1]) * 8.0)   # scale one matrix by 2^3
    q2, s2 = oracle.quant_fp8_tensor(W2)
    assert np.array_equal(q2, q) and s2[0] == s[0] and s2[1] == 8.0 * s[1]
    qz, sz = oracle.quant_fp8_tensor(np.zeros((1, 128, 128), np.uint16))
    assert sz[0] == 1.0 and np.all(qz == 0)


def test_static_activation_codes_saturate_and_match_torch():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(4096) * 3.0).astype(np.float32)
    s = np.float32(0.005)                         # deliberately small: many values saturate
    q = oracle.quant_fp8_static(v, s)
    scaled = (v / s).astype(np.float32).astype(np.float64)
    assert np.array_equal(q, _e4m3_torch(scaled))
    sat = np.abs(scaled) >= 464.0
    assert sat.any() and np.all(np.abs(oracle.e4m3_decode(q[sat])) == 448.0)


def _tensor_grid(rng, shape, scale):
    """e4m3 grid values times `scale`, the matrix maximum exactly 448 * scale."""
    codes = rng.integers(0, 256, shape).astype(np.uint8)
    codes[(codes & 0x7F) >= 0x7F] = 0x7E
    v = oracle.e4m3_decode(codes)
    v.flat[0] = 448.0
    return v * scale


def test_tensor_stages_equal_bf16_stages_on_grid_values():
    rng = np.random.default_rng(10)
    T, d, E, k, I = 12, 256, 3, 2, 128
    sx, sh = 2.0 ** -6, 2.0 ** -9
    w_gu = np.stack([oracle.bf16_round(_tensor_grid(rng, (2 * I, d), 2.0 ** -int(rng.integers(10, 14))))
                     for _ in range(E)])
    w_d = np.stack([oracle.bf16_round(_tensor_grid(rng, (d, I), 2.0 ** -int(rng.integers(10, 14))))
                    for _ in range(E)])
    ws_gu = oracle.bf16_round(_tensor_grid(rng, (2 * I, d), 2.0 ** -12))
    ws_d = oracle.bf16_round(_tensor_grid(rng, (d, I), 2.0 ** -12))
    x = oracle.bf16_round(_tensor_grid(rng, (T, d), sx))
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    layers = [oracle.Layer(T=T, d=d, E=E, k=k, I=I, Is=I, w_gu=w_gu, w_d=w_d, ws_gu=ws_gu,
                           ws_d=ws_d, router_w=np.zeros((E, d), np.float32), wdtype=wd,
                           act_sx=sx, act_sh=sh)
              for wd in (0, 3)]
    np.testing.assert_allclose(oracle.gateup(layers[1], x, perm, offsets),
                               oracle.gateup(layers[0], x, perm, offsets), rtol=1e-13, atol=0)
    hg = _tensor_grid(rng, (T * k + T, I), sh)
    np.testing.assert_allclose(oracle.down(layers[1], hg, offsets, T),
                               oracle.down(layers[0], hg, offsets, T), rtol=1e-13, atol=0)
    # off the grid (and with a static scale that clips) the per-tensor path differs
    hn = rng.standard_normal((T * k + T, I))
    assert np.max(np.abs(oracle.down(layers[1], hn, offsets, T) - oracle.down(layers[0], hn, offsets, T))) > 0
