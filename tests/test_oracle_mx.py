"""Pins of the oracle's MXFP8 quantisation (e4m3 elements, one E8M0 scale per
block of 32 along K).  The format is named by "PR #54160 完整报告", section
实现拆解 item 4 (FP8 blockwise 128x128 and MXFP8 scale parameters); its
definition (block of 32, power-of-two shared scale, e4m3 elements) is the OCP
microscaling one.  Each test checks a property that a plausible slip in the
oracle (a wrong exponent offset, a wrong block length or axis, a rounding
mode) would break, without restating the oracle's formula."""
import numpy as np
import torch

import oracle


def _mx_grid_block(rng, e):
    """32 values that MX quantisation reproduces exactly with scale 2^e: e4m3
    values times 2^e, one of them with a magnitude in [256, 448] * 2^e."""
    codes = rng.integers(0, 256, 32).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x7E            # no NaN codes
    codes[(codes & 0x7F) > 0x7E] = 0x7E
    codes[0] = (rng.integers(0, 2) << 7) | (15 << 3) | rng.integers(0, 7)  # exponent 8: 256..448
    v = oracle.e4m3_decode(codes)
    rng.shuffle(v)
    return v * 2.0**e


def _mx_grid_matrix(rng, rows, cols):
    return np.stack([np.concatenate([_mx_grid_block(rng, int(rng.integers(-20, -4)))
                                     for _ in range(cols // 32)]) for _ in range(rows)])


def test_scale_brackets_the_block_amax():
    # The element of largest magnitude lands in the top binade of e4m3 after
    # scaling: amax / X in [256, 512).  An exponent offset of 7 or 9 would put
    # it in [128, 256) or [512, 1024).
    rng = np.random.default_rng(0)
    v = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-12, 12, (64, 1)))).astype(np.float32)
    q, s = oracle.quant_mx_rows(v)
    amax = np.abs(v.reshape(64, 8, 32)).max(axis=2)
    X = np.vectorize(oracle.e8m0_decode)(s)
    assert np.all(amax / X >= 256) and np.all(amax / X < 512)
    # the amax element's code is the largest in its block (saturating at 448)
    deq = np.abs(oracle.e4m3_decode(q)).reshape(64, 8, 32)
    assert np.all(deq.max(axis=2) >= 256) and np.all(deq.max(axis=2) <= 448)


def test_zero_and_extreme_blocks():
    assert oracle.mx_scale_byte(0.0) == 0
    assert oracle.e8m0_decode(127) == 1.0 and oracle.e8m0_decode(0) == 2.0**-127
    assert np.isnan(oracle.e8m0_decode(255))
    v = np.zeros((1, 64), np.float32)
    v[0, 32:] = 1.0
    q, s = oracle.quant_mx_rows(v)
    assert s[0, 0] == 0 and np.all(q[0, :32] == 0)
    assert oracle.e8m0_decode(s[0, 1]) * oracle.e4m3_decode(q[0, 32]) == 1.0
    # huge and tiny amax clamp to the E8M0 range instead of wrapping
    assert oracle.mx_scale_byte(3.0e38) <= 254
    assert oracle.mx_scale_byte(1.0e-44) == 0


def test_codes_match_torch_e4m3_conversion():
    # Element rounding is e4m3 round-to-nearest-even of v / X, saturating at
    # 448: compare with PyTorch's float8_e4m3fn cast of the exactly scaled values.
    rng = np.random.default_rng(1)
    v = rng.standard_normal((32, 512)).astype(np.float32)
    q, s = oracle.quant_mx_rows(v)
    X = np.repeat(np.vectorize(oracle.e8m0_decode)(s), 32, axis=1)
    scaled = v.astype(np.float64) / X
    ref = torch.from_numpy(np.clip(scaled, -448.0, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    # relative error of the dequantised normal values stays within half an e4m3 ulp
    deq = oracle.e4m3_decode(q) * X
    big = np.abs(scaled) >= 2.0**-6
    unsat = np.abs(scaled) < 464.0
    assert np.all(np.abs(deq - v)[big & unsat] <= 2.0**-4 * np.abs(v)[big & unsat] + 1e-30)


def test_lossless_on_the_grid_and_blocks_are_32_wide_along_k():
    rng = np.random.default_rng(2)
    v = _mx_grid_matrix(rng, 5, 256)
    q, s = oracle.quant_mx_rows(v.astype(np.float32))
    deq = oracle.e4m3_decode(q) * np.repeat(np.vectorize(oracle.e8m0_decode)(s), 32, axis=1)
    assert np.array_equal(deq, v)
    # a large value in one block changes that block only
    v2 = v.copy()
    v2[3, 70] = 1e3
    q2, s2 = oracle.quant_mx_rows(v2.astype(np.float32))
    changed = np.argwhere(s2 != s)
    assert changed.tolist() == [[3, 2]]
    assert np.array_equal(np.delete(q2, np.s_[64:96], axis=1), np.delete(q, np.s_[64:96], axis=1))


def test_power_of_two_scaling_shifts_only_the_scale():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((8, 128)).astype(np.float32)
    q, s = oracle.quant_mx_rows(v)
    for j in (-5, 3, 17):
        qj, sj = oracle.quant_mx_rows(v * np.float32(2.0**j))
        assert np.array_equal(qj, q)
        assert np.array_equal(sj.astype(int), s.astype(int) + j)


def test_weight_quantisation_is_per_row_along_columns():
    rng = np.random.default_rng(4)
    W = oracle.bf16_round(rng.standard_normal((3, 64, 96)) * 0.05)
    q, s = oracle.quant_mx_bf16(W)
    assert q.shape == (3, 64, 96) and s.shape == (3, 64, 3)
    qr, sr = oracle.quant_mx_rows(oracle.bf16_decode(W).reshape(-1, 96).astype(np.float32))
    assert np.array_equal(q.reshape(-1, 96), qr) and np.array_equal(s.reshape(-1, 3), sr)


def test_mx_stages_equal_bf16_stages_on_grid_values():
    # Weights and activations that MX quantisation reproduces exactly: the MX
    # path must equal the BF16 path (pins the block axis and every scale index
    # of both operands in both GEMMs).
    rng = np.random.default_rng(10)
    T, d, E, k, I = 12, 256, 3, 2, 128

    def bf(a):
        return oracle.bf16_round(a)

    w_gu = np.stack([bf(_mx_grid_matrix(rng, 2 * I, d)) for _ in range(E)])
    w_d = np.stack([bf(_mx_grid_matrix(rng, d, I)) for _ in range(E)])
    ws_gu, ws_d = bf(_mx_grid_matrix(rng, 2 * I, d)), bf(_mx_grid_matrix(rng, d, I))
    x = bf(_mx_grid_matrix(rng, T, d))
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    layers = [oracle.Layer(T=T, d=d, E=E, k=k, I=I, Is=I, w_gu=w_gu, w_d=w_d, ws_gu=ws_gu,
                           ws_d=ws_d, router_w=np.zeros((E, d), np.float32), wdtype=wd)
              for wd in (0, 2)]
    h0 = oracle.gateup(layers[0], x, perm, offsets)
    h2 = oracle.gateup(layers[1], x, perm, offsets)
    np.testing.assert_allclose(h2, h0, rtol=1e-13, atol=0)
    hg = _mx_grid_matrix(rng, T * k + T, I)
    o0 = oracle.down(layers[0], hg, offsets, T)
    o2 = oracle.down(layers[1], hg, offsets, T)
    np.testing.assert_allclose(o2, o0, rtol=1e-13, atol=0)
    # off the grid the MX path differs from both BF16 and the 128x128 FP8 path
    hn = rng.standard_normal((T * k + T, I))
    l1 = oracle.Layer(T=T, d=d, E=E, k=k, I=I, Is=I, w_gu=w_gu, w_d=w_d, ws_gu=ws_gu, ws_d=ws_d,
                      router_w=np.zeros((E, d), np.float32), wdtype=1)
    o_mx, o_bf = oracle.down(layers[1], hn, offsets, T), oracle.down(layers[0], hn, offsets, T)
    assert np.max(np.abs(o_mx - o_bf)) > 0
    assert np.max(np.abs(o_mx - oracle.down(l1, hn, offsets, T))) > 0
