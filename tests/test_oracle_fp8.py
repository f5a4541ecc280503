"""Pins of the oracle's FP8 quantisation: 128x128 weight blocks and 1x128
activation groups.  Sources: "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫",
section HPC-Ops的主要功能 (GroupGEMM FP8, block-wise FP8; FusedMoE activation
quantisation stage) and "PR #54160 完整报告", section 实现拆解 item 4 (FP8
block-wise 128x128)."""
import numpy as np
import torch

import oracle


def _grid_values(rng, n, scale_exp):
    """Random e4m3 values times 2^scale_exp whose magnitudes reach exactly 448 * 2^scale_exp."""
    codes = rng.integers(0, 256, n).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x7E          # no NaN codes
    v = oracle.e4m3_decode(codes)
    v[0] = 448.0 * rng.choice([-1.0, 1.0])
    rng.shuffle(v)
    return v * 2.0**scale_exp


def test_rows_lossless_on_the_grid():
    rng = np.random.default_rng(0)
    rows, cols = 6, 384
    v = np.stack([np.concatenate([_grid_values(rng, 128, int(rng.integers(-9, 3)))
                                  for _ in range(cols // 128)]) for _ in range(rows)])
    q, s = oracle.quant_fp8_rows(v.astype(np.float32))
    assert np.all(np.log2(s) == np.round(np.log2(s)))    # power-of-two scales
    deq = oracle.e4m3_decode(q) * np.repeat(s.astype(np.float64), 128, axis=1)
    assert np.array_equal(deq, v)


def test_rows_codes_match_torch_conversion_and_error_bound():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal((9, 512)) * np.exp2(rng.uniform(-6, 6, (9, 1)))).astype(np.float32)
    v[3, 128:256] = 0.0                                    # an all-zero group: s = 1, q = 0
    q, s = oracle.quant_fp8_rows(v)
    assert s[3, 1] == 1.0 and np.all(q[3, 128:256] == 0)
    for r in range(v.shape[0]):
        for g in range(4):
            blk = v[r, g * 128:(g + 1) * 128]
            amax = np.float32(np.max(np.abs(blk)))
            if amax == 0:
                continue
            assert s[r, g] == np.float32(amax / np.float32(448.0))
            scaled = torch.from_numpy(blk / s[r, g])      # float32 division
            ref = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q[r, g * 128:(g + 1) * 128], ref)
    deq = oracle.e4m3_decode(q) * np.repeat(s.astype(np.float64), 128, axis=1)
    # 3 mantissa bits: relative error <= 2^-4 in the normal range of the scaled values
    scaled = np.abs(v) / np.repeat(s, 128, axis=1)
    normal = scaled >= 2.0**-6
    assert np.all(np.abs(deq - v)[normal] <= 2.0**-4 * np.abs(v)[normal] * (1 + 1e-6))


def test_blocks_are_independent_and_lossless_on_the_grid():
    rng = np.random.default_rng(2)
    E, rows, cols = 2, 256, 384
    exps = rng.integers(-10, -3, (E, rows // 128, cols // 128))
    W = np.zeros((E, rows, cols))
    for e in range(E):
        for i in range(rows // 128):
            for j in range(cols // 128):
                W[e, i * 128:(i + 1) * 128, j * 128:(j + 1) * 128] = \
                    _grid_values(rng, 128 * 128, int(exps[e, i, j])).reshape(128, 128)
    Wb = oracle.bf16_round(W)                       # grid values are exact in bf16
    assert np.array_equal(oracle.bf16_decode(Wb), W)
    q, s = oracle.quant_fp8_blocks(Wb)
    assert np.array_equal(s, np.exp2(exps).astype(np.float32))
    deq = oracle.e4m3_decode(q) * np.repeat(np.repeat(s, 128, 1), 128, 2)
    assert np.array_equal(deq, W)
    # doubling one block changes only that block's scale
    W2 = W.copy()
    W2[1, 128:, :128] *= 2
    q2, s2 = oracle.quant_fp8_blocks(oracle.bf16_round(W2))
    assert np.array_equal(q2, q)
    diff = s2 != s
    assert diff.sum() == 1 and diff[1, 1, 0] and s2[1, 1, 0] == 2 * s[1, 1, 0]
