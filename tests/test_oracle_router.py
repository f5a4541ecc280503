"""Pins of the oracle's dual-BF16 router (weight split and logits).

Source: "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section
HPC-Ops的技術原理, paragraph "Router GEMM 雙 BF16 模擬 FP32"."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "router_split_examples.txt")


def _bits_to_f32(b: int) -> np.float32:
    return np.array([b], dtype=np.uint32).view(np.float32)[0]


def test_split_worked_examples():
    rows = [l.split()[:3] for l in open(GOLDEN, encoding="utf-8")
            if l.strip() and not l.startswith("#")]
    assert len(rows) >= 5
    for w, hi, lo in rows:
        W = np.array([_bits_to_f32(int(w, 16))], dtype=np.float32)
        h, l = oracle.router_split(W)
        assert (int(h[0]), int(l[0])) == (int(hi, 16), int(lo, 16)), w


def test_split_reconstruction_bound():
    # |W - (hi + lo/256)| <= 2^(e-16) where 2^e <= |W| < 2^(e+1)
    rng = np.random.default_rng(0)
    W = (rng.standard_normal(200_000) * np.exp2(rng.uniform(-20, 20, 200_000))).astype(np.float32)
    hi, lo = oracle.router_split(W)
    rec = oracle.bf16_decode(hi) + oracle.bf16_decode(lo) / 256.0
    Wd = W.astype(np.float64)
    e = np.floor(np.log2(np.abs(Wd)))
    assert np.all(np.abs(Wd - rec) <= np.exp2(e - 16))
    # the hi part alone is only bf16-accurate: the low part is what buys the bits
    assert np.max(np.abs(Wd - oracle.bf16_decode(hi)) / np.abs(Wd)) > 2.0**-10


def test_split_of_bf16_values_has_zero_low_part():
    rng = np.random.default_rng(1)
    b = rng.integers(0, 65536, 5000).astype(np.uint16)
    v = oracle.bf16_decode(b)
    keep = np.isfinite(v) & (np.abs(v) > 1e-30)
    W = v[keep].astype(np.float32)
    hi, lo = oracle.router_split(W)
    assert np.array_equal(hi, b[keep]) and np.all((lo & 0x7FFF) == 0)


def _rand_bf16(rng, shape, std):
    return oracle.bf16_round(rng.standard_normal(shape) * std)


def test_logits_match_float64_matmul():
    rng = np.random.default_rng(2)
    T, d, E = 37, 256, 24
    x = _rand_bf16(rng, (T, d), 1.0)
    W = (rng.standard_normal((E, d)) / 16).astype(np.float32)
    bias = rng.standard_normal(E).astype(np.float32)
    hi, lo = oracle.router_split(W)
    got = oracle.router_logits(x, hi, lo, bias)
    weff = oracle.bf16_decode(hi) + oracle.bf16_decode(lo) / 256.0
    ref = oracle.bf16_decode(x) @ weff.T + bias.astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_one_hot_rows_give_the_split_weight_exactly():
    rng = np.random.default_rng(3)
    d, E = 128, 16
    W = (rng.standard_normal((E, d)) / 11).astype(np.float32)
    hi, lo = oracle.router_split(W)
    idx = np.array([0, 5, 77, 127])
    x = np.zeros((len(idx), d), np.uint16)
    x[np.arange(len(idx)), idx] = 0x3F80  # bf16 1.0
    got = oracle.router_logits(x, hi, lo)
    exact = oracle.bf16_decode(hi[:, idx]).T + oracle.bf16_decode(lo[:, idx]).T / 256.0
    assert np.array_equal(got, exact)


def test_dual_bf16_is_far_more_accurate_than_tf32():
    # The page reports the dual-BF16 error at about 1/36 of TF32's.  With
    # x in bf16, the split keeps ~16 bits of W, TF32 keeps 11: the error ratio
    # must be well below 1 (about 2^-5); dropping the low part would make it
    # larger than 1.
    rng = np.random.default_rng(4)
    T, d, E = 64, 1024, 64
    x = _rand_bf16(rng, (T, d), 1.0)
    W = (rng.standard_normal((E, d)) / 32).astype(np.float32)
    hi, lo = oracle.router_split(W)
    got = oracle.router_logits(x, hi, lo)
    xd = oracle.bf16_decode(x)
    exact = xd @ W.astype(np.float64).T
    wt = W.view(np.uint32)
    # TF32 keeps 10 mantissa bits: round to nearest even on the low 13 bits
    tf = ((wt.astype(np.uint64) + 0xFFF + ((wt >> 13) & 1)) & ~np.uint64(0x1FFF)).astype(np.uint32)
    tf32 = xd @ tf.view(np.float32).astype(np.float64).T
    ratio = np.sqrt(np.mean((got - exact) ** 2) / np.mean((tf32 - exact) ** 2))
    assert ratio < 1 / 8, ratio
