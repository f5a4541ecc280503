"""Pins of the oracle's fused all-reduce + residual + RMSNorm ("HPC-Ops ...",
HPC-Ops的技術原理, "Fused AllReduce+Norm": RMSNorm(AllReduce(x) + residual,
weight)) against what fixes it independently: PyTorch's own RMSNorm for a
single rank and no residual, closed forms, and invariants of the norm."""
import numpy as np
import pytest
import torch

import oracle
from expert_layer_dual_b200.inputs import random_bf16
from gpu_util import bits


def _x(G, T, d, seed, std=1.0):
    return bits(random_bf16((G, T, d), seed=seed, idx=30, std=std))


def test_one_rank_no_residual_is_torch_rms_norm():
    x = _x(1, 7, 256, 1)
    g = bits(random_bf16((256,), seed=1, idx=31, std=0.5))
    _, out = oracle.allreduce_rmsnorm(x, None, g, 1e-6)
    xt = torch.from_numpy(oracle.bf16_decode(x[0]))
    gt = torch.from_numpy(oracle.bf16_decode(g))
    ref = torch.nn.functional.rms_norm(xt, (256,), weight=gt, eps=1e-6).numpy()
    assert np.max(np.abs(out - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_sum_over_ranks_plus_residual_is_exact_for_equal_parts():
    # G equal parts (bf16 values times a small integer stay exact in FP64)
    x1 = _x(1, 5, 128, 2)
    x = np.repeat(x1, 4, axis=0)
    r = bits(random_bf16((5, 128), seed=2, idx=32))
    g = bits(torch.ones(128, dtype=torch.bfloat16))
    res, _ = oracle.allreduce_rmsnorm(x, r, g, 0.0)
    assert np.array_equal(res, 4 * oracle.bf16_decode(x1[0]) + oracle.bf16_decode(r))


def test_unit_rms_scale_invariance_and_gamma():
    x = _x(3, 9, 256, 3, std=2.0)
    r = bits(random_bf16((9, 256), seed=3, idx=33))
    ones = bits(torch.ones(256, dtype=torch.bfloat16))
    res, out = oracle.allreduce_rmsnorm(x, r, ones, 0.0)
    assert np.allclose(np.mean(out ** 2, axis=1), 1.0, rtol=0, atol=1e-12)
    # doubling every input (exact in bf16) leaves the normalised output unchanged
    x2 = bits(torch.from_numpy(oracle.bf16_decode(x) * 2).to(torch.bfloat16))
    r2 = bits(torch.from_numpy(oracle.bf16_decode(r) * 2).to(torch.bfloat16))
    res2, out2 = oracle.allreduce_rmsnorm(x2, r2, ones, 0.0)
    assert np.array_equal(res2, 2 * res) and np.max(np.abs(out2 - out)) <= 1e-13
    # gamma scales each column; a negative gamma flips it
    g = bits(torch.linspace(-2, 2, 256).to(torch.bfloat16))
    _, outg = oracle.allreduce_rmsnorm(x, r, g, 0.0)
    assert np.max(np.abs(outg - out * oracle.bf16_decode(g)[None])) <= 1e-12


def test_constant_row_closed_form_with_eps():
    # s = c everywhere: out = c / sqrt(c^2 + eps) * gamma
    c, eps = 0.75, 0.01
    x = bits(torch.full((2, 1, 128), c / 2, dtype=torch.bfloat16))
    g = bits(torch.full((128,), 1.5, dtype=torch.bfloat16))
    _, out = oracle.allreduce_rmsnorm(x, None, g, eps)
    assert np.allclose(out, c / np.sqrt(c * c + eps) * 1.5, rtol=1e-15, atol=0)
    zero = bits(torch.zeros((2, 1, 128), dtype=torch.bfloat16))
    _, out0 = oracle.allreduce_rmsnorm(zero, None, g, eps)
    assert np.all(out0 == 0.0)
