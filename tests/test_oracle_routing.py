"""Pins of the oracle's top-k routing and per-expert permutation.

Sources: "HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section
HPC-Ops的主要功能 (FusedMoE: routing index, Top-K weighted aggregation) and
section HPC-Ops的技術原理 ("FusedMoE 流水線重構": per-expert counting with one
contiguous output interval per expert); top-8 of 256 from "PR #54160 完整报告",
section 功能与动机."""
import numpy as np
import pytest
from scipy.special import softmax

import oracle
from expert_layer_dual_b200.inputs import random_ids, random_logits


@pytest.mark.parametrize("T,E,k", [(50, 8, 2), (40, 256, 8), (9, 16, 16), (33, 37, 5)])
def test_topk_matches_brute_force_sort(T, E, k):
    l = random_logits(T, E, seed=T + E).numpy()
    ids, w = oracle.route_topk(l, k, renorm=True)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(l[t, e]), e))[:k]
        assert list(ids[t]) == order
        ref = softmax(l[t, order].astype(np.float64))
        np.testing.assert_allclose(w[t], ref, rtol=1e-13, atol=0)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)


def test_topk_without_renormalisation_uses_full_softmax():
    l = random_logits(20, 32, seed=3).numpy()
    ids, w = oracle.route_topk(l, 4, renorm=False)
    full = softmax(l.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, ids.astype(np.int64), 1), rtol=1e-13)


def test_all_zero_logits_pick_lowest_ids_with_equal_weights():
    ids, w = oracle.route_topk(np.zeros((5, 256), np.float32), 8)
    assert np.array_equal(ids, np.tile(np.arange(8, dtype=np.int32), (5, 1)))
    assert np.all(w == 1.0 / 8)


def test_k_equals_E_is_the_full_softmax():
    l = random_logits(7, 12, seed=5, ties=False).numpy()
    ids, w = oracle.route_topk(l, 12)
    full = softmax(l.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, ids.astype(np.int64), 1), rtol=1e-13)
    assert np.all(np.diff(np.take_along_axis(l, ids.astype(np.int64), 1), axis=1) <= 0)


@pytest.mark.parametrize("T,E,k", [(64, 256, 8), (301, 16, 4), (16, 8, 2), (1, 4, 4)])
def test_permute_matches_stable_sort(T, E, k):
    ids = random_ids(T, E, k, seed=T).numpy()
    counts, offsets, perm, inv = oracle.permute(ids, E)
    flat = ids.reshape(-1)
    ref = sorted(range(T * k), key=lambda a: (int(flat[a]), a))
    assert list(perm) == ref
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts) and offsets[E] == T * k
    assert np.array_equal(inv[perm], np.arange(T * k))
    for e in range(E):  # rows of one expert form one interval, in token order
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg // k) > 0)


def test_permute_with_skew_keeps_empty_experts_empty():
    ids = np.array([[3, 1], [3, 0], [1, 3]], np.int32)
    counts, offsets, perm, inv = oracle.permute(ids, 6)
    assert list(counts) == [1, 2, 0, 3, 0, 0]
    assert list(offsets) == [0, 1, 3, 3, 6, 6, 6]
    assert list(perm) == [3, 1, 4, 0, 2, 5]
