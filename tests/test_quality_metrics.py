"""The selection-quality metrics of bench.py (recall, IoU, attention-mass recall, Spearman,
popcount) against closed forms and library routines, on the CPU."""
import math

import numpy as np
import pytest
import scipy.stats
import torch

import bench


def test_recall_at_k_ignores_padding():
    true = torch.tensor([3, 7, 9, 11])
    sel = torch.tensor([7, 11, 2, -1, -1])
    assert bench.recall_at_k(sel, true) == 0.5
    assert bench.recall_at_k(torch.tensor([-1]), true) == 0.0
    assert bench.recall_at_k(true.flip(0), true) == 1.0


def test_iou():
    a = torch.tensor([1, 2, 3, 4, -1])
    b = torch.tensor([3, 4, 5, 6])
    assert bench.iou(a, b) == pytest.approx(2 / 6)
    assert bench.iou(a[:4], a[:4]) == 1.0
    assert bench.iou(torch.tensor([-1]), torch.tensor([-1])) == 1.0


def test_mass_recall_closed_forms():
    # Equal logits: the mass on a set is its share of the keys.
    lg = torch.zeros(3, 10)
    assert bench.mass_recall(lg, torch.tensor([0, 5, -1]), 1.0) == pytest.approx(0.2)
    # Two keys, logits 0 and log(3): softmax (1/4, 3/4).
    lg = torch.tensor([[0.0, math.log(3.0)]])
    assert bench.mass_recall(lg, torch.tensor([1]), 1.0) == pytest.approx(0.75)
    # The scale multiplies the logits before the softmax.
    assert bench.mass_recall(lg * 2, torch.tensor([1]), 0.5) == pytest.approx(0.75)


def test_spearman_matches_scipy_with_ties():
    rng = np.random.default_rng(3)
    x = rng.integers(0, 20, 500).astype(np.float64)   # many ties
    y = x * 0.5 + rng.normal(0, 3, 500)
    ref = scipy.stats.spearmanr(x, y).statistic
    assert bench.spearman(torch.tensor(x), torch.tensor(y)) == pytest.approx(ref, abs=1e-12)
    assert bench.spearman(torch.arange(10.0), torch.arange(10.0) ** 3) == pytest.approx(1.0)
    assert bench.spearman(torch.arange(10.0), -torch.arange(10.0)) == pytest.approx(-1.0)


def test_popcount32_matches_bit_count():
    rng = np.random.default_rng(5)
    v = rng.integers(-2**31, 2**31, 1000, dtype=np.int64).astype(np.int32)
    v[:4] = [0, -1, np.int32(-2**31), 2**31 - 1]
    got = bench.popcount32(torch.tensor(v)).numpy()
    want = np.array([bin(int(x) & 0xFFFFFFFF).count("1") for x in v])
    assert (got == want).all()
