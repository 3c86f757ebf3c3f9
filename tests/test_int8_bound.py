"""The int8 scoring copy's error bound, checked on the CPU.

The first scoring pass reads, per centre row, a scale s = max|c| / 127 and
codes n = round(c * 127 / max|c|), and bounds its score's distance to the
fp32 score by Q8_BOUND * s * |q|_1 / sqrt(d).  These tests take the bound
constant from the kernel source and check, in float32 arithmetic, that it
holds on random rows, on rows built at the codes' rounding midpoints with
signs matched to q (the worst case of the quantisation term), and that a
bound of half the size fails there.
"""
import math
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(__file__), "..", "graph_community_sparse_b200", "csrc", "ckv_select.cu")


def kernel_bound() -> float:
    m = re.search(r"constexpr float Q8_BOUND = ([^;]+);", open(SRC).read())
    expr = m.group(1).replace("f", "")
    return float(eval(expr, {"__builtins__": {}}))


def quantise(c: np.ndarray):
    """The copy's definition in float32: scale, reciprocal, rounded codes."""
    amax = np.abs(c).max(axis=-1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    r = (np.float32(127.0) / np.where(amax > 0, amax, np.float32(1.0))).astype(np.float32)
    n = np.where(amax[:, None] > 0, np.rint(c * r[:, None]), 0.0)
    return np.clip(n, -127, 127).astype(np.float32), s


def fp32_dot(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Row-wise dot products accumulated in float32, one term at a time."""
    acc = np.zeros(a.shape[0], dtype=np.float32)
    for i in range(a.shape[1]):
        acc = (acc + a[:, i] * b[:, i]).astype(np.float32)
    return acc


def worst_gap(q: np.ndarray, c: np.ndarray, bound: float) -> float:
    """max over rows of |fp32 score - int8 score| / (bound * s |q|_1 / sqrt(d))."""
    d = c.shape[1]
    inv = np.float32(1.0 / math.sqrt(d))
    n, s = quantise(c)
    qq = np.broadcast_to(q, c.shape).astype(np.float32)
    exact = fp32_dot(qq, c) * inv
    approx = fp32_dot(qq, n) * s * inv
    e = np.float32(bound) * s * np.float32(np.abs(q).sum()) * inv
    ok = e > 0
    return float(np.max(np.abs(exact - approx)[ok] / e[ok])) if ok.any() else 0.0


@pytest.mark.parametrize("d", [64, 128])
def test_bound_holds_on_random_rows(d):
    rng = np.random.default_rng(d)
    bound = kernel_bound()
    for scale in (1e-3, 1.0, 30.0):
        q = rng.standard_normal(d).astype(np.float32)
        c = (rng.standard_normal((2000, d)) * scale).astype(np.float32)
        assert worst_gap(q, c, bound) <= 1.0


@pytest.mark.parametrize("d", [64, 128])
def test_bound_holds_at_rounding_midpoints(d):
    """Every element half a code step from its code, the offset signed like
    q: the quantisation error reaches s/2 |q|_1, the bound's main term."""
    rng = np.random.default_rng(100 + d)
    bound = kernel_bound()
    q = rng.standard_normal(d).astype(np.float32)
    rows = []
    for _ in range(500):
        k = rng.integers(-120, 121, d).astype(np.float64)
        k[0] = 127.0  # fixes max |c| = 127 s exactly
        s = float(np.float32(rng.uniform(0.01, 2.0)))
        off = 0.5 * np.sign(q) * 0.999
        off[0] = 0.0
        rows.append((k + off) * s)
    c = np.asarray(rows, dtype=np.float32)
    gap = worst_gap(q, c, bound)
    assert gap <= 1.0
    # the quantisation term is tight here: half the bound does not hold
    assert worst_gap(q, c, bound / 2) > 1.0
