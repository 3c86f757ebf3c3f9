"""The int8 scoring copy's error bound, checked on the CPU.

The first scoring pass reads, per centre row, a scale s = max|c| / 127 and
codes n = round(c * 127 / max|c|), and bounds its score's distance to the
fp32 score by Q8_BOUND * s * |q|_1 / sqrt(d).  These tests take the bound
constant from the kernel source and check, in float32 arithmetic, that it
holds on random rows, on rows built at the codes' rounding midpoints with
signs matched to q (the worst case of the quantisation term), and that a
bound of half the size fails there.

The kernel also replaces q by an integer vector: with sq = fl(max|q| /
Q_SPLIT), Q_i = round(q_i * fl(Q_SPLIT / max|q|)), split as 128 hi + lo,
and scores s * sq * (Q . n) / sqrt(d) from an exact integer dot product.
Its bound adds 127 d QSPLIT_BOUND sq s / sqrt(d).  The second group of tests
emulates that pass (integers exact, every float operation in float32, in the
kernel's order) and checks the bound on random inputs and on an adversarial
one where dropping the split term makes it fail.
"""
import math
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(__file__), "..", "graph_community_sparse_b200", "csrc", "ckv_select.cu")


def kernel_const(name: str, kind: str = "float") -> float:
    m = re.search(rf"constexpr {kind} {name} = ([^;]+);", open(SRC).read())
    expr = m.group(1).replace("f", "")
    return float(eval(expr, {"__builtins__": {}}))


def kernel_bound() -> float:
    return kernel_const("Q8_BOUND")


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


# ---------------------------------------------------------------------------
# the integer query split
# ---------------------------------------------------------------------------

F = np.float32


def split_query(q: np.ndarray, q_split: int):
    """The kernel's split of one head's query: sq, Q (= 128 hi + lo), hi, lo."""
    amax = F(np.abs(q).max())
    sq = F(amax / F(q_split)) if amax > 0 else F(0.0)
    rq = F(F(q_split) / amax) if amax > 0 else F(0.0)
    Q = np.clip(np.rint((q * rq).astype(F)), -q_split, q_split).astype(np.int64)
    hi = (Q + 64) >> 7
    lo = Q - 128 * hi
    return sq, Q, hi, lo


def first_pass(q: np.ndarray, c: np.ndarray):
    """Score and bound of every row as the kernel's first pass computes them
    (one head); also the fp32 score of the exact re-scoring."""
    d = c.shape[1]
    q_split = int(kernel_const("Q_SPLIT", "int"))
    b8, bs = F(kernel_bound()), F(kernel_const("QSPLIT_BOUND"))
    inv = F(1.0 / math.sqrt(d))
    n, s = quantise(c)
    sq, Q, hi, lo = split_query(q, q_split)
    assert np.array_equal(128 * hi + lo, Q) and hi.min() >= -127 and hi.max() <= 127
    assert lo.min() >= -64 and lo.max() <= 63
    acc = n.astype(np.int64) @ Q                   # exact, as the dp4a sums
    assert np.abs(acc).max() < 2 ** 31
    approx = ((acc.astype(F) * sq).astype(F) * s).astype(F) * inv
    qn = F(np.abs(q).astype(F).sum(dtype=F))
    eb = F(F(b8 * qn) + F(F(127.0 * d) * bs) * sq)
    err = (F(eb * inv) * s).astype(F) + F(1e-30)
    exact = fp32_dot(np.broadcast_to(q, c.shape).astype(F), c) * inv
    return exact.astype(np.float64), approx.astype(np.float64), err.astype(np.float64), (eb, qn, sq, inv, s)


@pytest.mark.parametrize("d", [64, 128])
def test_split_bound_holds_on_random_inputs(d):
    rng = np.random.default_rng(200 + d)
    for qscale, cscale in ((1.0, 1.0), (1e-3, 30.0), (40.0, 1e-2)):
        for trial in range(3):
            q = (rng.standard_normal(d) * qscale).astype(F)
            if trial == 2:  # bf16-valued queries, as the bf16 caches give
                q = (q.view(np.uint32) & np.uint32(0xFFFF0000)).view(F)
            c = (rng.standard_normal((1500, d)) * cscale).astype(F)
            exact, approx, err, _ = first_pass(q, c)
            assert np.all(np.abs(exact - approx) <= err)


@pytest.mark.parametrize("d", [64, 128])
def test_split_term_is_needed(d):
    """Both error terms at their worst together: every centre element but
    the row's maximum sits just inside a rounding midpoint of its code
    (|code| = 126), the offset signed like q; q is 0 where the centre has its
    maximum, max|q| sits on a midpoint element, and every other q_i lies
    just under half a split step from an integer, signed like its code.
    The kernel's bound holds; without the split term it does not."""
    rng = np.random.default_rng(300 + d)
    q_split = int(kernel_const("Q_SPLIT", "int"))
    sign = np.where(rng.random(d) < 0.5, -1.0, 1.0)
    amax = 3.0
    sq = float(F(F(amax) / F(q_split)))
    q = (sign * (1000.0 + 0.499) * sq).astype(F)
    q[0] = F(0.0)
    q[1] = F(amax * sign[1])
    rows = []
    for _ in range(300):
        s = float(F(rng.uniform(0.05, 2.0)))
        row = (126.0 + 0.4995) * sign * s
        row[0] = 127.0 * s
        rows.append(row)
    c = np.asarray(rows, dtype=F)
    exact, approx, err, (eb, qn, sq32, inv, s) = first_pass(q, c)
    gap = np.abs(exact - approx)
    assert np.all(gap <= err)
    no_split = (F(F(F(kernel_bound()) * qn) * inv) * s).astype(np.float64)
    assert np.all(gap > no_split)
