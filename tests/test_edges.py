"""The prefill token graph (ckv_build_edges) against the CPU oracle, on a B200.

Direct edges: each query's list must equal the oracle's (direct_edges_at:
the 8 best earlier non-sink keys by graph logit, ties to the lower
position), except for keys whose fp64 logit lies within BAND of the 8th;
the logits the GPU reports must match the fp64 ones within 1e-5.
Co-attention edges: the GPU's (src, dst, weight) set must equal, exactly,
the one the oracle derives (coattention_edges) from the GPU's own direct
lists; the direct lists are checked separately above.
"""
import numpy as np
import pytest
import torch

import graph_community_sparse_b200 as ckv
import oracle.ckv_oracle as O
import synth
from parity_util import BAND

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["qwen3_8b_32k"]


def shape(key, index, **kw):
    args = dict(key=key, title=key, index=index, B=1, T=1100, budgets=(300,), steps=1, update=False)
    args.update(kw)
    return BASE.replace(**args)


SHAPES = [
    shape("edges_group_gq4", 70, Hq=8, Hkv=2),
    shape("edges_head_gq1_d64", 71, Hq=4, Hkv=2, d=64, mode="head"),
    shape("edges_group_gq8", 72, Hq=16, Hkv=2, T=700),
    shape("edges_group_gq2_d64", 73, Hq=4, Hkv=2, d=64, T=900, B=2),
    shape("edges_group_gq1", 74, Hq=2, Hkv=2, T=333),
    shape("edges_no_sinks", 75, Hq=8, Hkv=2, S=0, T=517),
    shape("edges_group_gq4_d64", 79, Hq=8, Hkv=2, d=64, T=777),
]


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def build(wl, pair_cap=None, T_cap=None):
    draw = synth.draw_cache(wl, device="cuda", T_cap=T_cap)
    q = synth.draw_prefill_queries(wl, draw)
    cache = ckv.cache_desc(draw.K, draw.V, wl.Hq)
    mode = ckv.PER_HEAD if wl.mode == "head" else ckv.PER_GROUP
    e = ckv.new_edges(cache, mode, wl.S, wl.T, pair_cap)
    ckv.ckv_build_edges(cache, mode, wl.S, q, wl.T, e)
    torch.cuda.synchronize()
    return draw, q, e


def check_direct(got, got_lam, qh, K, S, i):
    """One query's list against the oracle; True when identical, False when
    it differs only by keys tied (within BAND) with the 8th; raises otherwise."""
    ref = [int(p) for p in O.direct_edges_at(qh, K, S, i)]
    n = int((got >= 0).sum())
    assert np.all(got[n:] == -1), "-1 padding must come last"
    g = [int(p) for p in got[:n]]
    assert n == len(ref), (i, n, len(ref))
    if n:
        lam = O.graph_logits(qh[:, i, :], K, np.asarray(g))
        assert np.abs(lam - got_lam[:n]).max() <= 1e-5, (i, np.abs(lam - got_lam[:n]).max())
    if g == ref:
        return True
    assert len(set(g)) == n and all(S <= p < i for p in g), "an edge outside [S, i)"
    allp = np.asarray(sorted(set(g) | set(ref)), dtype=np.int64)
    lam = dict(zip(allp.tolist(), O.graph_logits(qh[:, i, :], K, allp).tolist()))
    v8 = lam[ref[-1]]
    for p in set(g) ^ set(ref):
        assert abs(lam[p] - v8) <= BAND, f"query {i}: edge {p} differs outside the tie band"
    for a, b in zip(g, g[1:]):
        assert lam[a] >= lam[b] - BAND
    return False


def check_unit(wl, draw, q, e, b, g, queries=None):
    u = b * wl.G + g
    heads = O.graph_heads(wl.mode, g, wl.Hq, wl.Hkv)
    kvh = O.graph_kv_head(wl.mode, g, wl.Hq, wl.Hkv)
    K = draw.K[b, kvh, : wl.T].double().cpu().numpy()
    qh = q[b, heads].double().cpu().numpy()
    nbr = e.nbr[u].cpu().numpy()
    lam = e.lam[u].cpu().numpy()
    assert np.all(nbr[: wl.S] == -1)
    ties = 0
    for i in (range(wl.S, wl.T) if queries is None else queries):
        ties += not check_direct(nbr[i], lam[i], qh, K, wl.S, i)
    # co-attention: exactly the pairs of the GPU's own lists
    lists = [nbr[i][nbr[i] >= 0] for i in range(wl.S, wl.T)]
    ref = O.coattention_edges(lists)
    got = e.pairs(u).cpu().numpy()
    assert int(e.co_n[u].item()) == len(ref)
    assert {(int(a), int(c)): int(w) for a, c, w in got} == ref
    return ties


@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: w.key)
def test_edges_match_oracle(wl):
    draw, q, e = build(wl)
    assert int(e.dev_err.item()) == 0
    ties = sum(check_unit(wl, draw, q, e, b, g) for b in range(wl.B) for g in range(wl.G))
    print(wl.key, "tied lists", ties)


def test_edges_prefill_no_longer_than_sinks():
    wl = shape("edges_tiny_prefill", 76, Hq=8, Hkv=2, T=4)
    draw, q, e = build(wl)
    assert torch.all(e.nbr == -1) and torch.all(e.co_n == 0)


def test_edges_pair_capacity_overflow_is_flagged():
    wl = shape("edges_cap", 77, Hq=8, Hkv=2, T=400)
    _, _, full = build(wl)
    _, _, small = build(wl, pair_cap=50)
    assert int(small.dev_err.item()) & ckv.DEVERR_EDGE_CAP
    for u in range(wl.B * wl.G):
        assert torch.equal(small.co_n[u], full.co_n[u]) and int(full.co_n[u]) > 50
        every = {tuple(r) for r in full.pairs(u).tolist()}
        some = {tuple(r) for r in small.pairs(u).tolist()}
        assert len(some) == 50 and some <= every


def test_edges_full_size_sampled():
    """A Qwen3-8B-shaped prefill of 8192 tokens (one sequence, per-group
    graphs): sampled queries of two graphs checked against the oracle,
    every graph's co-attention set checked in full."""
    wl = synth.WORKLOADS["qwen3_8b_32k"].replace(key="edges_8k", index=78, T=8192, budgets=(2048,))
    draw, q, e = build(wl)
    assert int(e.dev_err.item()) == 0
    rng = np.random.default_rng(5)
    sample = sorted(set([wl.S, wl.S + 1, wl.T - 1] + rng.integers(wl.S, wl.T, 40).tolist()))
    for g in (0, 5):
        check_unit(wl, draw, q, e, 0, g, queries=sample)
    for g in range(wl.G):
        nbr = e.nbr[g].cpu().numpy()
        ref = O.coattention_edges([nbr[i][nbr[i] >= 0] for i in range(wl.S, wl.T)])
        got = e.pairs(g).cpu().numpy()
        assert {(int(a), int(c)): int(w) for a, c, w in got} == ref
