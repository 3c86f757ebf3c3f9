"""The synthetic input recipe (CPU): the size laws, the label layout and the
key/query construction the workloads are built from, and their seeding.

These stand in for the pages' model caches, so the tests check the recipe's
stated statistics rather than any value of the method.
"""
import math

import numpy as np
import torch

import synth


def test_size_laws_fill_the_context_with_their_means():
    rng = np.random.default_rng(0)
    n = 400_000
    logn = synth.community_sizes("lognormal", n, rng)
    zipf = synth.community_sizes("zipf", n, rng)
    multi = synth.community_sizes("multinomial", 1020, rng, n_comm=16, min_size=8)
    for sizes in (logn, zipf):
        assert sizes.sum() == n and sizes.min() >= 1
    assert multi.sum() == 1020 and len(multi) == 16 and multi.min() >= 8
    # log-normal with sigma 1 and mu = ln 64 - 1/2: mean 64
    assert abs(logn[:-1].mean() - 64.0) < 3.0
    # Zipf(1.2) on 1..4096: mean sum k^-0.2 / sum k^-1.2 (~209)
    k = np.arange(1, 4097, dtype=np.float64)
    zmean = (k ** -0.2).sum() / (k ** -1.2).sum()
    assert abs(zipf[:-1].mean() - zmean) / zmean < 0.15
    assert zipf.max() <= 4096


def test_labels_put_sinks_first_and_each_member_once():
    rng = np.random.default_rng(1)
    sizes = np.array([3, 5, 2, 7])
    T, S = 4 + sizes.sum(), 4
    for layout in ("scatter", "spans"):
        lab = synth.graph_labels(sizes, T, S, rng, layout)
        assert np.all(lab[:S] == -1)
        assert np.array_equal(np.bincount(lab[S:]), sizes)
        if layout == "spans":  # each community one contiguous run
            for c in range(len(sizes)):
                pos = np.flatnonzero(lab == c)
                assert pos[-1] - pos[0] + 1 == len(pos)


def test_draws_are_seeded_and_follow_the_cluster_partition():
    wl = synth.WORKLOADS["tiny"].replace(T=512, B=2)
    a, b = synth.draw_cache(wl, device="cpu"), synth.draw_cache(wl, device="cpu")
    assert torch.equal(a.K, b.K) and torch.equal(a.V, b.V) and np.array_equal(a.labels, b.labels)
    other = synth.draw_cache(wl, layer=1, device="cpu")
    assert not torch.equal(a.K, other.K)
    # keys of a community sit around its true centre (noise 0.3 per dimension)
    lab = a.labels[0, synth.cluster_graph(wl, 0)]
    K = a.K[0, 0, : wl.T].double()
    c = int(lab[wl.S])
    members = torch.from_numpy(np.flatnonzero(lab == c))
    resid = K[members] - a.mu[0, 0, c].double()
    assert abs(resid.std().item() - 0.3) < 0.05
    # rows past T are zero until appended
    assert torch.count_nonzero(a.K[:, :, wl.T:]) == 0
    # queries: half a cluster centre plus unit noise, in the cache dtype
    q = synth.draw_queries(wl, a, 0)
    assert q.shape == (wl.B, wl.Hq, wl.d) and q.dtype == synth.torch_dtype(wl.dtype)
    assert torch.equal(q, synth.draw_queries(wl, a, 0)) and not torch.equal(q, synth.draw_queries(wl, a, 1))
    kn, vn = synth.draw_new_tokens(wl, a, 0)
    assert kn.shape == vn.shape == (wl.B, wl.Hkv, wl.d)
    assert math.isfinite(float(kn.abs().sum())) and math.isfinite(float(vn.abs().sum()))
