"""Pins of the CPU oracle against facts fixed outside it (CPU only).

The pages print no worked example, so every pin is one of: a closed form
worked by hand, a special case that reduces to a library routine (dense
attention via torch's scaled_dot_product_attention in float64), brute-force
enumeration on tiny inputs, or an invariant the pages state (sinks always
present, cache never modified, one centre changed per new token).  The
mutation tests at the end plant plausible mistakes in copies of the oracle's
functions and check that some pin catches each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.ckv_oracle as O
import synth


GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def _num(x):
    """A fixture number: floats as written, plus "ln3" and "-inf"."""
    return {"ln3": math.log(3.0), "-inf": -math.inf}.get(x, x) if isinstance(x, str) else x


def _arr(a):
    return np.array([[_num(x) for x in row] for row in a] if a and isinstance(a[0], list) else [_num(x) for x in a],
                    dtype=np.float64)


def _sdpa(q, K, V):
    """Dense softmax attention of one query via torch (float64)."""
    qt = torch.from_numpy(np.asarray(q, dtype=np.float64))[None, None, None, :]
    Kt = torch.from_numpy(np.asarray(K, dtype=np.float64))[None, None]
    Vt = torch.from_numpy(np.asarray(V, dtype=np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[0, 0, 0].numpy()


def _random_graph(rng, T=160, S=4, C=7, d=16):
    sizes = synth.community_sizes("multinomial", T - S, rng, n_comm=C, min_size=2)
    labels = synth.graph_labels(sizes, T, S, rng)
    K = rng.standard_normal((T + 4, d))
    V = rng.standard_normal((T + 4, d))
    return labels, K, V


# ----------------------------------------------------------------------------
# pin checks, written against a function argument so mutants can be fed in
# ----------------------------------------------------------------------------

def check_attention_closed_form(attention):
    # tests/golden/worked_examples.json "attention" (worked by hand there)
    g = GOLDEN["attention"]
    o = attention(_arr(g["q"]), _arr(g["K"]), _arr(g["V"]), np.array(g["positions"]))
    return np.allclose(o, _arr(g["out"]), atol=1e-14)


def check_scores_closed_form(community_scores):
    # tests/golden/worked_examples.json "scores" (worked by hand there)
    g = GOLDEN["scores"]
    s = community_scores(_arr(g["q"]), _arr(g["cent"]), np.array(g["cnt"]))
    return bool(np.array_equal(s, _arr(g["scores"])))


def _brute_select(scores, cnt, budget):
    ids = [c for c in range(len(cnt)) if cnt[c] > 0]

    def above(a, b):  # a ranks above b
        return scores[a] > scores[b] or (scores[a] == scores[b] and a < b)

    best = []
    for r in range(len(ids) + 1):
        for sub in itertools.combinations(ids, r):
            sset = set(sub)
            closed = all(not above(o, c) for c in sset for o in ids if o not in sset)
            if closed and sum(cnt[c] for c in sub) <= budget and len(sub) > len(best):
                best = list(sub)
    if not best and ids:
        best = [c for c in ids if all(not above(o, c) for o in ids if o != c)]
    # rank order by counting how many selected members rank above each one
    return sorted(best, key=lambda c: sum(above(o, c) for o in best))


def check_select_bruteforce(select, trials=300, seed=3):
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        C = int(rng.integers(1, 10))
        scores = rng.integers(-3, 4, C).astype(np.float64)   # many ties
        cnt = rng.integers(0, 6, C)
        budget = int(rng.integers(0, 25))
        scores = np.where(cnt > 0, scores, -np.inf)
        if list(select(scores, cnt, budget)) != _brute_select(scores, cnt, budget):
            return False
    return True


def check_select_worked(select):
    # tests/golden/worked_examples.json "select" (worked by hand there)
    g = GOLDEN["select"]
    s, n = _arr(g["scores"]), np.array(g["cnt"])
    return all(list(select(s, n, budget)) == expect for budget, expect in g["cases"])


def _brute_neighbours(q_heads, K, positions, S, k=8):
    pos = [int(p) for p in positions if p >= S]
    lam = {p: max(float(np.dot(q, K[p])) for q in q_heads) for p in pos}

    def better(a, b):
        return lam[a] > lam[b] or (lam[a] == lam[b] and a < b)

    rank = {p: sum(better(o, p) for o in pos) for p in pos}
    return [p for p in sorted(pos, key=lambda p: rank[p]) if rank[p] < k]


def check_neighbours(neighbours, trials=50, seed=5):
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        d, T, S = 8, 40, 4
        K = rng.integers(-2, 3, (T, d)).astype(np.float64)   # integer keys: many ties
        K[:S] += 10.0                                         # sinks score highest
        q = rng.integers(-1, 2, (2, d)).astype(np.float64)
        positions = np.sort(rng.choice(T, size=int(rng.integers(1, T)), replace=False))
        if list(neighbours(q, K, positions, S)) != _brute_neighbours(q, K, positions, S):
            return False
    return True


def check_dense_equivalence(decode_graph, seed=11):
    rng = np.random.default_rng(seed)
    labels, K, V = _random_graph(rng)
    T, d, Hq, Hkv = len(labels), K.shape[1], 4, 1
    st = O.GraphState(labels, T + 4, 4, 7)
    q = rng.standard_normal((Hq, d))
    gs, outs = decode_graph("group", Hq, Hkv, 0, 0, st, K[None], V[None], q, budget=T)
    if not np.array_equal(gs.tokens, np.arange(T)):
        return False
    return all(np.allclose(outs[h], _sdpa(q[h], K[:T], V[:T]), rtol=0, atol=1e-12) for h in range(Hq))


# ----------------------------------------------------------------------------
# pins on the oracle itself
# ----------------------------------------------------------------------------

def test_attention_closed_form():
    assert check_attention_closed_form(O.attention)


def test_scores_closed_form():
    assert check_scores_closed_form(O.community_scores)


def test_select_worked_examples():
    assert check_select_worked(O.select)


def test_select_matches_bruteforce():
    assert check_select_bruteforce(O.select)


def test_neighbours_match_bruteforce():
    assert check_neighbours(O.neighbours)


def test_full_budget_equals_dense_attention():
    """Budget covering every token: the step is dense softmax attention."""
    assert check_dense_equivalence(O.decode_graph)


def test_one_community_per_head_is_mha_decode():
    """One community holding every non-sink token, one graph per head (Hq = Hkv):
    textbook multi-head decode, for any budget (the top community is always taken)."""
    rng = np.random.default_rng(2)
    T, S, d, H = 90, 4, 16, 3
    labels = np.zeros(T, dtype=np.int32)
    labels[:S] = -1
    K = rng.standard_normal((H, T, d))
    V = rng.standard_normal((H, T, d))
    q = rng.standard_normal((H, d))
    for h in range(H):
        st = O.GraphState(labels, T, S, 1)
        _, outs = O.decode_graph("head", H, H, 0, h, st, K, V, q, budget=1)
        assert np.allclose(outs[h], _sdpa(q[h], K[h], V[h]), rtol=0, atol=1e-12)


def test_sinks_always_present_and_cache_unchanged():
    rng = np.random.default_rng(7)
    labels, K, V = _random_graph(rng)
    K0, V0 = K.copy(), V.copy()
    q = rng.standard_normal((4, K.shape[1]))
    for budget in (0, 1, 20, 80, 1000):
        st = O.GraphState(labels, len(labels) + 4, 4, 7)
        gs, _ = O.decode_graph("group", 4, 1, 0, 0, st, K[None], V[None], q, budget)
        assert set(range(4)) <= set(gs.tokens.tolist())
        assert len(set(gs.tokens.tolist())) == len(gs.tokens)
        assert gs.cnt[gs.selected].sum() <= max(budget, gs.cnt[gs.selected[0]])
        assert not any(p < 4 for p in gs.nbr)
    assert np.array_equal(K, K0) and np.array_equal(V, V0)


def test_centroid_is_running_mean_of_members():
    """The recomputed mean equals the running mean c + (k - c)/(n + 1) applied
    once per joining token; counts always sum to the non-sink tokens."""
    rng = np.random.default_rng(13)
    T0, S, C, d, steps = 120, 4, 5, 8, 30
    sizes = synth.community_sizes("multinomial", T0 - S, rng, n_comm=C, min_size=3)
    labels = synth.graph_labels(sizes, T0, S, rng)
    K = rng.standard_normal((T0 + steps, d))
    st = O.GraphState(labels, T0 + steps, S, C)
    run_c, run_n = O.centroids(K[:T0], st.members())
    for i in range(steps):
        c = int(rng.integers(0, C))
        st.join(T0 + i, c)
        run_c[c] = run_c[c] + (K[T0 + i] - run_c[c]) / (run_n[c] + 1)
        run_n[c] += 1
        cent, cnt = O.centroids(K[: st.T], st.members())
        assert np.array_equal(cnt, run_n)
        assert cnt.sum() == st.T - S
        assert np.allclose(cent, run_c, rtol=0, atol=1e-12)


def check_assign_worked(assign) -> bool:
    """The default update rule on the hand-worked cases."""
    # tests/golden/worked_examples.json "assign" (worked by hand there)
    g = GOLDEN["assign"]
    k, cent = _arr(g["k"]), _arr(g["cent"])
    return all(assign(k, cent, cand) == expect for cand, expect in g["cases"])


def check_graph_logits_worked(graph_logits) -> bool:
    """Graph logits with their 1/sqrt(d) scale, in the order of the positions given."""
    # tests/golden/worked_examples.json "graph_logits" (worked by hand there)
    g = GOLDEN["graph_logits"]
    lam = graph_logits(_arr(g["q"]), _arr(g["K"]), np.array(g["positions"]))
    return bool(np.allclose(lam, _arr(g["logits"]), rtol=0, atol=1e-15))


def test_assign_worked_examples():
    assert check_assign_worked(O.assign)


def test_graph_logits_worked_example():
    assert check_graph_logits_worked(O.graph_logits)


def _assign_ties_high(k, cent, cand):
    best, bs = -1, -math.inf
    for c in sorted(set(cand)):
        s = float(np.dot(k, cent[c])) / math.sqrt(len(k))
        if s >= bs:
            best, bs = c, s
    return best


def _assign_first_candidate(k, cent, cand):
    return cand[0] if cand else -1


def _logits_unscaled(q, K, positions):
    return (np.asarray(K)[np.asarray(positions)] @ np.asarray(q).T).max(axis=1)


def _logits_mean_heads(q, K, positions):
    return (np.asarray(K)[np.asarray(positions)] @ np.asarray(q).T).mean(axis=1) / math.sqrt(np.asarray(q).shape[1])


def _logits_first_head(q, K, positions):
    return (np.asarray(K)[np.asarray(positions)] @ np.asarray(q)[0]) / math.sqrt(np.asarray(q).shape[1])


@pytest.mark.parametrize("mutant", [_assign_ties_high, _assign_first_candidate])
def test_pins_catch_assign_mutants(mutant):
    assert not check_assign_worked(mutant)


@pytest.mark.parametrize("mutant", [_logits_unscaled, _logits_mean_heads, _logits_first_head])
def test_pins_catch_graph_logit_mutants(mutant):
    assert not check_graph_logits_worked(mutant)


def test_assign_bruteforce_ties_and_one_update():
    rng = np.random.default_rng(17)
    d, C = 8, 6
    for _ in range(100):
        cent = rng.integers(-2, 3, (C, d)).astype(np.float64)
        cent[3] = cent[1]                       # a guaranteed tie between ids 1 and 3
        k = rng.integers(-2, 3, d).astype(np.float64)
        cand = list(rng.choice(C, size=int(rng.integers(1, C + 1)), replace=True))
        got = O.assign(k, cent, cand)
        vals = {c: float(np.dot(k, cent[c])) for c in set(cand)}
        top = max(vals.values())
        assert got == min(c for c in vals if vals[c] == top)
    assert O.assign(np.ones(d), np.ones((C, d)), []) == -1


def check_assign_vote(fn) -> bool:
    """The majority-vote rule: most frequent neighbour community, then the
    larger score, then the lower id; worked cases, then brute force."""
    # tests/golden/worked_examples.json "assign_vote" (worked by hand there)
    g = GOLDEN["assign_vote"]
    cent = _arr(g["cent"])
    d = cent.shape[1]
    ok = True
    for kname, nb, expect in g["cases"]:
        ok &= fn(_arr(g[kname]), cent, nb) == expect
    rng = np.random.default_rng(23)
    C = 6
    for _ in range(200):
        cent = rng.integers(-2, 3, (C, d)).astype(np.float64)
        k = rng.integers(-2, 3, d).astype(np.float64)
        nb = [int(x) for x in rng.integers(-1, C, size=8)]
        got = fn(k, cent, nb)
        valid = [c for c in nb if c >= 0]
        if not valid:
            ok &= got == -1
            continue
        # brute force: every named community, compared on (votes, score, -id)
        best = max(set(valid), key=lambda c: (valid.count(c), float(np.dot(k, cent[c])), -c))
        ok &= got == best
    return bool(ok)


def test_assign_vote_worked_examples_and_bruteforce():
    assert check_assign_vote(O.assign_vote)


@pytest.mark.parametrize("rule", ["score", "vote"])
def test_multi_step_invariants_on_tiny_workload(rule):
    """Tiny workload, all steps: sinks present, no duplicate positions, the
    top community always selected, exactly one count changes per graph and
    step, and it changes by one; under the vote rule the chosen community
    holds the most neighbours."""
    wl = synth.WORKLOADS["tiny"]
    draw = synth.draw_cache(wl, device="cpu")
    K = draw.K.double().numpy()
    V = draw.V.double().numpy()
    C = int(draw.labels.max()) + 1
    states = {(0, 0): O.GraphState(draw.labels[0, 0], wl.T_cap, wl.S, C)}
    for step in range(wl.steps):
        q = synth.draw_queries(wl, draw, step).double().numpy()
        res = O.decode_step(wl.mode, wl.Hq, wl.Hkv, states, K, V, q, wl.budget)
        gs = res.graphs[(0, 0)]
        assert set(range(wl.S)) <= set(gs.tokens.tolist())
        assert len(np.unique(gs.tokens)) == len(gs.tokens)
        assert gs.selected[0] == O.rank(gs.scores, gs.cnt)[0]
        pos = wl.T + step
        kn, vn = synth.draw_new_tokens(wl, draw, step)
        K[:, :, pos] = kn.double().numpy()
        V[:, :, pos] = vn.double().numpy()
        before = O.centroids(K[0, 0, :states[(0, 0)].T], states[(0, 0)].members())[1]
        named = [int(states[(0, 0)].comm_of[p]) for p in gs.nbr]
        a = O.assign_step(wl.mode, wl.Hq, wl.Hkv, states, K, res, pos, rule=rule)
        after = O.centroids(K[0, 0, :states[(0, 0)].T], states[(0, 0)].members())[1]
        diff = after - before
        assert a[(0, 0)] in named
        if rule == "vote":
            assert named.count(a[(0, 0)]) == max(named.count(c) for c in named if c >= 0)
        assert diff.sum() == 1 and diff[a[(0, 0)]] == 1


# ----------------------------------------------------------------------------
# planted mistakes: each mutant must fail at least one pin
# ----------------------------------------------------------------------------

def _mut_select_high_id(scores, cnt, budget):
    order = sorted([c for c in range(len(cnt)) if cnt[c] > 0], key=lambda c: (-scores[c], -c))
    out, tot = [], 0
    for c in order:
        if tot + cnt[c] > budget:
            break
        out.append(c)
        tot += cnt[c]
    return out or order[:1]


def _mut_select_overshoot(scores, cnt, budget):
    order = O.rank(scores, cnt)
    out, tot = [], 0
    for c in order:
        out.append(c)
        tot += cnt[c]
        if tot >= budget:
            break
    return out


def _mut_select_no_floor(scores, cnt, budget):
    order = O.rank(scores, cnt)
    out, tot = [], 0
    for c in order:
        if tot + cnt[c] > budget:
            break
        out.append(c)
        tot += cnt[c]
    return out


def _mut_select_skip(scores, cnt, budget):
    out, tot = [], 0
    for c in O.rank(scores, cnt):
        if tot + cnt[c] <= budget:
            out.append(c)
            tot += cnt[c]
    return out or O.rank(scores, cnt)[:1]


def _mut_scores_mean(q, cent, cnt):
    q = np.atleast_2d(q)
    return np.where(cnt > 0, (cent @ q.T).mean(axis=1) / math.sqrt(q.shape[1]), -np.inf)


def _mut_scores_noscale(q, cent, cnt):
    q = np.atleast_2d(q)
    return np.where(cnt > 0, (cent @ q.T).max(axis=1), -np.inf)


def _mut_attention_noscale(q, K, V, positions):
    lg = K[positions] @ q
    w = np.exp(lg - lg.max())
    return (w[:, None] * V[positions]).sum(0) / w.sum()


def _mut_attention_transposed(q, K, V, positions):
    lg = V[positions] @ q / math.sqrt(len(q))
    w = np.exp(lg - lg.max())
    return (w[:, None] * K[positions]).sum(0) / w.sum()


def _mut_neighbours_with_sinks(q, K, positions, S, k=8):
    return O.neighbours(q, K, positions, 0, k)


def _mut_neighbours_high_pos(q, K, positions, S, k=8):
    pos = np.asarray([p for p in positions if p >= S])
    if len(pos) == 0:
        return pos
    lam = O.graph_logits(q, K, pos)
    order = sorted(range(len(pos)), key=lambda i: (-lam[i], -pos[i]))
    return pos[order[:k]]


def _mut_neighbours_first_head(q, K, positions, S, k=8):
    return O.neighbours(np.atleast_2d(q)[:1], K, positions, S, k)


def _mut_vote_distinct(k_new, cent, neighbour_comms):
    # repeats dropped: degenerates to the score rule
    return O.assign(k_new, cent, [c for c in neighbour_comms if c >= 0])


def _mut_vote_no_score(k_new, cent, neighbour_comms):
    # equal votes go to the lower id, ignoring the score
    valid = [int(c) for c in neighbour_comms if c >= 0]
    return min(set(valid), key=lambda c: (-valid.count(c), c)) if valid else -1


def _mut_vote_high_id(k_new, cent, neighbour_comms):
    valid = [int(c) for c in neighbour_comms if c >= 0]
    return max(set(valid), key=lambda c: (valid.count(c), float(np.dot(k_new, cent[c])), c)) if valid else -1


_REAL_TOKEN_SET = O.token_set


def _mut_token_set_no_sinks(selected, members, S):
    return _REAL_TOKEN_SET(selected, members, 0)


@pytest.mark.parametrize("mutant", [_mut_select_high_id, _mut_select_overshoot,
                                    _mut_select_no_floor, _mut_select_skip])
def test_pins_catch_select_mutants(mutant):
    assert not (check_select_worked(mutant) and check_select_bruteforce(mutant))


@pytest.mark.parametrize("mutant", [_mut_scores_mean, _mut_scores_noscale])
def test_pins_catch_score_mutants(mutant):
    assert not check_scores_closed_form(mutant)


@pytest.mark.parametrize("mutant", [_mut_attention_noscale, _mut_attention_transposed])
def test_pins_catch_attention_mutants(mutant):
    assert not check_attention_closed_form(mutant)


@pytest.mark.parametrize("mutant", [_mut_neighbours_with_sinks, _mut_neighbours_high_pos,
                                    _mut_neighbours_first_head])
def test_pins_catch_neighbour_mutants(mutant):
    assert not check_neighbours(mutant)


@pytest.mark.parametrize("mutant", [_mut_vote_distinct, _mut_vote_no_score, _mut_vote_high_id])
def test_pins_catch_vote_mutants(mutant):
    assert not check_assign_vote(mutant)


def test_pins_catch_dropped_sinks(monkeypatch):
    monkeypatch.setattr(O, "token_set", _mut_token_set_no_sinks)
    assert not check_dense_equivalence(O.decode_graph)


# ----------------------------------------------------------------------------
# the token graph at prefill: direct and co-attention edges
# ----------------------------------------------------------------------------

def check_edges_worked(direct_edges, coattention_edges) -> bool:
    # tests/golden/worked_examples.json "edges" (worked by hand there)
    g = GOLDEN["edges"]
    q = _arr(g["q"])[None]            # one head: [1, T, d]
    K = _arr(g["K"])
    d = direct_edges(q, K, g["S"], g["T"], k=g["k"])
    if [list(map(int, x)) for x in d] != g["direct"]:
        return False
    w = coattention_edges(d)
    return sorted([j, l, c] for (j, l), c in w.items()) == g["coattention"]


def _brute_direct(q_heads_seq, K, S, T, k=8):
    """Per query, the keys before it (sinks excluded) ranked by counting how
    many beat each one (logit, then lower position), the first k."""
    out = []
    for i in range(S, T):
        pos = list(range(S, i))
        lam = {p: max(float(np.dot(q_heads_seq[h, i], K[p])) for h in range(q_heads_seq.shape[0])) for p in pos}

        def better(a, b):
            return lam[a] > lam[b] or (lam[a] == lam[b] and a < b)

        rank = {p: sum(better(o, p) for o in pos) for p in pos}
        out.append([p for p in sorted(pos, key=lambda p: rank[p]) if rank[p] < k])
    return out


def check_edges_bruteforce(direct_edges, coattention_edges, trials=12, seed=29) -> bool:
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        H, T, S, d = int(rng.integers(1, 4)), int(rng.integers(2, 40)), int(rng.integers(0, 5)), 8
        S = min(S, T - 1)
        q = rng.integers(-1, 2, (H, T, d)).astype(np.float64)    # integer data: many ties
        K = rng.integers(-2, 3, (T, d)).astype(np.float64)
        K[:S] += 10.0                                             # sinks would win if they were keys
        got = [list(map(int, x)) for x in direct_edges(q, K, S, T)]
        if got != _brute_direct(q, K, S, T):
            return False
        # co-attention: the weight of each key pair is the number of lists
        # holding both; their total is the number of pairs over the lists
        w = coattention_edges([np.array(x) for x in got])
        for (j, l), c in w.items():
            if not (j < l and c == sum(1 for x in got if j in x and l in x)):
                return False
        if sum(w.values()) != sum(len(x) * (len(x) - 1) // 2 for x in got):
            return False
    return True


def test_edges_worked_example():
    assert check_edges_worked(O.direct_edges, O.coattention_edges)


def test_edges_bruteforce():
    assert check_edges_bruteforce(O.direct_edges, O.coattention_edges)


def _edges_with_sinks(q, K, S, T, k=8):
    return O.direct_edges(q, K, 0, T, k)[S:] if S <= T else []


def _edges_with_self(q, K, S, T, k=8):
    out = []
    for i in range(S, T):
        pos = np.arange(S, i + 1)
        lam = O.graph_logits(np.asarray(q)[:, i, :], K, pos)
        out.append(pos[np.lexsort((pos, -lam))[:k]])
    return out


def _edges_future_keys(q, K, S, T, k=8):
    out = []
    for i in range(S, T):
        pos = np.array([p for p in range(S, T) if p != i], dtype=np.int64)
        lam = O.graph_logits(np.asarray(q)[:, i, :], K, pos) if len(pos) else np.zeros(0)
        out.append(pos[np.lexsort((pos, -lam))[:k]] if len(pos) else pos)
    return out


def _edges_ties_high(q, K, S, T, k=8):
    out = []
    for i in range(S, T):
        pos = np.arange(S, i)
        lam = O.graph_logits(np.asarray(q)[:, i, :], K, pos) if len(pos) else np.zeros(0)
        out.append(pos[np.lexsort((-pos, -lam))[:k]] if len(pos) else pos)
    return out


def _coattention_ordered(direct):
    w = {}
    for lst in direct:
        for a in lst:
            for b in lst:
                if a != b:
                    w[(int(a), int(b))] = w.get((int(a), int(b)), 0) + 1
    return {key: c for key, c in w.items()}


@pytest.mark.parametrize("mutant", [_edges_with_sinks, _edges_with_self, _edges_future_keys, _edges_ties_high])
def test_pins_catch_edge_mutants(mutant):
    assert not (check_edges_worked(mutant, O.coattention_edges)
                and check_edges_bruteforce(mutant, O.coattention_edges))


def test_pins_catch_coattention_mutant():
    assert not (check_edges_worked(O.direct_edges, _coattention_ordered)
                and check_edges_bruteforce(O.direct_edges, _coattention_ordered))
