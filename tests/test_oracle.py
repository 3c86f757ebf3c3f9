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
import math

import numpy as np
import pytest
import torch

import oracle.ckv_oracle as O
import synth


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
    # d = 4: q = (2,0,0,0); k1 = (ln 3,0,0,0) -> logit ln 3; k2 = 0 -> logit 0;
    # weights 3/4, 1/4; o = 3/4 (1,0,0,0) + 1/4 (0,4,0,0) = (0.75, 1, 0, 0)
    K = np.array([[math.log(3.0), 0, 0, 0], [0, 0, 0, 0]], dtype=np.float64)
    V = np.array([[1, 0, 0, 0], [0, 4, 0, 0]], dtype=np.float64)
    o = attention(np.array([2.0, 0, 0, 0]), K, V, np.array([0, 1]))
    return np.allclose(o, [0.75, 1.0, 0.0, 0.0], atol=1e-14)


def check_scores_closed_form(community_scores):
    # d = 4, two heads; community 0: dots 2 and -1 -> max 2 -> 2/sqrt(4) = 1.0
    # community 1: dots -2 and 3 -> 1.5; community 2 empty -> -inf
    q = np.array([[2.0, 0, 0, 0], [0, -1.0, 0, 0]])
    cent = np.array([[1.0, 1, 0, 0], [-1.0, -3, 0, 0], [5.0, 5, 5, 5]])
    s = community_scores(q, cent, np.array([3, 2, 0]))
    return s[0] == 1.0 and s[1] == 1.5 and s[2] == -np.inf


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
    s = np.array([3.0, 1.0, 2.0, 2.0])
    n = np.array([5, 4, 3, 2])
    # rank: 0 (3), 2 (2, lower id), 3 (2), 1 (1); prefix sizes 5, 8, 10, 14
    return (select(s, n, 10) == [0, 2, 3] and select(s, n, 9) == [0, 2]
            and select(s, n, 4) == [0] and select(s, n, 14) == [0, 2, 3, 1]
            and select(s, n, 0) == [0])


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
    d = 4
    cent = np.array([[1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 0], [2, 0, 0, 0]], dtype=np.float64)
    k = np.array([1.0, 0.5, 0.0, 0.0])
    ok = True
    # worked by hand: votes {2: 3, 0: 2, 1: 2} -> 2 wins although its score (0) is the lowest
    ok &= fn(k, cent, [2, 0, 2, 1, 0, 2, 1, -1]) == 2
    # equal votes {0: 2, 3: 2}: scores 1/2 and 2/2 -> 3
    ok &= fn(k, cent, [0, 3, 0, 3]) == 3
    # equal votes and equal scores (cent[1] and cent[2] seen from k2) -> the lower id
    k2 = np.array([0.0, 1.0, 1.0, 0.0])
    ok &= fn(k2, cent, [2, 1]) == 1
    ok &= fn(k, cent, [-1, -1]) == -1 and fn(k, cent, []) == -1
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
