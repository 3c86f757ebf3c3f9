"""Plain CPU oracle of the CommunityKV decode step, in float64.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import or run this module; the library and
its Python binding never do, and nothing here is shared with the CUDA path.

It follows "CommunityKV: Efficient Long-Context Decoding via Graph
Partitioning" as the pages state it (rit.work summary, section "A graph of
tokens replaces re-clustering"; omanscience.com abstract), step by step and
in that order:

1. Sink tokens (the first S positions) are not part of any community and are
   always added to the selected context (rit.work, "A graph of tokens ...",
   paragraph on the two edge types).
2. A centre is computed for every community (same section, paragraph on
   Leiden); read here as the mean of the member keys.
3. At each decode step the query is compared with the centres only.  Rule used
   (the pages leave it open): the score of community c for a graph is
   max over the graph's query heads h of q_h . c / sqrt(d).
4. The top communities are loaded up to a token budget (same paragraph, and
   section "Speed-up depends on how many graphs ..." for the small active
   budget).  Rule used: rank by (score descending, id ascending); take the
   longest ranked prefix whose total size is at most the budget, but at least
   the top community.  Sinks are outside the budget.
5. Exact softmax attention runs over the selected tokens only, read from the
   full cache, which is never pruned (same section, next paragraph).
6. A new token joins one neighbouring community and one centre is updated, at
   a cost independent of the context length (same section, last paragraph;
   the abstract calls the rule constant-time).  Rules used: the neighbour set is the
   communities of the 8 non-sink selected tokens with the largest graph logit
   (max over the graph's heads of q_h . k_t / sqrt(d); ties to the lower
   position); the token joins the candidate c maximising k_new . c / sqrt(d)
   (ties to the lower id), or, under the other reading (assign_vote), the
   community holding the most of the 8 neighbours, ties to the larger
   k_new . c / sqrt(d) and then the lower id.
7. At prefill (before decoding), the token graph the partition is computed
   from: direct edges from a query to the keys it attends most, and
   co-attention edges between keys attended together, with the sinks kept
   out (direct_edges, coattention_edges; the partition itself is not built).

Every centre is recomputed from the member lists whenever it is needed; the
oracle never updates a mean incrementally.  Pins: see tests/test_oracle.py
and the hand-worked cases in tests/golden/worked_examples.json; every
function here has one.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

NEIGHBOURS = 8


# ----------------------------------------------------------------------------
# one graph: membership state
# ----------------------------------------------------------------------------

class GraphState:
    """Community membership of one graph (one (sequence, KV group) or
    (sequence, query head) pair).  ``comm_of[t]`` is the community of position
    t, -1 for sinks and for positions not yet written."""

    def __init__(self, labels: np.ndarray, T_cap: int, S: int, C: int):
        labels = np.asarray(labels)
        self.T = int(labels.shape[0])
        self.S = int(S)
        self.C = int(C)
        self.comm_of = np.full(int(T_cap), -1, dtype=np.int64)
        self.comm_of[: self.T] = labels
        if np.any(self.comm_of[: self.S] != -1):
            raise ValueError("sink positions must carry label -1")
        rest = self.comm_of[self.S: self.T]
        if rest.size and (rest.min() < 0 or rest.max() >= self.C):
            raise ValueError("labels must lie in [0, C) outside the sinks")

    def members(self) -> List[np.ndarray]:
        """Ascending member positions of every community."""
        out = []
        for c in range(self.C):
            out.append(np.flatnonzero(self.comm_of[: self.T] == c))
        return out

    def join(self, pos: int, c: int) -> None:
        """Position ``pos`` (just appended) joins community ``c`` (-1: none)."""
        if pos != self.T:
            raise ValueError("tokens are appended in order")
        self.comm_of[pos] = c
        self.T += 1

    def copy(self) -> "GraphState":
        g = GraphState.__new__(GraphState)
        g.T, g.S, g.C = self.T, self.S, self.C
        g.comm_of = self.comm_of.copy()
        return g


# ----------------------------------------------------------------------------
# the steps
# ----------------------------------------------------------------------------

def centroids(K: np.ndarray, members: Sequence[np.ndarray]):
    """Step 2: cent_c = mean of the member keys; cnt_c = member count.
    Empty communities get a zero row and count 0."""
    K = np.asarray(K, dtype=np.float64)
    C = len(members)
    cent = np.zeros((C, K.shape[1]), dtype=np.float64)
    cnt = np.zeros(C, dtype=np.int64)
    for c, m in enumerate(members):
        cnt[c] = len(m)
        if len(m):
            cent[c] = K[m].sum(axis=0) / len(m)
    return cent, cnt


def community_scores(q_heads: np.ndarray, cent: np.ndarray, cnt: np.ndarray) -> np.ndarray:
    """Step 3: s_c = max over the graph's heads of q_h . cent_c / sqrt(d);
    -inf for empty communities."""
    q_heads = np.atleast_2d(np.asarray(q_heads, dtype=np.float64))
    d = q_heads.shape[1]
    s = np.full(len(cnt), -np.inf)
    for c in range(len(cnt)):
        if cnt[c] > 0:
            s[c] = max(float(np.dot(q, cent[c])) for q in q_heads) / math.sqrt(d)
    return s


def rank(scores: np.ndarray, cnt: np.ndarray) -> List[int]:
    """Non-empty community ids ordered by (score descending, id ascending)."""
    ids = [c for c in range(len(cnt)) if cnt[c] > 0]
    return sorted(ids, key=lambda c: (-scores[c], c))


def select(scores: np.ndarray, cnt: np.ndarray, budget: int) -> List[int]:
    """Step 4: the longest ranked prefix with total size <= budget, and at
    least the top-ranked community.  Returned in rank order."""
    order = rank(scores, cnt)
    chosen: List[int] = []
    total = 0
    for c in order:
        if total + int(cnt[c]) > budget:
            break
        chosen.append(c)
        total += int(cnt[c])
    if not chosen and order:
        chosen = [order[0]]
    return chosen


def token_set(selected: Sequence[int], members: Sequence[np.ndarray], S: int) -> np.ndarray:
    """Steps 1 and 4: sinks plus every member of the selected communities,
    as ascending positions."""
    parts = [np.arange(S, dtype=np.int64)] + [members[c] for c in selected]
    return np.sort(np.concatenate(parts)) if parts else np.zeros(0, dtype=np.int64)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, positions: np.ndarray) -> np.ndarray:
    """Step 5: exact softmax attention of one query head over the given cache
    positions.  An empty set gives a zero vector."""
    q = np.asarray(q, dtype=np.float64)
    if len(positions) == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    Kp = np.asarray(K[positions], dtype=np.float64)
    Vp = np.asarray(V[positions], dtype=np.float64)
    logits = Kp @ q / math.sqrt(q.shape[0])
    w = np.exp(logits - logits.max())
    return (w[:, None] * Vp).sum(axis=0) / w.sum()


def graph_logits(q_heads: np.ndarray, K: np.ndarray, positions: np.ndarray) -> np.ndarray:
    """lambda_t = max over the graph's heads of q_h . k_t / sqrt(d)."""
    q_heads = np.atleast_2d(np.asarray(q_heads, dtype=np.float64))
    Kp = np.asarray(K[positions], dtype=np.float64)
    return (Kp @ q_heads.T).max(axis=1) / math.sqrt(q_heads.shape[1])


def neighbours(q_heads: np.ndarray, K: np.ndarray, positions: np.ndarray, S: int,
               k: int = NEIGHBOURS) -> np.ndarray:
    """Step 6, first half: the k non-sink selected positions with the largest
    graph logit, ties to the lower position, best first."""
    pos = np.asarray([p for p in positions if p >= S], dtype=np.int64)
    if len(pos) == 0:
        return pos
    lam = graph_logits(q_heads, K, pos)
    order = sorted(range(len(pos)), key=lambda i: (-lam[i], pos[i]))
    return pos[order[:k]]


def assign(k_new: np.ndarray, cent: np.ndarray, candidates: Sequence[int]) -> int:
    """Step 6, second half: the candidate community maximising
    k_new . cent_c / sqrt(d), ties to the lower id; -1 without candidates."""
    k_new = np.asarray(k_new, dtype=np.float64)
    best, best_s = -1, -np.inf
    for c in sorted(set(int(x) for x in candidates)):
        s = float(np.dot(k_new, cent[c])) / math.sqrt(k_new.shape[0])
        if best < 0 or s > best_s:
            best, best_s = c, s
    return best


def assign_vote(k_new: np.ndarray, cent: np.ndarray, neighbour_comms: Sequence[int]) -> int:
    """Step 6, second half, the alternative "graph-like" rule (the pages say
    only that the token joins a suitable neighbouring community): the
    community holding the most of the 8 neighbours wins; among equally
    frequent ones the larger k_new . cent_c / sqrt(d), then the lower id;
    -1 without candidates.  neighbour_comms lists each neighbour's community
    (repeats count)."""
    k_new = np.asarray(k_new, dtype=np.float64)
    votes = {}
    for c in neighbour_comms:
        c = int(c)
        if c >= 0:
            votes[c] = votes.get(c, 0) + 1
    best, best_key = -1, None
    for c in sorted(votes):
        s = float(np.dot(k_new, cent[c])) / math.sqrt(k_new.shape[0])
        key = (votes[c], s)
        if best < 0 or key > best_key:
            best, best_key = c, key
    return best


# ----------------------------------------------------------------------------
# the token graph at prefill (the input of the partition, which is not built)
# ----------------------------------------------------------------------------

def direct_edges(q_heads_seq: np.ndarray, K: np.ndarray, S: int, T: int,
                 k: int = NEIGHBOURS) -> List[np.ndarray]:
    """Direct edges of the prefill token graph (rit.work summary, section "A
    graph of tokens replaces re-clustering", paragraph 3: a query that pays a
    key much attention links the two; the first tokens are kept out of the
    graph).  Reading used: for every query position i in [S, T), the k key
    positions j in [S, i) with the largest graph logit
    max over the graph's heads of q_{h,i} . k_j / sqrt(d) (the rule of the
    decode-time neighbours), ties to the lower position, best first.
    q_heads_seq: [heads, >=T, d] (the graph's query heads over the prefill);
    K: [>=T, d].  Returns one array per query position, indexed by i - S."""
    return [direct_edges_at(q_heads_seq, K, S, i, k) for i in range(S, T)]


def direct_edges_at(q_heads_seq: np.ndarray, K: np.ndarray, S: int, i: int, k: int = NEIGHBOURS) -> np.ndarray:
    """The direct edges of query position i alone (see direct_edges)."""
    pos = np.arange(S, i, dtype=np.int64)
    if len(pos) == 0:
        return pos
    lam = graph_logits(np.asarray(q_heads_seq, dtype=np.float64)[:, i, :], K, pos)
    order = np.lexsort((pos, -lam))   # logit descending, then position ascending
    return pos[order[:k]]


def coattention_edges(direct: Sequence[np.ndarray]) -> Dict[tuple, int]:
    """Co-attention edges of the prefill token graph (same paragraph: keys
    that are looked at together are linked).  Reading used: every pair of
    keys j < l that appear in the same query's direct edges is linked, with
    the number of such queries as its weight."""
    w: Dict[tuple, int] = {}
    for lst in direct:
        ps = sorted(int(p) for p in lst)
        for a in range(len(ps)):
            for b in range(a + 1, len(ps)):
                w[(ps[a], ps[b])] = w.get((ps[a], ps[b]), 0) + 1
    return w


# ----------------------------------------------------------------------------
# a whole decode step over a batch
# ----------------------------------------------------------------------------

def graph_heads(mode: str, g: int, Hq: int, Hkv: int) -> List[int]:
    gq = Hq // Hkv
    return list(range(g * gq, (g + 1) * gq)) if mode == "group" else [g]


def graph_kv_head(mode: str, g: int, Hq: int, Hkv: int) -> int:
    return g if mode == "group" else g // (Hq // Hkv)


@dataclass
class GraphStep:
    scores: np.ndarray
    cnt: np.ndarray
    cent: np.ndarray
    selected: List[int]
    tokens: np.ndarray
    nbr: np.ndarray
    assigned: Optional[int] = None


@dataclass
class StepResult:
    out: Dict[tuple, np.ndarray] = field(default_factory=dict)      # (b, h) -> o_h
    graphs: Dict[tuple, GraphStep] = field(default_factory=dict)    # (b, g) -> GraphStep


def decode_graph(mode: str, Hq: int, Hkv: int, b: int, g: int, state: GraphState,
                 K: np.ndarray, V: np.ndarray, q: np.ndarray, budget: int,
                 selected: Optional[Sequence[int]] = None):
    """Steps 2-5 plus the neighbour set for one graph.  K, V: [Hkv, >=T, d]
    of sequence b; q: [Hq, d].  ``selected`` overrides step 4 (used to
    re-check attention on another implementation's selection).
    Returns (GraphStep, {head: o_h})."""
    kvh = graph_kv_head(mode, g, Hq, Hkv)
    heads = graph_heads(mode, g, Hq, Hkv)
    Kh, Vh = K[kvh], V[kvh]
    members = state.members()
    cent, cnt = centroids(Kh[: state.T], members)
    s = community_scores(q[heads], cent, cnt)
    sel = list(select(s, cnt, budget) if selected is None else selected)
    toks = token_set(sel, members, state.S)
    outs = {h: attention(q[h], Kh, Vh, toks) for h in heads}
    nbr = neighbours(q[heads], Kh, toks, state.S)
    return GraphStep(s, cnt, cent, sel, toks, nbr), outs


def decode_step(mode: str, Hq: int, Hkv: int, states: Dict[tuple, GraphState],
                K: np.ndarray, V: np.ndarray, q: np.ndarray, budget: int,
                units: Optional[Sequence[tuple]] = None) -> StepResult:
    """One decode step (steps 2-5 and the neighbour sets) for the listed
    (b, g) units, by default all of them.  K, V: [B, Hkv, >=T, d]; q: [B, Hq, d]."""
    res = StepResult()
    for (b, g) in (units if units is not None else sorted(states)):
        gs, outs = decode_graph(mode, Hq, Hkv, b, g, states[(b, g)], K[b], V[b], q[b], budget)
        res.graphs[(b, g)] = gs
        for h, o in outs.items():
            res.out[(b, h)] = o
    return res


def assign_step(mode: str, Hq: int, Hkv: int, states: Dict[tuple, GraphState],
                K: np.ndarray, res: StepResult, pos: int,
                units: Optional[Sequence[tuple]] = None, rule: str = "score") -> Dict[tuple, int]:
    """Step 6 for the token written at ``pos`` (the cache row is already
    there): each graph's new token joins the best neighbouring community,
    by score (``assign``) or by majority vote (``assign_vote``)."""
    out = {}
    for (b, g) in (units if units is not None else sorted(res.graphs)):
        st = states[(b, g)]
        gs = res.graphs[(b, g)]
        kvh = graph_kv_head(mode, g, Hq, Hkv)
        cand = [int(st.comm_of[p]) for p in gs.nbr]
        cand = [c for c in cand if c >= 0]
        pick = assign_vote if rule == "vote" else assign
        c_star = pick(K[b, kvh, pos], gs.cent, cand)
        st.join(pos, c_star)
        gs.assigned = c_star
        out[(b, g)] = c_star
    return out
