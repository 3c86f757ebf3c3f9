"""Drive the CUDA path through the C ABI and compare it with the CPU oracle.

Comparison rules:
  * selection: the ranked community list must equal the oracle's, except for
    communities whose oracle score lies within BAND of a cut score (the last
    selected or first unselected); the GPU's own set must still respect the
    budget rule and its order must agree with the oracle scores up to BAND;
  * token list: bit-exact as a set against the oracle token set of the GPU's
    own selection (sinks once each, no duplicates);
  * outputs: the oracle recomputes attention on the GPU's own selection,
    max-abs within 2e-3 for bf16 K/V and 1e-5 for fp32 K/V;
  * neighbours: equal to the oracle's on the same token set, except for
    positions whose logit lies within BAND of the 8th;
  * assignment: equal, or the two candidates' oracle scores within BAND (then
    the oracle adopts the GPU's choice and the resync is counted); under the
    vote rule the two must also hold the same number of neighbours;
  * counts bit-exact and centres within 1e-5 of the oracle's recomputed means.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import oracle.ckv_oracle as O
import synth
from graph_community_sparse_b200.layer import LayerState

BAND = 1e-5
TOL = {"bf16": 2e-3, "f32": 1e-5}
CENT_TOL = 1e-5


@dataclass
class Report:
    steps: int = 0
    units_checked: int = 0
    band_selections: int = 0
    band_neighbours: int = 0
    resyncs: int = 0
    rule_decisive: int = 0   # vote rule: units where the score rule would have chosen otherwise
    max_out_err: float = 0.0
    max_cent_err: float = 0.0
    notes: List[str] = field(default_factory=list)


def check_selection(gpu_sel: Sequence[int], scores: np.ndarray, cnt: np.ndarray, budget: int,
                    band: float = BAND) -> bool:
    """True when exact, False when tolerated within the band; raises otherwise."""
    ref = O.select(scores, cnt, budget)
    gpu_sel = [int(c) for c in gpu_sel]
    if gpu_sel == ref:
        return True
    order = O.rank(scores, cnt)
    k = len(ref)
    cuts = [scores[ref[-1]]] if ref else []
    if k < len(order):
        cuts.append(scores[order[k]])
    diff = set(gpu_sel) ^ set(ref)
    for c in diff:
        assert cuts and min(abs(scores[c] - v) for v in cuts) <= band, \
            f"community {c} (score {scores[c]}) differs outside the tie band; cuts {cuts}"
    assert len(set(gpu_sel)) == len(gpu_sel), "duplicate community in selection"
    tot = int(sum(cnt[c] for c in gpu_sel))
    assert tot <= budget or len(gpu_sel) == 1, "GPU selection breaks the budget"
    for a, b in zip(gpu_sel, gpu_sel[1:]):
        assert scores[a] >= scores[b] - band, "GPU rank order disagrees with the oracle scores"
    return False


def check_neighbours(gpu_nbr: Sequence[int], qh: np.ndarray, Kh: np.ndarray, toks: np.ndarray, S: int,
                     band: float = BAND) -> bool:
    ref = [int(p) for p in O.neighbours(qh, Kh, toks, S)]
    got = [int(p) for p in gpu_nbr if p >= 0]
    assert all(p < 0 for p in list(gpu_nbr)[len(got):]), "-1 padding must come last"
    if got == ref:
        return True
    assert len(got) == len(ref), f"neighbour count {len(got)} != {len(ref)}"
    assert len(set(got)) == len(got)
    tset = set(int(t) for t in toks)
    assert all(p in tset and p >= S for p in got), "neighbour outside the non-sink selection"
    allp = np.asarray(sorted(set(got) | set(ref)), dtype=np.int64)
    lam = dict(zip(allp.tolist(), O.graph_logits(qh, Kh, allp).tolist()))
    v8 = lam[ref[-1]]
    for p in set(got) ^ set(ref):
        assert abs(lam[p] - v8) <= band, f"neighbour {p} differs outside the tie band"
    for a, b in zip(got, got[1:]):
        assert lam[a] >= lam[b] - band
    return False


class Case:
    """One synthetic layer on the GPU plus the oracle's membership state."""

    def __init__(self, wl: synth.Workload, device="cuda", Cmax: Optional[int] = None,
                 max_tail: Optional[int] = None, tok_cap: Optional[int] = None,
                 labels: Optional[np.ndarray] = None, layer: int = 0):
        self.wl = wl
        self.layer_idx = layer
        self.draw = synth.draw_cache(wl, layer=layer, device=device, labels=labels)
        labs = self.draw.labels
        self.C = int(labs.max()) + 1 if labs.size else 1
        self.Cmax = Cmax or max(self.C, 1)
        self.U = wl.B * wl.G
        mt = wl.steps if max_tail is None else max_tail
        self.st = LayerState(self.draw.K, self.draw.V, wl.Hq, wl.mode, wl.S, self.Cmax, mt, tok_cap,
                             rule=wl.assign_rule)
        lab_t = torch.from_numpy(labs.reshape(self.U, wl.T).astype(np.int32)).to(device)
        self.st.build(lab_t, wl.T)
        self.states: Dict[tuple, O.GraphState] = {}
        self._kv: Dict[tuple, tuple] = {}
        self.step_idx = 0
        self.T_step = self.st.T

    # oracle-side helpers -------------------------------------------------
    def state(self, b: int, g: int) -> O.GraphState:
        """Oracle membership of one unit.  A unit first checked after some
        updates starts from the labels plus the joins the GPU made meanwhile
        (those joins were not checked; later counts and centres are)."""
        if (b, g) not in self.states:
            st = O.GraphState(self.draw.labels[b, g], self.st.cache.T_cap, self.wl.S, self.Cmax)
            # the cache length when the current step began (a fused step has
            # already appended its own token when the checks run)
            T_known = min(self.st.T, self.T_step)
            if T_known > self.wl.T:
                u = b * self.wl.G + g
                joined = self.st.graph.comm_of[u, self.wl.T: T_known].cpu().numpy()
                for i, c in enumerate(joined):
                    st.join(self.wl.T + i, int(c))
            self.states[(b, g)] = st
        return self.states[(b, g)]

    def kv(self, b: int, kvh: int):
        """fp64 copies of one (sequence, KV head) slice (refreshed after appends)."""
        key = (b, kvh, self.st.T)
        if key not in self._kv:
            self._kv = {k: v for k, v in self._kv.items() if k[2] == self.st.T}
            K = self.st.K[b, kvh, : self.st.T].double().cpu().numpy()
            V = self.st.V[b, kvh, : self.st.T].double().cpu().numpy()
            self._kv[key] = (K, V)
        return self._kv[key]

    def heads(self, g: int) -> List[int]:
        return O.graph_heads(self.wl.mode, g, self.wl.Hq, self.wl.Hkv)

    def kv_head(self, g: int) -> int:
        return O.graph_kv_head(self.wl.mode, g, self.wl.Hq, self.wl.Hkv)

    # one step ----------------------------------------------------------------
    def step(self, budget: int, units: Optional[Sequence[tuple]] = None, rep: Optional[Report] = None,
             update: Optional[bool] = None, check_all_units: bool = True, fused: bool = False) -> Report:
        """One decode step, checked.  fused=True runs the attention and the
        update as the benchmark does (ckv_sparse_decode_append, one call);
        otherwise ckv_sparse_decode, then ckv_append_assign."""
        wl = self.wl
        rep = rep or Report()
        update = wl.update if update is None else update
        self.T_step = self.st.T
        q = synth.draw_queries(wl, self.draw, self.step_idx, self.layer_idx)
        fused_assigned = None
        if fused and update:
            self.st.select(q, budget)
            cnt_before = self.st.graph.cnt.clone()  # the update below changes the counts
            kn, vn = synth.draw_new_tokens(wl, self.draw, self.step_idx, self.layer_idx)
            pos = self.st.T
            out = self.st.attend_append(q, kn, vn).clone()
            fused_assigned = self.st.assigned.clone()
        else:
            out = self.st.decode(q, budget).clone()
            cnt_before = None
        torch.cuda.synchronize()
        sel_comm = self.st.sel.sel_comm.cpu().numpy()
        n_sel = self.st.sel.n_sel.cpu().numpy()
        sel_tok = self.st.sel.sel_tok.cpu().numpy()
        n_tok = self.st.sel.n_tok.cpu().numpy()
        prefix = self.st.sel.unit_prefix.cpu().numpy()
        tok_prefix = self.st.sel.tok_prefix.cpu().numpy()
        tail_sel = self.st.sel.tail_sel.cpu().numpy()
        nbr = self.st.nbr8.cpu().numpy()
        cnt_gpu = (cnt_before if cnt_before is not None else self.st.graph.cnt).cpu().numpy()
        assert prefix[0] == 0 and np.array_equal(np.diff(prefix), n_tok), "unit_prefix is not the scan of n_tok"
        if check_all_units:
            # cheap invariants on every unit
            for u in range(self.U):
                sel = sel_comm[u, : n_sel[u]]
                expect = wl.S + int(cnt_gpu[u, sel].sum())
                assert n_tok[u] == min(expect, self.st.sel.desc.tok_cap), (u, n_tok[u], expect)
                assert np.array_equal(sel_tok[u, : min(wl.S, n_tok[u])], np.arange(min(wl.S, n_tok[u])))
        qn = q.double().cpu().numpy()
        units = units if units is not None else [(b, g) for b in range(wl.B) for g in range(wl.G)]
        cand_cache = {}
        for (b, g) in units:
            u = b * wl.G + g
            st = self.state(b, g)
            K, V = self.kv(b, self.kv_head(g))
            heads = self.heads(g)
            members = st.members()
            cent, cnt = O.centroids(K, members)
            assert np.array_equal(cnt_gpu[u], cnt), f"unit {u}: counts differ"
            scores = O.community_scores(qn[b, heads], cent, cnt)
            gsel = sel_comm[u, : n_sel[u]].tolist()
            if not check_selection(gsel, scores, cnt, budget):
                rep.band_selections += 1
            toks = O.token_set(gsel, members, wl.S)
            # the list's runs: build-time member counts of the ranked
            # communities, cumulated; then the tail members' communities in
            # tail (position) order
            T0 = wl.T
            built = np.bincount(st.comm_of[wl.S: T0][st.comm_of[wl.S: T0] >= 0], minlength=self.Cmax)
            runs = np.concatenate([[0], np.cumsum(built[gsel])]) if gsel else np.zeros(1, dtype=np.int64)
            assert np.array_equal(tok_prefix[u, : len(gsel) + 1], runs), f"unit {u}: run offsets differ"
            tails = [int(st.comm_of[t]) for t in range(T0, st.T) if int(st.comm_of[t]) in set(gsel)]
            assert np.array_equal(tail_sel[u, : len(tails)], tails), f"unit {u}: tail communities differ"
            gt = sel_tok[u, : n_tok[u]]
            tok_cap = self.st.sel.desc.tok_cap
            if len(toks) <= tok_cap:
                assert len(gt) == len(toks) and np.array_equal(np.sort(gt), toks), f"unit {u}: token set differs"
            else:
                assert len(gt) == tok_cap and len(np.unique(gt)) == tok_cap and set(gt.tolist()) <= set(toks.tolist())
                toks = np.sort(gt)
            for h in heads:
                o = O.attention(qn[b, h], K, V, toks)
                err = float(np.abs(o - out[b, h].double().cpu().numpy()).max())
                rep.max_out_err = max(rep.max_out_err, err)
                assert err <= TOL[wl.dtype], f"unit {u} head {h}: max abs err {err}"
            if not check_neighbours(nbr[u], qn[b, heads], K, toks, wl.S):
                rep.band_neighbours += 1
            cand_cache[(b, g)] = cent
            rep.units_checked += 1
        if update:
            if fused_assigned is not None:
                assigned = fused_assigned.cpu().numpy()
            else:
                kn, vn = synth.draw_new_tokens(wl, self.draw, self.step_idx, self.layer_idx)
                pos = self.st.T
                assigned = self.st.append(kn, vn).cpu().numpy()
            torch.cuda.synchronize()
            for (b, g) in units:
                u = b * wl.G + g
                st = self.state(b, g)
                cent = cand_cache[(b, g)]
                kvh = self.kv_head(g)
                k_new = kn[b, kvh].double().cpu().numpy()
                named = [int(st.comm_of[p]) for p in nbr[u] if p >= 0 and st.comm_of[p] >= 0]
                cands = sorted(set(named))
                vote = wl.assign_rule == "vote"
                ref = O.assign_vote(k_new, cent, named) if vote else O.assign(k_new, cent, cands)
                if vote and ref != O.assign(k_new, cent, cands):
                    rep.rule_decisive += 1
                got = int(assigned[u])
                if got != ref:
                    assert got in cands, f"unit {u}: assigned {got} not a candidate {cands}"
                    if vote:
                        assert named.count(got) == named.count(ref), f"unit {u}: {got} has fewer votes than {ref}"
                    sr = float(np.dot(k_new, cent[ref])) / math.sqrt(wl.d)
                    sg = float(np.dot(k_new, cent[got])) / math.sqrt(wl.d)
                    assert abs(sr - sg) <= BAND, f"unit {u}: assignment {got} vs {ref}"
                    rep.resyncs += 1
                st.join(pos, got)
            checked = set(units)
            for (b, g), st in self.states.items():
                if (b, g) not in checked:       # tracked but not checked this step
                    st.join(pos, int(assigned[b * wl.G + g]))
            # counts and centres after the update
            cnt_gpu = self.st.graph.cnt.cpu().numpy()
            cent_gpu = self.st.graph.cent.cpu().numpy()
            for (b, g) in units:
                u = b * wl.G + g
                st = self.state(b, g)
                K, _ = self.kv(b, self.kv_head(g))
                cent, cnt = O.centroids(K, st.members())
                assert np.array_equal(cnt_gpu[u], cnt), f"unit {u}: counts differ after update"
                err = float(np.abs(cent_gpu[u, : self.Cmax] - cent).max()) if self.Cmax else 0.0
                rep.max_cent_err = max(rep.max_cent_err, err)
                assert err <= CENT_TOL, f"unit {u}: centroid error {err}"
        self.step_idx += 1
        rep.steps += 1
        return rep

    def check_build(self, units: Optional[Sequence[tuple]] = None) -> float:
        """CSR, counts and centres right after the build."""
        wl = self.wl
        offs = self.st.graph.offs.cpu().numpy()
        tok = self.st.graph.tok.cpu().numpy()
        cnt = self.st.graph.cnt.cpu().numpy()
        num = self.st.graph.num_comm.cpu().numpy()
        cent = self.st.graph.cent.cpu().numpy()
        comm_of = self.st.graph.comm_of.cpu().numpy()
        worst = 0.0
        units = units if units is not None else [(b, g) for b in range(wl.B) for g in range(wl.G)]
        for (b, g) in units:
            u = b * wl.G + g
            lab = self.draw.labels[b, g]
            assert np.array_equal(comm_of[u, : wl.T], lab)
            assert np.all(comm_of[u, wl.T:] == -1)
            present = lab[lab >= 0]
            assert num[u] == (int(present.max()) + 1 if present.size else 0)
            bc = np.bincount(present, minlength=self.Cmax)
            assert np.array_equal(cnt[u], bc)
            assert offs[u, 0] == 0 and np.array_equal(np.diff(offs[u]), bc)
            # members sorted by (community, position): the stable order of positions
            order = np.argsort(np.where(lab >= 0, lab, self.Cmax + 1), kind="stable")[: present.size]
            assert np.array_equal(tok[u, : present.size], order)
            K, _ = self.kv(b, self.kv_head(g))
            ref, _ = O.centroids(K, self.state(b, g).members())
            err = float(np.abs(cent[u] - ref).max())
            worst = max(worst, err)
            assert err <= CENT_TOL, f"unit {u}: centroid error {err}"
        return worst
