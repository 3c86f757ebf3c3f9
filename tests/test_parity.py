"""CUDA path (through the C ABI) against the CPU oracle, on a B200.

Small cases run every unit through the oracle, span many warps' slices and
ragged tails, and cover both graph modes, both dtypes, d = 64/128 and every
supported GQA ratio.  Edge cases: budget 0 (the top community is still
taken), a budget covering everything (equals dense attention), no sinks, a
single community, empty community ids, a full tail, a token list longer than
its capacity, and labels the build must reject.
"""
import numpy as np
import pytest
import torch

import graph_community_sparse_b200 as ckv
import oracle.ckv_oracle as O
import synth
from parity_util import BAND, TOL, Case, Report

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["qwen3_8b_32k"]


def small(key, index, **kw):
    args = dict(key=key, title=key, index=index, B=2, T=3000, budgets=(300,), steps=3, update=True)
    args.update(kw)
    return BASE.replace(**args)


SHAPES = [
    synth.WORKLOADS["tiny"],
    small("bf16_group_gq4", 20),
    small("bf16_head_gq1", 21, mode="head", T=2500, budgets=(200,)),
    small("bf16_d64_gq2", 22, d=64, Hq=16, Hkv=8),
    small("f32_d128_gq8", 23, dtype="f32", Hq=32, Hkv=4, budgets=(500,)),
    small("bf16_gq1_mha", 24, Hq=8, Hkv=8),
    small("f32_d64_head", 25, dtype="f32", d=64, mode="head", Hq=8, Hkv=4),
    small("bf16_zipf", 26, sizes="zipf", T=6000, budgets=(700,), update=False),
    small("bf16_spans", 27, layout="spans"),
    small("bf16_d128_gq8", 28, Hq=32, Hkv=4),
    small("bf16_d64_gq4_head", 29, d=64, mode="head", Hq=16, Hkv=4, budgets=(150,)),
    small("bf16_group_vote", 44, assign_rule="vote", steps=4),
    small("f32_d64_head_vote", 45, dtype="f32", d=64, mode="head", Hq=8, Hkv=4, assign_rule="vote"),
]


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("wl", SHAPES, ids=[w.key for w in SHAPES])
def test_build_matches_oracle(wl):
    case = Case(wl)
    assert case.check_build() <= 1e-5
    assert int(case.st.graph.dev_err.item()) == 0


@pytest.mark.parametrize("wl", SHAPES, ids=[w.key for w in SHAPES])
def test_steps_match_oracle(wl):
    case = Case(wl)
    K0 = case.st.K[:, :, : wl.T].clone()
    V0 = case.st.V[:, :, : wl.T].clone()
    rep = Report()
    for _ in range(wl.steps):
        case.step(wl.budget, rep=rep)
    assert rep.units_checked == wl.steps * wl.B * wl.G
    assert rep.max_out_err <= TOL[wl.dtype]
    # the library never writes the cache
    assert torch.equal(case.st.K[:, :, : wl.T], K0) and torch.equal(case.st.V[:, :, : wl.T], V0)
    assert int(case.st.graph.dev_err.item()) == 0
    print(f"{wl.key}: {rep}")


@pytest.mark.parametrize("wl", SHAPES[:4], ids=[w.key for w in SHAPES[:4]])
def test_budget_zero_takes_top_community(wl):
    case = Case(wl)
    case.step(0, update=False)
    n_sel = case.st.sel.n_sel.cpu().numpy()
    assert np.all(n_sel == 1)


@pytest.mark.parametrize("wl", SHAPES[:5], ids=[w.key for w in SHAPES[:5]])
def test_full_budget_equals_dense(wl):
    case = Case(wl.replace(update=False))
    q = synth.draw_queries(wl, case.draw, 0)
    sparse = case.st.decode(q, wl.T).clone()
    dense = case.st.dense(q)
    torch.cuda.synchronize()
    assert float((sparse - dense).abs().max()) <= TOL[wl.dtype]
    n_tok = case.st.sel.n_tok.cpu().numpy()
    assert np.all(n_tok == wl.T)
    # and both match the oracle's dense softmax attention
    K = case.st.K.double().cpu().numpy()
    V = case.st.V.double().cpu().numpy()
    qn = q.double().cpu().numpy()
    gq = wl.Hq // wl.Hkv
    for b in range(wl.B):
        for h in range(wl.Hq):
            o = O.attention(qn[b, h], K[b, h // gq], V[b, h // gq], np.arange(wl.T))
            assert np.abs(o - dense[b, h].double().cpu().numpy()).max() <= TOL[wl.dtype]


@pytest.mark.parametrize("T", [1, 7, 100, 4099, 20000])
def test_dense_decode_lengths(T):
    wl = small("dense_len", 30, T=max(T, 8), update=False, B=3)
    case = Case(wl)
    q = synth.draw_queries(wl, case.draw, 0)
    case.st.T = T
    dense = case.st.dense(q)
    torch.cuda.synchronize()
    K = case.st.K.double().cpu().numpy()
    V = case.st.V.double().cpu().numpy()
    qn = q.double().cpu().numpy()
    for b in range(wl.B):
        for h in range(0, wl.Hq, 5):
            o = O.attention(qn[b, h], K[b, h // 4], V[b, h // 4], np.arange(T))
            assert np.abs(o - dense[b, h].double().cpu().numpy()).max() <= TOL[wl.dtype]


def test_no_sinks():
    wl = small("no_sinks", 31, S=0)
    case = Case(wl)
    for _ in range(2):
        case.step(wl.budget)


def test_single_community():
    wl = small("one_comm", 32, update=True)
    labels = np.zeros((wl.B, wl.G, wl.T), dtype=np.int32)
    labels[:, :, : wl.S] = -1
    case = Case(wl, labels=labels)
    case.check_build()
    case.step(5)          # budget below the community size: the top community is still taken
    assert np.all(case.st.sel.n_tok.cpu().numpy() == wl.T)
    case.step(5)          # the token appended after the first step joined the only community
    assert np.all(case.st.sel.n_tok.cpu().numpy() == wl.T + 1)


def test_empty_ids_and_slack_capacity():
    wl = small("gaps", 33)
    labels = np.stack([synth.sequence_labels(wl, 0, b) for b in range(wl.B)])
    labels = np.where(labels >= 0, labels * 3 + 1, -1).astype(np.int32)   # ids 1, 4, 7, ...
    case = Case(wl, labels=labels, Cmax=int(labels.max()) + 50)
    case.check_build()
    for _ in range(2):
        case.step(wl.budget)


def test_tail_full_sets_error_and_skips():
    wl = small("tail_full", 34, steps=3)
    case = Case(wl, max_tail=1)
    case.step(wl.budget)
    assert int(case.st.graph.dev_err.item()) == 0
    cnt0 = case.st.graph.cnt.clone()
    cent0 = case.st.graph.cent.clone()
    q = synth.draw_queries(wl, case.draw, 1)
    case.st.decode(q, wl.budget)
    kn, vn = synth.draw_new_tokens(wl, case.draw, 1)
    assigned = case.st.append(kn, vn)
    torch.cuda.synchronize()
    assert int(case.st.graph.dev_err.item()) & 4
    assert bool((assigned == -1).all())
    assert torch.equal(case.st.graph.cnt, cnt0) and torch.equal(case.st.graph.cent, cent0)
    assert bool((case.st.graph.comm_of[:, case.st.T - 1] == -1).all())


def test_token_capacity_truncates_with_error():
    wl = small("tok_cap", 35, update=False)
    case = Case(wl, tok_cap=wl.S + 37)
    case.step(wl.budget, update=False)
    assert int(case.st.graph.dev_err.item()) & 8
    assert np.all(case.st.sel.n_tok.cpu().numpy() == wl.S + 37)


def test_bad_labels_are_flagged_and_skipped():
    wl = small("bad_labels", 36, update=False, B=1)
    labels = np.stack([synth.sequence_labels(wl, 0, b) for b in range(wl.B)])
    C = int(labels.max()) + 1
    bad = labels.copy()
    bad[0, 0, 1] = 3          # a sink with a label
    bad[0, 1, 100] = C + 5    # beyond Cmax
    case = Case(wl, labels=bad, Cmax=C)
    err = int(case.st.graph.dev_err.item())
    assert err & 1 and err & 2
    # the same word through the library's reader, which can also clear it
    assert ckv.ckv_get_device_error(case.st.graph) == err
    assert ckv.ckv_get_device_error(case.st.graph, reset=True) == err
    assert ckv.ckv_get_device_error(case.st.graph) == 0 and int(case.st.graph.dev_err.item()) == 0
    comm_of = case.st.graph.comm_of.cpu().numpy()
    assert comm_of[0, 1] == -1 and comm_of[1, 100] == -1
    assert int(case.st.graph.cnt.sum().item()) == wl.B * wl.G * (wl.T - wl.S) - 1


@pytest.mark.parametrize("T", [6000, 40000])
def test_neighbours_crowded_threshold(T):
    """Tokens planted with identical keys, all in one thread's share of the
    list (every 128th entry of a single community), crowd the neighbour
    search's candidate set past one warp (T = 6000) and past its shared-memory
    capacity (T = 40000).  The exact ties resolve to the lowest positions."""
    wl = small(f"crowded_{T}", 37, B=1, Hq=1, Hkv=1, T=T, budgets=(64,), steps=1)
    labels = np.zeros((wl.B, wl.G, wl.T), dtype=np.int32)
    labels[:, :, : wl.S] = -1
    case = Case(wl, labels=labels)
    q = synth.draw_queries(wl, case.draw, 0)
    planted = np.arange(wl.S, wl.T, 128)
    case.st.K[0, 0, torch.from_numpy(planted).cuda()] = (3.0 * q[0, 0].float()).to(case.st.K.dtype)
    case.st.build(torch.from_numpy(labels.reshape(case.U, wl.T)).cuda(), wl.T)
    rep = case.step(wl.budget)
    assert rep.band_neighbours == 0
    assert case.st.nbr8[0].cpu().tolist() == planted[:8].tolist()


def test_append_assign_matches_external_append():
    """ckv_append_assign (the library writes row pos, key from k_new) leaves
    the cache and graph exactly as a PyTorch append + ckv_assign_update."""
    wl = small("append", 38, steps=3)
    a, b = Case(wl), Case(wl)
    for i in range(wl.steps):
        q = synth.draw_queries(wl, a.draw, i)
        a.st.decode(q, wl.budget)
        b.st.decode(q, wl.budget)
        kn, vn = synth.draw_new_tokens(wl, a.draw, i)
        kn, vn = kn.to(a.st.K.dtype), vn.to(a.st.V.dtype)
        ga = a.st.append(kn, vn).clone()
        gb = b.st.append_external(kn, vn).clone()
        torch.cuda.synchronize()
        assert torch.equal(ga, gb)
        pos = a.st.T - 1
        assert torch.equal(a.st.K[:, :, pos], kn) and torch.equal(a.st.V[:, :, pos], vn)
        assert torch.equal(a.st.K, b.st.K) and torch.equal(a.st.V, b.st.V)
        for name in ("comm_of", "cnt", "cent", "tail_tok", "tail_comm", "tail_len", "dev_err"):
            assert torch.equal(getattr(a.st.graph, name), getattr(b.st.graph, name)), name


@pytest.mark.parametrize("budget_frac", [1.0, 0.5])
def test_many_candidates_global_sort(budget_frac):
    """More than 256 communities at or above the crossing bin: the selection
    takes its global-memory sort path (every community, or about half)."""
    T = 60000
    wl = small(f"many_cand_{budget_frac}", 39, B=1, Hq=4, Hkv=1, T=T, budgets=(int(T * budget_frac),),
               steps=2, update=True)
    case = Case(wl)
    assert case.C > 600
    for _ in range(wl.steps):
        case.step(wl.budget)
    assert int(case.st.sel.n_sel.max().item()) > 256


@pytest.mark.parametrize("budget", [6000, 9000])
def test_candidates_between_the_two_rankings(budget):
    """Between 129 and 256 candidates: the selection ranks them with its
    sorting network instead of the quadratic loop (one head per graph, ~65
    tokens per community; by the oracle these budgets select 61-155 and
    101-206 communities in the four graphs)."""
    T = 40000
    wl = small(f"mid_cand_{budget}", 49, B=1, Hq=4, Hkv=1, T=T, mode="head", budgets=(budget,), steps=2,
               update=True)
    case = Case(wl)
    for _ in range(wl.steps):
        case.step(wl.budget)
    n_sel = case.st.sel.n_sel.cpu().numpy()
    assert n_sel.max() > 128 and n_sel.max() <= 230, n_sel


def test_largest_community_count():
    """Cmax = 8192 communities (the largest supported) of 1-3 tokens each in
    one graph, with updates: the scoring grid's last row block is full, the
    histogram and the re-scoring see every community, and the selection of
    ~300 communities takes the global-memory sort."""
    wl = small("max_comm", 50, B=1, Hq=4, Hkv=1, T=8192 * 2 + 4, sizes="multinomial", n_comm=8192,
               min_size=1, budgets=(600,), steps=2, update=True)
    case = Case(wl)
    assert case.C == 8192 and case.Cmax == 8192
    for _ in range(wl.steps):
        case.step(wl.budget)
    assert int(case.st.graph.dev_err.item()) == 0
    assert int(case.st.sel.n_sel.max().item()) > 256


def test_fused_decode_append_matches_separate_calls():
    """ckv_sparse_decode_append (update run by the merge kernel) gives the
    same outputs, neighbours, cache and graph state, bit for bit, as
    ckv_sparse_decode followed by ckv_append_assign."""
    for wl in (small("fused_head", 40, mode="head", T=2500, budgets=(200,), steps=3),
               small("fused_group", 41, steps=3), synth.WORKLOADS["tiny"].replace(steps=3),
               small("fused_vote", 46, mode="head", Hq=16, Hkv=4, d=64, steps=3, assign_rule="vote")):
        a, b = Case(wl), Case(wl)
        for i in range(wl.steps):
            q = synth.draw_queries(wl, a.draw, i)
            kn, vn = synth.draw_new_tokens(wl, a.draw, i)
            kn, vn = kn.to(a.st.K.dtype), vn.to(a.st.V.dtype)
            a.st.select(q, wl.budget)
            b.st.select(q, wl.budget)
            oa = a.st.attend_append(q, kn, vn).clone()
            ob = b.st.attend(q).clone()
            b.st.append(kn, vn)
            torch.cuda.synchronize()
            assert torch.equal(oa, ob), wl.key
            assert torch.equal(a.st.nbr8, b.st.nbr8) and torch.equal(a.st.assigned, b.st.assigned)
            assert torch.equal(a.st.K, b.st.K) and torch.equal(a.st.V, b.st.V)
            for name in ("comm_of", "cnt", "cent", "tail_tok", "tail_comm", "tail_len", "dev_err"):
                assert torch.equal(getattr(a.st.graph, name), getattr(b.st.graph, name)), (wl.key, name)


def _int8_copy(cent: torch.Tensor):
    """The scoring copy's definition, in float32 numpy (IEEE arithmetic): per
    row s = max |c| / 127, r = 127 / max |c|, code = round-half-even(c * r),
    0 for an all-zero row."""
    c = cent.cpu().numpy()
    amax = np.abs(c).max(axis=-1)
    s = amax / np.float32(127.0)
    r = np.float32(127.0) / np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    codes = np.where(amax[..., None] > 0, np.rint(c * r[..., None]), 0.0)
    return (torch.from_numpy(np.clip(codes, -127, 127).astype(np.int8)).to(cent.device),
            torch.from_numpy(s.astype(np.float32)).to(cent.device))


def test_scoring_copy_tracks_centres():
    """(cent_q, cent_qs) is cent quantised per row, bit for bit, after the
    build and after every update."""
    for wl in (small("cent_q", 42, steps=3), small("cent_q_f32_d64", 48, dtype="f32", d=64, mode="head",
                                                  Hq=8, Hkv=4, steps=3)):
        case = Case(wl)
        for i in range(wl.steps + 1):
            if i:
                case.step(wl.budget)
            codes, s = _int8_copy(case.st.graph.cent)
            assert torch.equal(case.st.graph.cent_qs, s), (wl.key, i)
            assert torch.equal(case.st.graph.cent_q, codes), (wl.key, i)


def test_cut_among_scores_closer_than_the_int8_pass():
    """Every community's keys are v + 1e-4 id w (v, w fixed per graph), so
    neighbouring communities' scores differ by ~1e-4, far below what the int8
    scoring pass resolves (its codes barely change from one community to the
    next; its bounds are ~1e-1 wide) and far above the 1e-5 tie band: the
    exact re-scoring alone decides the ranking and the cut, which must equal
    the oracle's."""
    wl = small("near_ties", 43, dtype="f32", B=1, T=3000, budgets=(1000,), steps=1, update=False)
    case = Case(wl)
    q = synth.draw_queries(wl, case.draw, 0)
    labels = case.draw.labels
    gq = wl.Hq // wl.Hkv
    for g in range(wl.G):
        lab = torch.from_numpy(labels[0, g].astype(np.int64)).cuda()
        v = q[0, g * gq].float()
        w = torch.roll(v, 1)
        rows = v[None, :] + (1e-4 * lab.clamp(min=0).float())[:, None] * w[None, :]
        keep = lab < 0  # sinks keep their keys
        case.st.K[0, g, : wl.T] = torch.where(keep[:, None], case.st.K[0, g, : wl.T], rows)
    case.st.build(torch.from_numpy(labels.reshape(case.U, wl.T).astype(np.int32)).cuda(), wl.T)
    rep = case.step(wl.budget, update=False)
    assert rep.band_selections == 0
    n_sel = case.st.sel.n_sel.cpu().numpy()
    assert np.all(n_sel > 3)


def test_vote_rule_is_decisive_and_matches_oracle():
    """Under the vote rule the assignments follow the oracle's majority vote
    (checked inside Case.step), and on these inputs the vote picks another
    community than the score rule would in some units, so the check has
    teeth; the same layer under the score rule makes different choices."""
    wl = small("vote_decisive", 47, Hq=16, Hkv=4, mode="head", steps=4, assign_rule="vote")
    vote, score = Case(wl), Case(wl.replace(assign_rule="score"))
    rep = Report()
    picks_v, picks_s = [], []
    for _ in range(wl.steps):
        vote.step(wl.budget, rep=rep)
        score.step(wl.budget)
        picks_v.append(vote.st.assigned.cpu().clone())
        picks_s.append(score.st.assigned.cpu().clone())
    assert rep.rule_decisive > 0, rep
    assert any(not torch.equal(a, b) for a, b in zip(picks_v, picks_s))
    assert int(vote.st.graph.dev_err.item()) == 0
    print(rep)


def test_cuda_graph_capture_replays_the_step():
    """After one eager call, the selection and the attention can be captured
    in a CUDA graph (no call allocates or synchronises, and the launches carry
    their programmatic dependencies); replays with new queries in the
    captured buffer give the eager results bit for bit."""
    wl = small("graph_capture", 51, update=False, steps=3)
    case = Case(wl)
    st = case.st
    qs = [synth.draw_queries(wl, case.draw, i) for i in range(wl.steps)]
    eager = []
    for q in qs:
        st.decode(q, wl.budget)
        eager.append((st.out.clone(), st.nbr8.clone(), st.sel.sel_tok.clone(), st.sel.n_tok.clone()))
    q_static = qs[0].clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st.decode(q_static, wl.budget)
    for q, (out, nbr, tok, ntok) in zip(qs, eager):
        q_static.copy_(q)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(st.out, out) and torch.equal(st.nbr8, nbr)
        assert torch.equal(st.sel.n_tok, ntok)
        for u in range(st.U):  # the token lists (entries past n_tok are stale by design)
            n = int(ntok[u])
            assert torch.equal(st.sel.sel_tok[u, :n], tok[u, :n]), u
    assert int(st.graph.dev_err.item()) == 0


def test_kernel_timing_counts_each_launch():
    """With timing on, one step records one launch of each of its kernels
    (positive durations); with it off nothing more is recorded."""
    wl = small("kernel_timing", 52, steps=1)
    case = Case(wl)
    q = synth.draw_queries(wl, case.draw, 0)
    kn, vn = synth.draw_new_tokens(wl, case.draw, 0)
    ckv.ckv_kernel_times()
    ckv.ckv_kernel_timing(True)
    try:
        case.st.select(q, wl.budget)
        case.st.attend_append(q, kn.to(case.st.K.dtype), vn.to(case.st.V.dtype))
    finally:
        ckv.ckv_kernel_timing(False)
    t = ckv.ckv_kernel_times()
    for kind in ("score", "attention", "merge"):
        assert t[kind][1] == 1 and t[kind][0] > 0.0, (kind, t[kind])
    # scoring and selection are one kernel; the update runs in the merge kernel
    assert all(t[k][1] == 0 for k in ("build", "select", "update"))
    case.st.select(q, wl.budget)
    assert all(v[1] == 0 for v in ckv.ckv_kernel_times().values())
