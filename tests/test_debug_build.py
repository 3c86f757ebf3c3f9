"""The debug build of the library (libckv_debug.so, compiled with CKV_DEBUG).

It checks, on the device, every index that a caller's array feeds to a kernel
(positions and token counts of the selection, CSR run offsets, tail lengths):
a bad one sets CKV_DEVERR_INDEX and the access is skipped, nothing traps.
On valid inputs it must give the release build's results bit for bit.

Each corrupted index below is chosen so that, even unchecked, the access would
stay inside the arrays (unit 0's rows are followed by unit 1's, the position
T_cap + 1 of sequence 0, KV head 0 lies in KV head 1's rows): the tests cannot
fault a GPU whatever the checks do.  The release build is never given a
corrupted position, run offset or token count.
"""
import ctypes
import os
import re

import pytest
import torch

import graph_community_sparse_b200 as ckv
import synth
from parity_util import Case

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE = synth.WORKLOADS["qwen3_8b_32k"]


def test_debug_library_exports_and_reports_itself():
    dl = ckv.load_debug_library()
    names = sorted(set(re.findall(r"CKV_API\s+[\w\s\*]+?\b(ckv_\w+)\s*\(", open(os.path.join(ROOT, "include",
                                                                                          "ckv.h")).read())))
    for n in names:
        assert hasattr(dl, n), n
    assert int(dl.ckv_debug_build()) == 1
    assert ckv.ckv_debug_build() == 0
    assert int(dl.ckv_abi_version()) == ckv.ckv_abi_version()


def _shape(key, index, **kw):
    args = dict(key=key, title=key, index=index, B=2, T=3000, budgets=(300,), steps=3, update=True)
    args.update(kw)
    return BASE.replace(**args)


SHAPES = [
    _shape("debug_group_gq4", 60),                                   # tensor-core attention path
    _shape("debug_head_gq1", 61, mode="head", T=2500, budgets=(200,)),  # scalar attention path
]


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _select(dl, st, q):
    return dl.ckv_score_select(ctypes.byref(st.cache), ctypes.byref(st.graph.desc), q.data_ptr(), st.budget_used,
                               ctypes.byref(st.sel.desc), st.ws.data_ptr(), st.ws.numel(), _stream())


def _decode(dl, st, q, out, nbr):
    return dl.ckv_sparse_decode(ctypes.byref(st.cache), q.data_ptr(), ctypes.byref(st.graph.desc),
                                ctypes.byref(st.sel.desc), out.data_ptr(), nbr.data_ptr(), st.ws.data_ptr(),
                                st.ws.numel(), _stream())


def _dev_err(st):
    torch.cuda.synchronize()
    return int(st.graph.dev_err.item())


@pytest.mark.gpu
@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: w.key)
def test_debug_build_matches_release_and_flags_bad_indices(wl):
    dl = ckv.load_debug_library()
    case = Case(wl, max_tail=16)
    st = case.st
    st.budget_used = wl.budget
    q = synth.draw_queries(wl, case.draw, 0)

    # valid inputs: the same selection and outputs, bit for bit
    st.select(q, wl.budget)
    ref = {k: getattr(st.sel, k).clone() for k in ("sel_comm", "n_sel", "sel_tok", "n_tok", "tok_prefix")}
    ref_out = st.attend(q).clone()
    ref_nbr = st.nbr8.clone()
    assert _select(dl, st, q) == 0
    for k, v in ref.items():
        assert torch.equal(getattr(st.sel, k), v), k
    out = torch.empty_like(ref_out)
    nbr = torch.empty_like(ref_nbr)
    assert _decode(dl, st, q, out, nbr) == 0
    assert torch.equal(out, ref_out) and torch.equal(nbr, ref_nbr)
    assert _dev_err(st) == 0

    T_cap, tok_cap = st.cache.T_cap, st.sel.desc.tok_cap
    # a position past the cache length in unit 0's list
    st.sel.sel_tok[0, wl.S] = T_cap + 1
    assert _decode(dl, st, q, out, nbr) == 0
    assert _dev_err(st) & ckv.DEVERR_INDEX
    st.graph.dev_err.zero_()
    st.sel.sel_tok.copy_(ref["sel_tok"])

    # a token count above the list's capacity
    st.sel.n_tok[0] = tok_cap + 5
    assert _decode(dl, st, q, out, nbr) == 0
    assert _dev_err(st) & ckv.DEVERR_INDEX
    st.graph.dev_err.zero_()
    st.sel.n_tok.copy_(ref["n_tok"])

    # member runs reaching past the list: every community's run of unit 0
    # ends beyond T_cap
    offs0 = st.graph.offs[0].clone()
    st.graph.offs[0, 1:] = T_cap + 7
    assert _select(dl, st, q) == 0
    assert _dev_err(st) & ckv.DEVERR_INDEX
    st.graph.dev_err.zero_()
    st.graph.offs[0].copy_(offs0)

    # a negative tail length: the selection flags it, and the update neither
    # joins unit 1 nor writes before its tail (unit 0's entry max_tail - 3)
    st.graph.tail_len[1] = -3
    assert _select(dl, st, q) == 0
    assert _dev_err(st) & ckv.DEVERR_INDEX
    st.graph.dev_err.zero_()
    mt = st.graph.desc.max_tail
    before = (st.graph.tail_tok[:2].clone(), st.graph.tail_comm[:2].clone())
    status = dl.ckv_assign_update(ctypes.byref(st.cache), ctypes.byref(st.graph.desc), st.T, ref_nbr.data_ptr(),
                                  None, _stream())
    assert status == 0
    assert _dev_err(st) & ckv.DEVERR_INDEX
    assert int(st.graph.tail_len[1]) == -3
    for t, b in zip((st.graph.tail_tok, st.graph.tail_comm), before):
        assert torch.equal(t[1], b[1]) and torch.equal(t[0, mt - 3:], b[0, mt - 3:])
