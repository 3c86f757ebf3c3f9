"""ckv_sparse_decode_noalloc: the sparse attention for callers that cannot
allocate device memory for a workspace (for instance a serving engine that
keeps nearly all of HBM in its own KV pools and offers plug-ins no allocator,
or a decode loop that must not call cudaMalloc because it can synchronise the
device).  Its scratch is a fixed array inside the library.

Checked through the C ABI against ckv_sparse_decode (the workspace version)
on two calls in a row: both run the same kernels in the same order, so the
outputs and neighbours must be identical bit for bit (which also catches a
slip in how the fixed scratch is laid out); sizes beyond the fixed scratch
are refused with a clear error before anything runs.  This file is
collected last on purpose, and passes alone in a fresh process too.
"""
import pytest
import torch

import graph_community_sparse_b200 as ckv
import synth
from parity_util import TOL, Case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("key,extra", [
    ("group", dict(index=40)),
    ("head", dict(index=41, mode="head", T=2500, budgets=(200,))),
])
def test_noalloc_matches_workspace_decode_twice(key, extra):
    args = dict(key=f"noalloc_{key}", title=key, B=2, T=3000, budgets=(300,), steps=2, update=False)
    args.update(extra)
    wl = synth.WORKLOADS["qwen3_8b_32k"].replace(**args)
    case = Case(wl)
    st = case.st
    out2 = torch.empty_like(st.out)
    nbr2 = torch.empty_like(st.nbr8)
    for step in range(2):
        q = synth.draw_queries(wl, case.draw, step)
        st.select(q, wl.budget)
        ref_out = st.attend(q).clone()
        ref_nbr = st.nbr8.clone()
        out2.fill_(float("nan"))
        nbr2.fill_(-7)
        ckv.ckv_sparse_decode_noalloc(st.cache, q, st.graph, st.sel, out2, nbr2)
        torch.cuda.synchronize()
        assert torch.isfinite(out2).all()
        assert float((out2 - ref_out).abs().max()) <= TOL[wl.dtype]
        assert torch.equal(out2, ref_out)
        assert torch.equal(nbr2, ref_nbr)


def test_noalloc_refuses_oversized_scratch():
    # per-group graphs with Hq/Hkv = 8 and d = 128 need more than the fixed scratch
    wl = synth.WORKLOADS["qwen3_8b_32k"].replace(key="noalloc_big", index=42, B=1, T=600, Hq=64, Hkv=8,
                                                 budgets=(100,), update=False)
    case = Case(wl)
    q = synth.draw_queries(wl, case.draw, 0)
    case.st.select(q, wl.budget)
    with pytest.raises(ckv.CKVError) as e:
        ckv.ckv_sparse_decode_noalloc(case.st.cache, q, case.st.graph, case.st.sel, case.st.out, case.st.nbr8)
    assert e.value.status == 3
    assert "scratch" in str(e.value)
