"""The five workloads at full size, in the launch configuration the benchmark
times, checked on sampled graph units (every unit gets the cheap invariants:
token counts, unit prefix, sinks first).  The 32-layer Llama-3.1-8B workload
is checked on full-size layers: its layers are independent caches and graphs
driven by the same calls.  Two tests follow a whole update episode, as the
benchmark runs it (the attention and the update in one call), so the tail's
growth, the running means after dozens of joins and the list's run offsets
and tail communities are checked at the measured shapes."""
import pytest
import torch

import synth
from parity_util import TOL, Case, Report

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _run(case, budget, steps, units):
    rep = Report()
    for s in range(steps):
        case.step(budget, units=units[s % len(units)], rep=rep)
    assert rep.max_out_err <= TOL[case.wl.dtype]
    assert int(case.st.graph.dev_err.item()) == 0
    print(case.wl.key, budget, rep)
    return rep


def test_tiny_all_steps():
    wl = W["tiny"]
    case = Case(wl)
    case.check_build()
    _run(case, wl.budget, wl.steps, [None])


def test_qwen3_8b_32k_group():
    wl = W["qwen3_8b_32k"]
    case = Case(wl)
    case.check_build(units=[(0, 0), (0, 5)])
    _run(case, wl.budget, 3, [[(0, 0), (0, 7)], [(0, 3)], [(0, 6)]])


def test_qwen3_8b_128k_per_head_with_update():
    wl = W["qwen3_8b_128k_head"]
    case = Case(wl)
    case.check_build(units=[(0, 0), (7, 31)])
    _run(case, wl.budget, 3, [[(0, 0), (3, 17)], [(7, 31), (3, 17)], [(0, 0), (5, 2)]])


def test_llama31_8b_64k_one_layer_with_update():
    wl = W["llama31_8b_64k"]
    case = Case(wl, layer=5)
    _run(case, wl.budget, 2, [[(0, 0), (15, 7)], [(15, 7), (8, 3)]])


@pytest.mark.parametrize("budget", [512, 2048, 8192])
def test_qwen3_8b_128k_zipf(budget):
    wl = W["qwen3_8b_128k_zipf"]
    case = Case(wl)
    _run(case, budget, 2, [[(0, 0), (31, 7)], [(16, 4)]])


def test_qwen3_8b_128k_head_whole_episode_fused():
    """All 64 steps of the per-head 128K workload (batch 8, one join per
    graph and step), through ckv_sparse_decode_append; two fixed units are
    checked against the oracle every step (selection, token list, run
    offsets, tail communities, outputs, neighbours, the assignment, counts,
    and centres within 1e-5 of the recomputed means after every join), the
    cheap invariants on all 256 units."""
    wl = W["qwen3_8b_128k_head"]
    case = Case(wl)
    rep = Report()
    units = [(2, 9), (7, 30)]
    for _ in range(wl.steps):
        case.step(wl.budget, units=units, rep=rep, fused=True)
    assert rep.steps == wl.steps and rep.max_out_err <= TOL[wl.dtype]
    assert rep.max_cent_err <= 1e-5
    assert int(case.st.graph.dev_err.item()) == 0
    # every unit's tail holds this episode's joins (or fewer, for tokens that
    # had no candidate community)
    tl = case.st.graph.tail_len.cpu()
    assert int(tl.max()) <= wl.steps and int(tl.sum()) > 0
    print(wl.key, rep)


@pytest.mark.parametrize("layer", [0, 15, 31])
def test_llama31_8b_64k_layers_fused(layer):
    """Layers 0, 15 and 31 of the 32-layer Llama-shaped step (each its own
    full-size cache and graphs, seeded by the layer), three fused steps each,
    two units checked per step."""
    wl = W["llama31_8b_64k"]
    case = Case(wl, layer=layer)
    rep = Report()
    for s, units in enumerate([[(0, 0), (15, 7)], [(15, 7), (8, 3)], [(0, 0), (11, 5)]]):
        case.step(wl.budget, units=units, rep=rep, fused=True)
    assert rep.max_out_err <= TOL[wl.dtype] and rep.max_cent_err <= 1e-5
    assert int(case.st.graph.dev_err.item()) == 0
    print(wl.key, layer, rep)
