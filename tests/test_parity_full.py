"""The five workloads at full size, in the launch configuration the benchmark
times, checked on sampled graph units (every unit gets the cheap invariants:
token counts, unit prefix, sinks first).  The 32-layer Llama-3.1-8B workload
is checked on one full-size layer: its layers are independent caches and
graphs driven by the same calls."""
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
