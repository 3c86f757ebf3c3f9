"""Host logic of bench.py's multi-GPU run, exercised on CPU with gloo ranks.

With N GPUs every rank decodes its own batch (weak scaling, no collective on
the data path); the reported value is N*K steps over the slowest rank's
device time, which the ranks agree on with one MAX all-reduce.
"""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        n, r, local = bench.dist_env()
        cpu = torch.device("cpu")
        # each rank "measured" a different time; all must report the slowest
        seconds = 1.0 + 0.5 * rank
        bench.barrier(cpu)
        tmax = bench.reduce_max(seconds, cpu)
        wl, layer = bench.rank_workload(synth.WORKLOADS["tiny"], r)
        draw = synth.draw_cache(wl, layer, cpu)
        digest = float(draw.K.double().abs().sum())
        json.dump({"rank": r, "n": n, "local": local, "tmax": tmax, "layer": layer,
                   "value": bench.job_value(n, 10, tmax), "digest": digest},
                  open(os.path.join(out_dir, f"r{rank}.json"), "w"))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_sharding(tmp_path):
    ws = 2
    mp.start_processes(_rank_main, args=(ws, _free_port(), str(tmp_path)), nprocs=ws,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(ws)]
    for r, d in enumerate(res):
        assert d["rank"] == r and d["n"] == ws and d["local"] == r
        # max over ranks, identical on every rank
        assert d["tmax"] == pytest.approx(1.5)
        # whole-job value: all ranks' steps over the slowest rank's time
        assert d["value"] == pytest.approx(ws * 10 / 1.5)
        assert d["layer"] == r
    # each rank decodes its own batch: different seeds give different caches
    assert res[0]["digest"] != res[1]["digest"]


def test_single_process_helpers():
    cpu = torch.device("cpu")
    assert not dist.is_initialized()
    assert bench.reduce_max(3.25, cpu) == 3.25
    bench.barrier(cpu)  # no process group: a no-op
    assert bench.job_value(4, 100, 2.0) == 200.0
    assert np.isnan(bench.job_value(1, 10, 0.0))


def test_assignment_drift_on_a_hand_built_layer():
    """One sequence, one KV head, one graph: two communities with centres
    e0 and e1; positions 0-1 are sinks, 2-5 build-time members, 6-7 joined
    later.  Every relative distance is worked out by hand."""
    from types import SimpleNamespace

    wl = synth.WORKLOADS["tiny"].replace(B=1, Hq=1, Hkv=1, d=2, S=2, T=6, mode="group")
    K = torch.zeros(1, 1, 8, 2)
    K[0, 0, 2:] = torch.tensor([[1.0, 0], [2, 0], [0, 1], [0, 2], [3, 4], [0, 1]])
    comm_of = torch.tensor([[-1, -1, 0, 0, 1, 1, 0, -1]], dtype=torch.int32)
    cent = torch.tensor([[[1.0, 0.0], [0.0, 1.0]]])
    st = SimpleNamespace(K=K, U=1, T=8, graph=SimpleNamespace(comm_of=comm_of, cent=cent))
    d = bench.assignment_drift([SimpleNamespace(st=st)], wl, T0=6, n_members=4)
    # tail: position 6 -> |(3,4)-(1,0)|/5 = sqrt(20)/5; position 7 unassigned (skipped)
    assert d["tail_tokens"] == 1
    assert d["tail_rel_dist"] == pytest.approx(np.sqrt(20) / 5)
    # members 2..5: 0, 1/2, 0, 1/2 -> 1/4
    assert d["member_rel_dist"] == pytest.approx(0.25)
    assert d["rule"] == "score"


def test_cpu_baseline_reports_single_and_all_core_oracle_rates():
    cb = bench.cpu_baseline(synth.WORKLOADS["tiny"], 128, torch.device("cpu"), 4)
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
    assert cb["all_cores"]["cores"] == (os.cpu_count() or 1) and cb["all_cores"]["value"] > 0


def test_reference_arm_prints_one_contract_line(capsys):
    """`bench.py --impl reference` (the CPU oracle) on the tiny workload: one
    JSON line with the base contract's keys and the reference arm's."""
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"]) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
