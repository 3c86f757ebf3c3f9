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
