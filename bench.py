"""Benchmark of the CommunityKV decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--budget B]
    python bench.py --impl reference ...      # the float64 CPU oracle, timed on host cores

One step = ckv_score_select + ckv_sparse_decode, or, when the workload
updates, ckv_score_select + ckv_sparse_decode_append (the attention with the
cache append and community update run by its merge kernel) for the whole batch of one
layer, with inputs resident in HBM.  Every timed step is bracketed by CUDA
events on the launching stream; L2 is flushed (a 1 GiB write, then a 512 MiB
read so no dirty lines are left) before each step, outside the events.  Rank 0 prints one JSON line.  With N GPUs each rank
runs its own batch (weak scaling, no collective on the data path); the value
is N*K steps over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "sparse decode steps/s at 128K ctx; achieved HBM GB/s vs B200 peak"
DEFAULT_WORKLOAD = "qwen3_8b_128k_head"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal
# score+select, attention, merge (the update runs inside the merge kernel)
KERNELS_PER_STEP_UPDATE = 3
KERNELS_PER_STEP_STATIC = 3


# ----------------------------------------------------------------------------
# host logic shared by all ranks (tested on CPU with gloo)
# ----------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return ws, rank, local


def rank_workload(wl: synth.Workload, rank: int) -> tuple:
    """Weak scaling: every rank decodes its own batch of sequences, drawn from
    the workload's law with rank-specific seeds (layer index = rank)."""
    return wl, rank


def reduce_max(x: float, device) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def job_value(n_ranks: int, steps: int, max_seconds: float) -> float:
    return n_ranks * steps / max_seconds if max_seconds > 0 else float("nan")


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def csrc_digest() -> str:
    """sha256 over the decode kernels' sources (every .cu and .cuh file but
    the host-only ckv_api.cu (argument checks) and ckv_timing.cu (diagnostic
    events), and ckv_edges.cu, the prefill token graph's own translation unit,
    which no decode kernel includes; names and contents, in name order): any
    decode kernel or launch change alters it."""
    d = os.path.join(ROOT, "graph_community_sparse_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh", ".h")) and f not in ("ckv_api.cu", "ckv_timing.cu", "ckv_edges.cu"):
            h.update(f.encode() + b"\0" + open(os.path.join(d, f), "rb").read())
    return h.hexdigest()


def call_traffic(workload: str):
    """ncu DRAM bytes of one ckv_sparse_decode(_append) call: its attention
    and merge kernels' committed figures, while both are current."""
    a = profile_traffic("decode_main", workload)
    m = profile_traffic("decode_merge", workload)
    return a + m if a is not None and m is not None else None


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded by the committed ncu summary for this
    kernel and workload, valid only while no kernel source has changed since
    the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        d = json.load(open(path))
        ent = d[kernel][workload]
        if ent["csrc_sha256"] != csrc_digest():
            return None
        return float(ent["bytes_per_launch"])
    except Exception:
        return None


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for r in csv.reader(f):
                if len(r) >= 9:
                    rows.append([x.strip() for x in r])
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# the CUDA arm
# ----------------------------------------------------------------------------

class RowCounter:
    """Distinct (sequence, KV head, position) rows a step's selection reads,
    counted on the device without a host sync (a byte map per KV head)."""

    def __init__(self, wl: synth.Workload, U: int, T_cap: int, cap: int, device):
        self.per_head = wl.mode == "head"
        self.T_cap = T_cap
        units = torch.arange(U, device=device)
        gq = wl.Hq // wl.Hkv
        kv = (units // wl.G) * wl.Hkv + ((units % wl.G) // gq if self.per_head else units % wl.G)
        self.base = (kv.long() * T_cap)[:, None]
        self.col = torch.arange(cap, device=device)[None, :]
        self.dummy = wl.B * wl.Hkv * T_cap
        self.map = torch.zeros(self.dummy + 1, dtype=torch.uint8, device=device)

    def __call__(self, sel) -> torch.Tensor:
        n_tok = sel.n_tok.long()
        if not self.per_head:
            return n_tok.sum()
        cap = self.col.shape[1]
        key = torch.where(self.col < n_tok[:, None], self.base + sel.sel_tok[:, :cap].long(), self.dummy)
        self.map.zero_()
        self.map.index_fill_(0, key.reshape(-1), 1)
        return self.map[: self.dummy].sum(dtype=torch.long)


class BenchLayer:
    """One layer of the step: its cache, graph state, labels and the per-step
    queries and new tokens (seeded by the layer index)."""

    def __init__(self, wl: synth.Workload, seed_layer: int, device, T_cap: int, max_tail: int, n_total: int):
        from graph_community_sparse_b200.layer import LayerState

        draw = synth.draw_cache(wl, layer=seed_layer, device=device, T_cap=T_cap)
        C = int(draw.labels.max()) + 1
        self.st = LayerState(draw.K, draw.V, wl.Hq, wl.mode, wl.S, C, max_tail, rule=wl.assign_rule)
        self.labels = torch.from_numpy(draw.labels.reshape(self.st.U, wl.T).astype(np.int32)).to(device)
        self.qs = [synth.draw_queries(wl, draw, i, seed_layer) for i in range(n_total)]
        self.news = ([synth.draw_new_tokens(wl, draw, i, seed_layer) for i in range(n_total)]
                     if wl.update else [])

    def build(self, T: int) -> None:
        self.st.build(self.labels, T)


@torch.no_grad()
def assignment_drift(layers, wl: synth.Workload, T0: int, n_members: int = 1024) -> dict:
    """How well the running-mean centres still describe their members: the
    mean of |k - c| / |k| over the tokens joined since the last build (k the
    token's key, c its community's current centre), beside the same quantity
    over a sample of build-time members.  A diagnostic read after the timed
    steps, not part of the step."""
    tail, mem = [], []
    for L in layers:
        st, gr = L.st, L.st.graph
        dev = st.K.device
        u = torch.arange(st.U, device=dev)
        b, g = u // wl.G, u % wl.G
        kvh = g // (wl.Hq // wl.Hkv) if wl.mode == "head" else g
        rng = torch.Generator(device="cpu").manual_seed(7)
        sample = wl.S + torch.randperm(T0 - wl.S, generator=rng)[:n_members].to(dev)
        for pos, acc in ((torch.arange(T0, st.T, device=dev), tail), (sample, mem)):
            if pos.numel() == 0:
                continue
            comm = gr.comm_of[:, pos].long()                           # [U, P]
            k = st.K[b[:, None], kvh[:, None], pos[None, :]].float()   # [U, P, d]
            c = gr.cent[u[:, None], comm.clamp(min=0)]                  # [U, P, d]
            r = (k - c).norm(dim=-1) / k.norm(dim=-1).clamp_min(1e-30)
            acc.append(r[comm >= 0])
    tail = torch.cat(tail) if tail else torch.zeros(0)
    mem = torch.cat(mem) if mem else torch.zeros(0)
    return {"rule": wl.assign_rule, "tail_tokens": int(tail.numel()),
            "tail_rel_dist": float(tail.mean()) if tail.numel() else None,
            "member_rel_dist": float(mem.mean()) if mem.numel() else None,
            "metric": "mean |k - c(k)| / |k| over tokens joined since the build (tail) and over "
                      f"{n_members} sampled build-time members per graph"}


def run_cuda(args, wl: synth.Workload, rank: int, n_ranks: int, device) -> dict:
    K_steps, W_steps = args.steps, args.warmup
    budget = args.budget if args.budget is not None else wl.budget
    n_layers = args.layers if args.layers is not None else wl.layers
    B_steps = min(K_steps, 100)
    n_total = W_steps + K_steps + B_steps + args.e2e_steps
    # Update workloads run in episodes of the workload's own length (e.g. 64
    # generated tokens): the graph is rebuilt from the labels and the cache
    # length reset between episodes, outside the timed events.
    episode = wl.steps if wl.update else 0
    extra = episode + 8 if wl.update else 0
    T_cap = wl.T + extra
    # per-rank seeds: each rank owns a different batch of sequences
    layers = [BenchLayer(wl, rank * n_layers + l, device, T_cap, max(extra, 1), n_total) for l in range(n_layers)]
    st0 = layers[0].st
    U = st0.U
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record()
    for L in layers:
        L.build(wl.T)
    b1.record()
    torch.cuda.synchronize()
    build_ms = b0.elapsed_time(b1)

    def check_dev_err(what: str):
        for li, L in enumerate(layers):
            err = int(L.st.graph.dev_err.item())
            if err != 0:
                raise RuntimeError(f"{what}: layer {li} reported device error {err}")

    check_dev_err("build")
    # 1 GiB > L2; its ~0.3 ms on the GPU also lets the host enqueue a whole step
    # before the GPU reaches it, so the events time device work, not launch gaps
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.float32, device=device)
    # then reading another 512 MiB leaves L2 clean: the dirty lines of the
    # write are written back here, not charged to the step's first kernel
    clean_buf = torch.ones(128 * 1024 * 1024, dtype=torch.float32, device=device)
    sink = torch.zeros((), dtype=torch.float32, device=device)

    def flush():
        flush_buf.fill_(1.0)
        torch.sum(clean_buf, dim=0, out=sink)

    esz = 2 if wl.dtype == "bf16" else 4
    row_bytes = 2 * wl.d * esz
    per_head = wl.mode == "head"
    episodes = [0]

    def new_episode_if_due():
        if wl.update and st0.T - wl.T >= episode:
            for L in layers:
                L.build(wl.T)
            episodes[0] += 1

    def one_step(i, ev=None, per_call=False):
        """ev: [start, end] events, or with per_call [start, then after each
        layer's selection and after its attention]: events between the calls
        break the programmatic-launch chain from the selection into the
        attention, so the timed steps do not use them."""
        if ev:
            ev[0].record()
        for li, L in enumerate(layers):
            q = L.qs[i]
            L.st.select(q, budget)
            if ev and per_call:
                ev[1 + 2 * li].record()
            if wl.update:
                k, v = L.news[i]
                L.st.attend_append(q, k, v)
            else:
                L.st.attend(q, want_nbr=False)
            if ev and per_call:
                ev[2 + 2 * li].record()
        if ev and not per_call:
            ev[-1].record()

    # a selection never holds more than S + max(budget, largest community) tokens
    max_cnt = max(int(L.st.graph.cnt.max().item()) for L in layers) + extra
    cap = min(st0.sel.sel_tok.shape[1], wl.S + max(budget, max_cnt))
    count_rows = RowCounter(wl, U, T_cap, cap, device)
    clock_sampler = ClockSampler(device.index).__enter__()
    time.sleep(0.5)  # let the sampler start before the warm-up
    for i in range(W_steps):
        new_episode_if_due()
        flush()
        one_step(i)
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_steps)]
    host_s = 0.0
    barrier(device)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    clk = clock_sampler
    for j in range(K_steps):
        new_episode_if_due()
        flush()
        h0 = time.perf_counter()
        one_step(W_steps + j, evs[j])
        host_s += time.perf_counter() - h0
    torch.cuda.synchronize()
    barrier(device)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    # a longer sample of the same steps (each timed alone, L2 flushed before
    # each), for the spread of the step time; not part of `value`
    long_ms = []
    if args.long_steps > 0:
        lev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.long_steps)]
        for j in range(args.long_steps):
            new_episode_if_due()
            flush()
            one_step((W_steps + j) % n_total, lev[j])
        torch.cuda.synchronize()
        long_ms = [e[0].elapsed_time(e[1]) for e in lev]
    clk.__exit__()
    clocks = clk.summary()
    total_s = sum(step_ms) / 1e3
    max_total_s = reduce_max(total_s, device)

    # per-call breakdown (for the roofline), in its own pass of steps right
    # after the timed ones, with an event between the calls
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(1 + 2 * n_layers)] for _ in range(B_steps)]
    rows_hist, ntok_hist, nsel_hist = [], [], []
    for j in range(B_steps):
        new_episode_if_due()
        flush()
        one_step(W_steps + K_steps + j, bevs[j], per_call=True)
        rows_hist.append(sum(count_rows(L.st.sel) for L in layers))
        ntok_hist.append(sum(L.st.sel.n_tok.long().sum() for L in layers))
        nsel_hist.append(sum(L.st.sel.n_sel.long().sum() for L in layers))
    torch.cuda.synchronize()
    check_dev_err("timed steps")
    # per-kernel durations: the library brackets each launch with CUDA events
    # on its stream in a pass of its own (the events cost the programmatic
    # overlap between a call's kernels, so neither the timed steps nor the
    # per-call pass carry them)
    import graph_community_sparse_b200 as ckv
    ckv.ckv_kernel_times()  # drop anything recorded before
    ckv.ckv_kernel_timing(True)
    try:
        for j in range(B_steps):
            new_episode_if_due()
            flush()
            one_step(W_steps + K_steps + j)
        torch.cuda.synchronize()
    finally:
        ckv.ckv_kernel_timing(False)
    ktimes = ckv.ckv_kernel_times()
    check_dev_err("kernel timing pass")
    drift = assignment_drift(layers, wl, wl.T) if wl.update else None
    # per step, summed over the layers: each selection from the previous
    # layer's attention end (or the step start), each attention from its
    # selection end
    sel_ms = [sum((e[0] if li == 0 else e[2 * li]).elapsed_time(e[1 + 2 * li]) for li in range(n_layers))
              for e in bevs]
    dec_ms = [sum(e[1 + 2 * li].elapsed_time(e[2 + 2 * li]) for li in range(n_layers)) for e in bevs]

    rows = np.array([int(r.item()) for r in rows_hist], dtype=np.float64)
    ntok = np.array([int(r.item()) for r in ntok_hist], dtype=np.float64)
    nsel = np.array([int(r.item()) for r in nsel_hist], dtype=np.float64)
    ncomm = float(sum(int(L.st.graph.num_comm.long().sum().item()) for L in layers))
    q_bytes = n_layers * wl.B * wl.Hq * wl.d * esz
    out_bytes = n_layers * wl.B * wl.Hq * wl.d * 4
    dec_bytes = rows * row_bytes + ntok * 4 + q_bytes + out_bytes
    if wl.update:
        # neighbours, the logit of every list entry (written and read back),
        # up to 8 candidate centres read per unit, one centre row updated,
        # and the new K/V rows copied into the cache
        dec_bytes = dec_bytes + ntok * 8 + n_layers * (U * (8 * 4 + 8 * wl.d * 4 + 2 * wl.d * 4)
                                                       + 4 * wl.B * wl.Hkv * wl.d * esz)
    # the scoring pass reads every centre's int8 codes and scale; the selected
    # communities (at least) are re-scored from the fp32 centres; per
    # community a size is read and a score bound written and read back; the
    # token list is written
    sel_bytes = ncomm * (wl.d + 4) + nsel * wl.d * 4 + q_bytes + ncomm * 4 * 3 + ntok * 4
    peak, peak_src = measured_peaks()

    def gbs(bytes_, ms):
        return float(np.mean(bytes_) / (np.mean(ms) * 1e-3) / 1e9)

    dec_gbs = gbs(dec_bytes, dec_ms)
    sel_gbs = gbs(sel_bytes, sel_ms)
    per = f" (sum over {n_layers} layers)" if n_layers > 1 else ""
    kernels = {
        "ckv_score_select": {"ms": float(np.mean(sel_ms)), "bytes": float(np.mean(sel_bytes)), "GB/s": sel_gbs,
                             "frac": sel_gbs / peak},
    }
    dec_name = "ckv_sparse_decode_append" if wl.update else "ckv_sparse_decode"
    kernels[dec_name] = {"ms": float(np.mean(dec_ms)), "bytes": float(np.mean(dec_bytes)), "GB/s": dec_gbs,
                         "frac": dec_gbs / peak, "rows_per_step": float(rows.mean()),
                         "tokens_per_step": float(ntok.mean())}
    # the whole step against the same peak: both calls' bytes over the timed
    # steps' mean duration
    step_bytes = float(np.mean(sel_bytes) + np.mean(dec_bytes))
    step_gbs = step_bytes / (float(np.mean(step_ms)) * 1e-3) / 1e9
    step_roofline = {"ms": float(np.mean(step_ms)), "bytes": step_bytes, "GB/s": step_gbs, "frac": step_gbs / peak}
    # per-layer breakdown of the multi-layer step (means over the per-call pass)
    per_layer = None
    if n_layers > 1:
        per_layer = {
            "sel_us": [round(float(np.mean([(e[0] if li == 0 else e[2 * li]).elapsed_time(e[1 + 2 * li])
                                            for e in bevs])) * 1e3, 2) for li in range(n_layers)],
            "attn_us": [round(float(np.mean([e[1 + 2 * li].elapsed_time(e[2 + 2 * li]) for e in bevs])) * 1e3, 2)
                        for li in range(n_layers)]}
    # the kernels one by one (per step, summed over the layers): the attention
    # kernel's algorithmic bytes are the distinct selected K/V rows, their
    # indices, q and (with neighbours) the logit of every list entry; the
    # split-K partials it writes for the merge are not algorithmic
    attn_bytes = rows * row_bytes + ntok * 4 + q_bytes + (ntok * 4 if wl.update else 0)
    per_kernel = {}
    for kind, (tot_ms, nlaunch) in ktimes.items():
        # the episodes' rebuilds between steps are not part of the step
        if nlaunch and kind != "build":
            per_kernel[kind] = {"ms": tot_ms / B_steps, "launches_per_step": nlaunch / B_steps,
                                "share": tot_ms / B_steps / float(np.mean(step_ms))}
    if "attention" in per_kernel:
        a = per_kernel["attention"]
        a["bytes"] = float(np.mean(attn_bytes))
        a["GB/s"] = a["bytes"] / (a["ms"] * 1e-3) / 1e9
        a["frac"] = a["GB/s"] / peak
    # the roofline of the call the target names (ckv_sparse_decode, here with
    # the fused append when the workload updates): its algorithmic bytes over
    # its duration, against the measured copy peak and the nominal 8 TB/s;
    # the attention kernel alone is in per_kernel
    dk = kernels[dec_name]
    roofline = {"kernel": dec_name + " (the call: split-K attention kernel, then the merge kernel"
                          + (" that also runs the update)" if wl.update else ")"),
                "bound": "hbm", "achieved": dk["GB/s"], "peak": peak, "unit": "GB/s", "frac": dk["GB/s"] / peak,
                "peak_source": peak_src, "peak_nominal": NOMINAL_HBM_GBS,
                "frac_nominal": dk["GB/s"] / NOMINAL_HBM_GBS,
                "traffic": call_traffic(wl.key) if n_layers == 1 else None,
                "bytes_per_launch": dk["bytes"] / n_layers,
                "timing": "CUDA events on the launching stream around the call, mean over a pass of "
                          f"{B_steps} steps right after the timed ones{per}"}
    if "attention" in per_kernel:
        per_kernel["attention"]["frac_nominal"] = per_kernel["attention"]["GB/s"] / NOMINAL_HBM_GBS
    if n_layers == 1:
        # the committed ncu DRAM bytes per launch, beside the algorithmic ones
        kernels["ckv_score_select"]["traffic"] = profile_traffic("score_select_kernel", wl.key)
        for name, kern in (("attention", "decode_main"), ("merge", "decode_merge")):
            if name in per_kernel:
                per_kernel[name]["traffic"] = profile_traffic(kern, wl.key)

    # dense comparator on the same caches and queries
    dense_out = torch.empty_like(st0.out)
    dms = []
    for j in range(max(3, min(K_steps, 10)) + 2):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for L in layers:
            L.st.dense(L.qs[j % len(L.qs)], dense_out)
        e1.record()
        dms.append((e0, e1))
    torch.cuda.synchronize()
    dms = [a.elapsed_time(b) for a, b in dms[2:]]
    dense_bytes = n_layers * wl.B * wl.Hkv * st0.T * row_bytes + q_bytes + out_bytes
    dense_gbs = dense_bytes / (np.mean(dms) * 1e-3) / 1e9
    dense = {"ms": float(np.mean(dms)), "bytes": float(dense_bytes), "GB/s": float(dense_gbs),
             "frac": float(dense_gbs / peak), "T": st0.T,
             "sparse_step_speedup": float(np.mean(dms) / np.mean(step_ms))}

    # end to end through the public API with host buffers: every layer's q
    # (and new K/V rows) in from pinned memory, its outputs back
    e2e = None
    if args.e2e_steps > 0:
        # per layer and step, the inputs (q, and the new K/V rows) packed in
        # one pinned host buffer and copied in one transfer into a packed
        # device buffer that q, k_new and v_new are views of; the results
        # (out, and nbr8 and assigned when the step updates) share one
        # allocation in LayerState and come back in one transfer
        first = W_steps + K_steps + B_steps
        io = []
        for L in layers:
            nq = L.qs[0].numel()
            nkv = L.news[0][0].numel() if wl.update else 0
            dev_in = torch.empty(nq + 2 * nkv, dtype=L.qs[0].dtype, device=device)
            host_in = []
            for j in range(args.e2e_steps):
                parts = [L.qs[first + j].flatten()]
                if wl.update:
                    parts += [L.news[first + j][0].flatten(), L.news[first + j][1].flatten()]
                host_in.append(torch.cat(parts).cpu().pin_memory())
            res = L.st.results if wl.update else L.st.results[: L.st.out.numel()]
            io.append(dict(host_in=host_in, dev_in=dev_in, q=dev_in[:nq].view(L.qs[0].shape),
                           k=dev_in[nq: nq + nkv].view(L.news[0][0].shape) if wl.update else None,
                           v=dev_in[nq + nkv:].view(L.news[0][1].shape) if wl.update else None,
                           res=res, res_h=torch.empty(res.shape, dtype=res.dtype, pin_memory=True)))
        h2d = sum(b["dev_in"].numel() * b["dev_in"].element_size() for b in io)
        d2h = sum(b["res"].numel() * b["res"].element_size() for b in io)
        e_ms = []
        for j in range(args.e2e_steps):
            new_episode_if_due()
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for L, b in zip(layers, io):
                b["dev_in"].copy_(b["host_in"][j], non_blocking=True)
                L.st.select(b["q"], budget)
                if wl.update:
                    L.st.attend_append(b["q"], b["k"], b["v"])
                else:
                    L.st.attend(b["q"], want_nbr=False)
                b["res_h"].copy_(b["res"], non_blocking=True)
            e1.record()
            e_ms.append((e0, e1))
        torch.cuda.synchronize()
        e_ms = [a.elapsed_time(b) for a, b in e_ms]
        e_total = reduce_max(sum(e_ms) / 1e3, device)
        e2e = {"value": job_value(n_ranks, len(e_ms), e_total), "unit": "steps/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": float(np.mean(e_ms)),
               "copies_per_layer": "one host-to-device (packed inputs) and one device-to-host (packed results)"}

    # host enqueue time of one step with the GPU idle (a synchronize before
    # each): in the timed loop the host also waits on a launch queue filled by
    # the flushes, so its time there is not the enqueue cost
    enq = []
    for j in range(20):
        new_episode_if_due()
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        one_step(j % n_total)  # any step's inputs: only the host time is kept
        enq.append(time.perf_counter() - h0)
    torch.cuda.synchronize()
    check_dev_err("host enqueue pass")

    value = job_value(n_ranks, K_steps, max_total_s)

    def stats(ms):
        a = np.asarray(ms, dtype=np.float64)
        return {"n": int(a.size), "median": float(np.median(a)), "p10": float(np.percentile(a, 10)),
                "p90": float(np.percentile(a, 90)), "min": float(a.min()), "max": float(a.max())}

    spread = {"timed_steps": stats(step_ms)}
    if long_ms:
        spread["long_sample"] = dict(stats(long_ms), steps_per_s=1e3 / float(np.mean(long_ms)),
                                     note="the same steps, each timed alone after an L2 flush, after the "
                                          "timed ones; not part of value")
    if clocks.get("sm_mhz"):
        spread["median_ms_x_sm_mhz"] = float(np.median(step_ms)) * clocks["sm_mhz"]
    return {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": n_ranks, "steps": K_steps,
        "warmup": W_steps, "ms_per_step": max_total_s * 1e3 / K_steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": config_dict(wl, budget, n_layers, float(ncomm / (U * n_layers)), n_ranks),
        "step_spread": spread,
        "tokens_per_s": value * wl.B,
        "roofline": roofline,
        "kernels": kernels,
        "per_kernel": per_kernel,
        "step_roofline": step_roofline,
        "per_layer": per_layer,
        "dense": dense,
        "drift": drift,
        "e2e": e2e,
        "gpu_launches": K_steps * n_layers * (KERNELS_PER_STEP_UPDATE if wl.update else KERNELS_PER_STEP_STATIC),
        "clocks": clocks,
        "build_ms": build_ms,
        "wall_s_timed_region": wall,
        "host_us_per_step": float(np.median(enq)) * 1e6,
        "host_us_per_step_timed_loop": host_s / K_steps * 1e6,
        "episodes": episodes[0],
    }


# ----------------------------------------------------------------------------
# the other 128K / 64K configurations, measured in the same run (N = 1)
# ----------------------------------------------------------------------------

def measure_point(layers, wl: synth.Workload, budget: int, device, flush, steps: int, warmup: int,
                  call_steps: int, dense_reps: int, first: int = 0) -> dict:
    """One (workload, budget) point on already built layers: the step time
    (`steps` steps, each bracketed by CUDA events after an L2 flush), the two
    calls' times (events between them, `call_steps` steps), each kernel's time
    (the library's own launch events, `call_steps` steps) and the dense
    comparator (`dense_reps` runs)."""
    import graph_community_sparse_b200 as ckv
    n_layers = len(layers)
    esz = 2 if wl.dtype == "bf16" else 4
    row_bytes = 2 * wl.d * esz
    T0 = wl.T

    def step(i, ev=None):
        for li, L in enumerate(layers):
            if wl.update and L.st.T - T0 >= wl.steps:
                L.build(T0)
            q = L.qs[i]
            if ev:
                ev[2 * li].record()
            L.st.select(q, budget)
            if ev:
                ev[2 * li + 1].record()
            if wl.update:
                k, v = L.news[i]
                L.st.attend_append(q, k, v)
            else:
                L.st.attend(q, want_nbr=False)
        if ev:
            ev[-1].record()

    i = first
    for _ in range(warmup):
        flush()
        step(i)
        i += 1
    evs = []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record()
        step(i)
        e[1].record()
        evs.append(e)
        i += 1
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    # per call, with the rows each step reads
    cevs, ntok, nsel = [], [], []
    for _ in range(call_steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_layers + 1)]
        step(i, e)
        cevs.append(e)
        ntok.append(sum(L.st.sel.n_tok.long().sum() for L in layers))
        nsel.append(sum(L.st.sel.n_sel.long().sum() for L in layers))
        i += 1
    torch.cuda.synchronize()
    sel_ms = [sum(e[2 * li].elapsed_time(e[2 * li + 1]) for li in range(n_layers)) for e in cevs]
    dec_ms = [sum(e[2 * li + 1].elapsed_time(e[2 * li + 2]) for li in range(n_layers)) for e in cevs]
    per_layer = None
    if n_layers > 1:
        per_layer = {"sel_us": [round(float(np.mean([e[2 * li].elapsed_time(e[2 * li + 1]) for e in cevs])) * 1e3, 2)
                                for li in range(n_layers)],
                     "attn_us": [round(float(np.mean([e[2 * li + 1].elapsed_time(e[2 * li + 2]) for e in cevs])) * 1e3,
                                       2) for li in range(n_layers)]}
    # per kernel (the library's launch events)
    ckv.ckv_kernel_times()
    ckv.ckv_kernel_timing(True)
    try:
        for _ in range(call_steps):
            flush()
            step(i)
            i += 1
        torch.cuda.synchronize()
    finally:
        ckv.ckv_kernel_timing(False)
    kt = ckv.ckv_kernel_times()
    for L in layers:
        err = int(L.st.graph.dev_err.item())
        if err:
            raise RuntimeError(f"{wl.key} budget {budget}: device error {err}")
    ntok = float(np.mean([int(t.item()) for t in ntok]))
    nsel = float(np.mean([int(t.item()) for t in nsel]))
    peak, _ = measured_peaks()
    q_bytes = n_layers * wl.B * wl.Hq * wl.d * esz
    out_bytes = n_layers * wl.B * wl.Hq * wl.d * 4
    # per-group graphs: one graph per KV head, so every list entry is a
    # distinct K/V row
    attn_bytes = ntok * row_bytes + ntok * 4 + q_bytes + (ntok * 4 if wl.update else 0)
    dec_bytes = ntok * row_bytes + ntok * 4 + q_bytes + out_bytes
    attn_ms = kt["attention"][0] / call_steps
    res = {"budget": budget, "timed_steps": steps, "ms_per_step": float(np.mean(step_ms)),
           "ms_per_step_median": float(np.median(step_ms)), "steps_per_s": 1e3 / float(np.mean(step_ms)),
           "tokens_per_step": ntok, "communities_selected_per_step": nsel,
           "select_ms": float(np.mean(sel_ms)), "decode_call_ms": float(np.mean(dec_ms)),
           "decode_call_frac": dec_bytes / (float(np.mean(dec_ms)) * 1e-3) / 1e9 / peak,
           "kernel_ms": {k: v[0] / call_steps for k, v in kt.items() if v[1] and k != "build"},
           "attention_frac": attn_bytes / (attn_ms * 1e-3) / 1e9 / peak if attn_ms > 0 else None,
           "per_layer": per_layer}
    if dense_reps > 0:
        dense_out = torch.empty_like(layers[0].st.out)
        dms = []
        for j in range(dense_reps + 1):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for L in layers:
                L.st.dense(L.qs[0], dense_out)
            e1.record()
            dms.append((e0, e1))
        torch.cuda.synchronize()
        dms = [a.elapsed_time(b) for a, b in dms[1:]]
        dense_bytes = n_layers * wl.B * wl.Hkv * layers[0].st.T * row_bytes + q_bytes + out_bytes
        res["dense_ms"] = float(np.mean(dms))
        res["dense_frac"] = dense_bytes / (res["dense_ms"] * 1e-3) / 1e9 / peak
        res["sparse_step_speedup"] = res["dense_ms"] / res["ms_per_step"]
    return res


def measured_bf16_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            return float(json.load(open(p))["bf16_tflops"]), "measured"
        except Exception:
            pass
    return 1590.0, "fallback"


def measure_edges(device, T: int = 32768, reps: int = 3) -> dict:
    """The prefill token graph (ckv_build_edges) of one Qwen3-8B-shaped layer
    at T tokens (one sequence, per-group graphs): call time, and the causal
    Q K^T's FLOPs (2 Hq d (T - S)(T - S - 1) / 2) over it against the measured
    dense bf16 peak."""
    import graph_community_sparse_b200 as ckv
    wl = synth.WORKLOADS["qwen3_8b_32k"].replace(key="prefill_edges", index=78, T=T, budgets=(2048,))
    draw = synth.draw_cache(wl, device=device)
    q = synth.draw_prefill_queries(wl, draw)
    cache = ckv.cache_desc(draw.K, draw.V, wl.Hq)
    e = ckv.new_edges(cache, ckv.PER_GROUP, wl.S, wl.T, device=device)
    ckv.ckv_build_edges(cache, ckv.PER_GROUP, wl.S, q, wl.T, e)
    torch.cuda.synchronize()
    evs = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ckv.ckv_build_edges(cache, ckv.PER_GROUP, wl.S, q, wl.T, e)
        e1.record()
        evs.append((e0, e1))
    torch.cuda.synchronize()
    if int(e.dev_err.item()):
        raise RuntimeError("ckv_build_edges reported a device error")
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    n = wl.T - wl.S
    flop = 2.0 * wl.B * wl.Hq * wl.d * n * (n - 1) / 2
    peak, src = measured_bf16_tflops()
    tf = flop / (ms * 1e-3) / 1e12
    return {"title": f"prefill token graph, Qwen3-8B-shaped layer, {T} tokens, one sequence, per-group graphs",
            "ms": ms, "reps": reps, "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                                                 "frac": tf / peak, "peak_source": peak_src_note(src),
                                                 "flop": flop},
            "co_attention_pairs_per_graph": float(e.co_n.float().mean().item())}


def peak_src_note(src: str) -> str:
    return "measured dense bf16 (cuBLAS)" if src == "measured" else "fallback bf16 figure"


def run_sweeps(device, steps: int = 10, warmup: int = 3, call_steps: int = 5) -> dict:
    """The Zipf budget sweep (128K, B 32, per-group graphs) and one 32-layer
    Llama-3.1-8B-shaped step (64K, B 16, update), each with the dense
    comparator, on the same GPU after the headline workload."""
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.float32, device=device)
    clean_buf = torch.ones(128 * 1024 * 1024, dtype=torch.float32, device=device)
    sink = torch.zeros((), dtype=torch.float32, device=device)

    def flush():
        flush_buf.fill_(1.0)
        torch.sum(clean_buf, dim=0, out=sink)

    out = {"note": f"{steps} timed steps per point after {warmup} warm-up steps, {call_steps} steps for the "
                   "per-call and per-kernel times; L2 flushed before every step; peak = the measured copy peak"}
    wl = synth.WORKLOADS["qwen3_8b_128k_zipf"]
    n = warmup + steps + 2 * call_steps
    t0 = time.perf_counter()
    layers = [BenchLayer(wl, 0, device, wl.T, 1, n)]
    for L in layers:
        L.build(wl.T)
    out[wl.key] = {"title": wl.title, "points": [measure_point(layers, wl, b, device, flush, steps, warmup,
                                                               call_steps, 2) for b in wl.budgets],
                   "setup_s": None}
    out[wl.key]["setup_s"] = round(time.perf_counter() - t0, 1)
    del layers
    torch.cuda.empty_cache()
    wl = synth.WORKLOADS["llama31_8b_64k"]
    t0 = time.perf_counter()
    layers = [BenchLayer(wl, l, device, wl.T + wl.steps + 8, wl.steps + 8, n) for l in range(wl.layers)]
    for L in layers:
        L.build(wl.T)
    out[wl.key] = dict(title=wl.title, **measure_point(layers, wl, wl.budget, device, flush, steps, warmup,
                                                        call_steps, 1))
    out[wl.key]["setup_s"] = round(time.perf_counter() - t0, 1)
    del layers
    torch.cuda.empty_cache()
    out["prefill_edges"] = measure_edges(device)
    torch.cuda.empty_cache()
    return out


def config_dict(wl: synth.Workload, budget: int, n_layers: int, comm_per_graph: float, n_ranks: int) -> dict:
    """The `config` object of both arms' JSON lines."""
    return {"workload": wl.key, "title": wl.title, "B_per_gpu": wl.B, "layers": n_layers, "Hq": wl.Hq,
            "Hkv": wl.Hkv, "d": wl.d, "ctx": wl.T, "graphs": "per query head" if wl.mode == "head" else "per KV group",
            "communities_per_graph": round(comm_per_graph, 3), "budget": budget, "sinks": wl.S,
            "update": wl.update, "assign_rule": wl.assign_rule if wl.update else None, "layout": wl.layout,
            "l2": "flushed by a 1 GiB write then a 512 MiB read before every timed step, outside the CUDA events",
            "parallelism": f"dp{n_ranks} (independent batches, no collective)"}


# ----------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ----------------------------------------------------------------------------

def oracle_unit_seconds(wl: synth.Workload, draw: synth.CacheDraw, units, budget: int, step: int,
                        layer: int = 0, threads: int = 1) -> float:
    """Wall time of the oracle's steps for the given (b, g) units of one step,
    with the numerical library limited to ``threads`` threads, inputs already
    converted to float64."""
    import oracle.ckv_oracle as O
    from threadpoolctl import threadpool_limits

    C = int(draw.labels.max()) + 1
    q = synth.draw_queries(wl, draw, step, layer).double().cpu().numpy()
    kvs = {}
    for (b, g) in units:
        kvh = O.graph_kv_head(wl.mode, g, wl.Hq, wl.Hkv)
        if (b, kvh) not in kvs:
            kvs[(b, kvh)] = (draw.K[b, kvh, : wl.T].double().cpu().numpy(),
                             draw.V[b, kvh, : wl.T].double().cpu().numpy())
    if wl.update:
        kn, _ = synth.draw_new_tokens(wl, draw, step, layer)
        kn = kn.double().cpu().numpy()
    t = 0.0
    with threadpool_limits(threads):
        for (b, g) in units:
            st = O.GraphState(draw.labels[b, g], wl.T_cap, wl.S, C)
            kvh = O.graph_kv_head(wl.mode, g, wl.Hq, wl.Hkv)
            K, V = kvs[(b, kvh)]
            t0 = time.perf_counter()
            heads = O.graph_heads(wl.mode, g, wl.Hq, wl.Hkv)
            members = st.members()
            cent, cnt = O.centroids(K, members)
            s = O.community_scores(q[b, heads], cent, cnt)
            sel = O.select(s, cnt, budget)
            toks = O.token_set(sel, members, wl.S)
            for h in heads:
                O.attention(q[b, h], K, V, toks)
            nbr = O.neighbours(q[b, heads], K, toks, wl.S)
            if wl.update:
                pick = O.assign_vote if wl.assign_rule == "vote" else O.assign
                pick(kn[b, kvh], cent, [int(st.comm_of[p]) for p in nbr])
            t += time.perf_counter() - t0
    return t


def sample_units(wl: synth.Workload, n: int, seed: int):
    rng = np.random.default_rng(seed)
    allu = [(b, g) for b in range(wl.B) for g in range(wl.G)]
    idx = rng.choice(len(allu), size=min(n, len(allu)), replace=False)
    return [allu[i] for i in sorted(idx)]


def cpu_baseline(wl: synth.Workload, budget: int, device, n_units: int, n_layers: int = 1) -> dict:
    draw = synth.draw_cache(wl, device=device)
    units = sample_units(wl, n_units, 1)
    t = oracle_unit_seconds(wl, draw, units, budget, 0)
    per_step = t / len(units) * (wl.B * wl.G) * n_layers
    # the same oracle with the numerical library free to use every host core
    # (its Python loops stay on one), on half the sample
    ncpu = os.cpu_count() or 1
    half = units[: max(1, len(units) // 2)]
    t_all = oracle_unit_seconds(wl, draw, half, budget, 0, threads=ncpu)
    del draw
    lay = f" x {n_layers} layers" if n_layers > 1 else ""
    return {"value": 1.0 / per_step, "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(units)} of {wl.B * wl.G} graph units of one decode step{lay} "
                      f"({t:.1f} s single-threaded float64 numpy), scaled to the whole step",
            "all_cores": {"value": 1.0 / (t_all / len(half) * (wl.B * wl.G) * n_layers), "unit": "steps/s",
                          "cores": ncpu, "sample": f"{len(half)} of the same units, numpy free to use {ncpu} "
                                                   f"threads ({t_all:.1f} s)"}}


def run_reference(args, wl: synth.Workload, device) -> dict:
    budget = args.budget if args.budget is not None else wl.budget
    draw = synth.draw_cache(wl, device=device)
    per_step_units = max(1, args.ref_units)
    times = []
    for i in range(args.warmup + args.steps):
        units = sample_units(wl, per_step_units, 100 + i)
        t = oracle_unit_seconds(wl, draw, units, budget, i)
        if i >= args.warmup:
            times.append(t / len(units) * (wl.B * wl.G))
    value = args.steps / sum(times)
    cb = {"value": value, "unit": "steps/s", "cores": 1, "kind": "oracle",
          "sample": f"{per_step_units} of {wl.B * wl.G} graph units per step, scaled to the whole step"}
    return {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_dict(wl, budget, wl.layers if args.layers is None else args.layers,
                                  float(np.mean(draw.labels.max(axis=2) + 1)), 1),
            "cpu_baseline": cb, "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------

def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None, help="override the batch (small profiling captures)")
    ap.add_argument("--assign-rule", default=None, choices=["score", "vote"],
                    help="how a new token picks a neighbouring community (update workloads)")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step (default: the workload's; each has its own cache and graphs)")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-units", type=int, default=48, help="graph units the CPU baseline times")
    ap.add_argument("--ref-units", type=int, default=4, help="graph units per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--long-steps", type=int, default=300,
                    help="extra steps timed one by one after the timed ones, for the step-time spread")
    ap.add_argument("--edges-only", type=int, default=None, metavar="T",
                    help="measure only the prefill token graph (ckv_build_edges) at T tokens and print its line")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="skip the Zipf budget sweep and the 32-layer step run after the headline (N = 1 only)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return args


def main(argv=None):
    args = parse(argv)
    ws, rank, local = dist_env()
    wl = synth.WORKLOADS[args.workload]
    if args.batch is not None:
        wl = wl.replace(B=args.batch)
    if args.assign_rule is not None:
        wl = wl.replace(assign_rule=args.assign_rule)
    if args.impl == "reference":
        if rank != 0:
            return 0
        device = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
        print(json.dumps(run_reference(args, wl, device)), flush=True)
        return 0
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.edges_only is not None:
        if rank == 0:
            print(json.dumps({"prefill_edges": measure_edges(device, T=args.edges_only)}), flush=True)
        return 0
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=120))
    try:
        res = run_cuda(args, wl, rank, ws, device)
        if rank == 0 and ws == 1 and not args.no_cpu_baseline:
            torch.cuda.empty_cache()
            res["cpu_baseline"] = cpu_baseline(wl, res["config"]["budget"], device, args.cpu_units,
                                               res["config"]["layers"])
        if ws == 1 and not args.no_sweeps and args.workload == DEFAULT_WORKLOAD and args.batch is None:
            torch.cuda.empty_cache()
            res["sweeps"] = run_sweeps(device)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
