"""Seeded synthetic inputs for the CommunityKV decode path.

This module only draws inputs: community labels (the stand-in for the Leiden
partition, which is not built here), key/value caches clustered around
per-community centres, decode queries and the K/V rows of newly generated
tokens.  It holds none of the method's arithmetic (no centroid means, no
scores, no selection, no attention), so both the CUDA path and the CPU
oracle may use it without sharing any of the computation they are compared on.

Workload shapes follow the CommunityKV evaluation envelope (Qwen3-8B and
Llama-3.1-8B, contexts up to 128K, at most 128 generated tokens per run;
"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning", rit.work
summary, section "When CommunityKV is worth enabling").  The datasets the
pages evaluate on (LongBench v2, BABILong, RULER) and the model weights are
not used: these seeded draws stand in for them.

Recipe (all draws seeded; see `Workload`):

* community sizes: ``multinomial`` (n communities, each at least ``min_size``,
  the rest spread uniformly), ``lognormal`` (mean 64: sigma 1,
  mu = ln 64 - 1/2, rounded, at least 1) or ``zipf`` (s = 1.2 on 1..4096),
  drawn until the T - S non-sink positions are filled; the last one truncated;
* labels: -1 on the S sink positions 0..S-1; elsewhere a random permutation
  of the label multiset (``scatter``) or one contiguous run per community in
  random order (``spans``);
* keys: K[t] = mu_{label(t)} + 0.3 N(0, I) with centres mu_c ~ N(0, I); sink
  keys N(0, I); values N(0, I);
* queries: q_h = 0.5 mu_{c_h} + N(0, I), c_h uniform per head and step;
* new tokens: k = mu_c + 0.3 N(0, I) with c uniform, v ~ N(0, I);
* prefill queries (the token graph's input): q_{h,i} = 0.5 mu_{label(i)} +
  N(0, I), the label that of position i's key in its KV head's clustering,
  and N(0, I) at the sinks.

In per-head mode the first head of each GQA group owns the partition the keys
are clustered by; the other heads of the group get independent partitions
drawn from the same law.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "community_sizes", "graph_labels",
           "sequence_labels", "CacheDraw", "draw_cache", "draw_queries",
           "draw_new_tokens", "draw_prefill_queries", "torch_dtype"]


@dataclasses.dataclass(frozen=True)
class Workload:
    key: str
    title: str
    index: int              # position in the list of workloads; seeds derive from it
    layers: int
    B: int
    Hq: int
    Hkv: int
    d: int
    dtype: str              # "f32" | "bf16"
    T: int                  # context length when decoding starts
    S: int                  # attention-sink tokens (positions 0..S-1)
    budgets: Tuple[int, ...]
    steps: int
    mode: str               # "group" (one graph per KV group) | "head" (one per query head)
    sizes: str              # "multinomial" | "lognormal" | "zipf"
    n_comm: int = 0         # multinomial only
    min_size: int = 1
    update: bool = False    # assign each new token and append it to the cache
    layout: str = "scatter"
    assign_rule: str = "score"  # "score" | "vote": how a new token picks a neighbouring community

    @property
    def G(self) -> int:
        return self.Hkv if self.mode == "group" else self.Hq

    @property
    def gq(self) -> int:
        """Query heads per graph."""
        return self.Hq // self.Hkv if self.mode == "group" else 1

    @property
    def T_cap(self) -> int:
        return self.T + (self.steps if self.update else 0)

    @property
    def budget(self) -> int:
        return self.budgets[0]

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    w.key: w for w in [
        Workload("tiny", "Tiny: 1 layer, Hkv 1, Hq 4, d 64, fp32, 1K cache, 16 communities",
                 0, 1, 1, 4, 1, 64, "f32", 1024, 4, (128,), 8, "group",
                 "multinomial", n_comm=16, min_size=8, update=True),
        Workload("qwen3_8b_32k", "Qwen3-8B-shaped layer, 32K ctx, B 1, one graph per KV group",
                 1, 1, 1, 32, 8, 128, "bf16", 32768, 4, (2048,), 64, "group",
                 "lognormal"),
        Workload("qwen3_8b_128k_head", "Qwen3-8B shapes, 128K ctx, B 8, one graph per query head, update",
                 2, 1, 8, 32, 8, 128, "bf16", 131072, 4, (2048,), 64, "head",
                 "lognormal", update=True),
        Workload("llama31_8b_64k", "Llama-3.1-8B-shaped step, 32 layers, 64K ctx, B 16, update",
                 3, 32, 16, 32, 8, 128, "bf16", 65536, 4, (4096,), 128, "group",
                 "lognormal", update=True),
        Workload("qwen3_8b_128k_zipf", "Qwen3-8B shapes, 128K ctx, B 32, Zipf sizes, budget sweep",
                 4, 1, 32, 32, 8, 128, "bf16", 131072, 4, (512, 1024, 2048, 4096, 8192), 32,
                 "group", "zipf"),
    ]
}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


# ----------------------------------------------------------------------------
# community sizes and labels (numpy, host)
# ----------------------------------------------------------------------------

_ZIPF_CACHE: Dict[Tuple[float, int], np.ndarray] = {}


def _zipf_cdf(s: float, kmax: int) -> np.ndarray:
    key = (s, kmax)
    if key not in _ZIPF_CACHE:
        k = np.arange(1, kmax + 1, dtype=np.float64)
        p = k ** (-s)
        _ZIPF_CACHE[key] = np.cumsum(p) / p.sum()
    return _ZIPF_CACHE[key]


def community_sizes(law: str, n_tokens: int, rng: np.random.Generator,
                    n_comm: int = 0, min_size: int = 1) -> np.ndarray:
    """Sizes of the communities that partition ``n_tokens`` non-sink positions."""
    if n_tokens <= 0:
        return np.zeros(0, dtype=np.int64)
    if law == "multinomial":
        base = n_comm * min_size
        if base > n_tokens:
            raise ValueError("min_size * n_comm exceeds the token count")
        extra = rng.multinomial(n_tokens - base, np.full(n_comm, 1.0 / n_comm))
        return (extra + min_size).astype(np.int64)
    out = []
    total = 0
    while total < n_tokens:
        if law == "lognormal":
            draw = np.rint(rng.lognormal(math.log(64.0) - 0.5, 1.0, 1024))
            draw = np.maximum(draw, 1).astype(np.int64)
        elif law == "zipf":
            u = rng.random(1024)
            draw = np.searchsorted(_zipf_cdf(1.2, 4096), u, side="left").astype(np.int64) + 1
        else:
            raise ValueError(f"unknown size law {law!r}")
        for x in draw:
            x = int(x)
            if total + x >= n_tokens:
                out.append(n_tokens - total)
                total = n_tokens
                break
            out.append(x)
            total += x
    return np.asarray(out, dtype=np.int64)


def graph_labels(sizes: np.ndarray, T: int, S: int, rng: np.random.Generator,
                 layout: str = "scatter") -> np.ndarray:
    """int32 labels of length T: -1 on positions < S, community ids elsewhere."""
    lab = np.full(T, -1, dtype=np.int32)
    ids = np.repeat(np.arange(len(sizes), dtype=np.int32), sizes)
    if layout == "scatter":
        lab[S:] = ids[rng.permutation(len(ids))]
    elif layout == "spans":
        order = rng.permutation(len(sizes))
        lab[S:] = np.repeat(order.astype(np.int32), sizes[order])
    else:
        raise ValueError(f"unknown layout {layout!r}")
    return lab


def sequence_labels(wl: Workload, layer: int, b: int) -> np.ndarray:
    """Labels of every graph of sequence ``b`` at ``layer``: int32 [G, T]."""
    rng = np.random.default_rng(1000 * wl.index + 17 * layer + b)
    out = np.empty((wl.G, wl.T), dtype=np.int32)
    for g in range(wl.G):
        sizes = community_sizes(wl.sizes, wl.T - wl.S, rng, wl.n_comm, wl.min_size)
        out[g] = graph_labels(sizes, wl.T, wl.S, rng, wl.layout)
    return out


def cluster_graph(wl: Workload, kvh: int) -> int:
    """Index of the graph whose partition the keys of KV head ``kvh`` follow."""
    return kvh if wl.mode == "group" else kvh * (wl.Hq // wl.Hkv)


# ----------------------------------------------------------------------------
# caches, queries, new tokens (torch, any device)
# ----------------------------------------------------------------------------

def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


@dataclasses.dataclass
class CacheDraw:
    K: torch.Tensor          # [B, Hkv, T_cap, d]; rows >= T are zero
    V: torch.Tensor          # [B, Hkv, T_cap, d]
    labels: np.ndarray       # int32 [B, G, T]
    mu: torch.Tensor         # fp32 [B, Hkv, Cc, d] true centres of the key clusters
    n_cluster: np.ndarray    # int64 [B, Hkv] communities in each key-cluster partition


def draw_cache(wl: Workload, layer: int = 0, device="cpu",
               labels: Optional[np.ndarray] = None, T_cap: Optional[int] = None) -> CacheDraw:
    """Draw one layer's cache for the whole batch (labels drawn unless given)."""
    T_cap = wl.T_cap if T_cap is None else T_cap
    if labels is None:
        labels = np.stack([sequence_labels(wl, layer, b) for b in range(wl.B)])
    cl = np.stack([labels[:, cluster_graph(wl, h)] for h in range(wl.Hkv)], axis=1)  # [B,Hkv,T]
    n_cluster = cl.max(axis=2).astype(np.int64) + 1
    Cc = int(n_cluster.max())
    dt = torch_dtype(wl.dtype)
    gen = _gen(device, 7_000_003 * wl.index + 1009 * layer + 11)
    mu = torch.randn((wl.B, wl.Hkv, Cc, wl.d), generator=gen, device=device, dtype=torch.float32)
    K = torch.zeros((wl.B, wl.Hkv, T_cap, wl.d), device=device, dtype=dt)
    V = torch.zeros((wl.B, wl.Hkv, T_cap, wl.d), device=device, dtype=dt)
    for b in range(wl.B):
        for h in range(wl.Hkv):
            lab = torch.from_numpy(cl[b, h, wl.S:].astype(np.int64)).to(device)
            noise = torch.randn((wl.T - wl.S, wl.d), generator=gen, device=device)
            K[b, h, wl.S:wl.T] = (mu[b, h].index_select(0, lab) + 0.3 * noise).to(dt)
            K[b, h, :wl.S] = torch.randn((wl.S, wl.d), generator=gen, device=device).to(dt)
            V[b, h, :wl.T] = torch.randn((wl.T, wl.d), generator=gen, device=device).to(dt)
    return CacheDraw(K, V, labels, mu, n_cluster)


def draw_queries(wl: Workload, draw: CacheDraw, step: int, layer: int = 0) -> torch.Tensor:
    """Decode queries for one step: [B, Hq, d] in the cache dtype."""
    dev = draw.mu.device
    gen = _gen(dev, 9_000_011 * wl.index + 104_729 * layer + 31 * step + 5)
    gq = wl.Hq // wl.Hkv
    u = torch.rand((wl.B, wl.Hq), generator=gen, device=dev)
    nc = torch.from_numpy(np.repeat(draw.n_cluster, gq, axis=1)).to(dev)       # [B, Hq]
    c = torch.clamp((u * nc).long(), max=draw.mu.shape[2] - 1)
    kvh = torch.arange(wl.Hq, device=dev) // gq
    bidx = torch.arange(wl.B, device=dev)[:, None]
    centre = draw.mu[bidx, kvh[None, :], c]                                      # [B, Hq, d]
    q = 0.5 * centre + torch.randn((wl.B, wl.Hq, wl.d), generator=gen, device=dev)
    return q.to(torch_dtype(wl.dtype)).contiguous()


def draw_new_tokens(wl: Workload, draw: CacheDraw, step: int, layer: int = 0):
    """K/V rows of the token generated at ``step``: two [B, Hkv, d] tensors."""
    dev = draw.mu.device
    gen = _gen(dev, 5_000_077 * wl.index + 104_723 * layer + 37 * step + 3)
    u = torch.rand((wl.B, wl.Hkv), generator=gen, device=dev)
    nc = torch.from_numpy(draw.n_cluster).to(dev)
    c = torch.clamp((u * nc).long(), max=draw.mu.shape[2] - 1)
    bidx = torch.arange(wl.B, device=dev)[:, None]
    hidx = torch.arange(wl.Hkv, device=dev)[None, :]
    k = draw.mu[bidx, hidx, c] + 0.3 * torch.randn((wl.B, wl.Hkv, wl.d), generator=gen, device=dev)
    v = torch.randn((wl.B, wl.Hkv, wl.d), generator=gen, device=dev)
    dt = torch_dtype(wl.dtype)
    return k.to(dt).contiguous(), v.to(dt).contiguous()


def draw_prefill_queries(wl: Workload, draw: CacheDraw, layer: int = 0) -> torch.Tensor:
    """The queries of the prefill tokens: [B, Hq, T, d] in the cache dtype.
    Query i of a head leans towards the centre of the cluster its own key was
    drawn from (so attention is strongest within a community), sinks are
    N(0, I)."""
    dev = draw.mu.device
    gen = _gen(dev, 3_000_017 * wl.index + 104_711 * layer + 13)
    gq = wl.Hq // wl.Hkv
    q = torch.randn((wl.B, wl.Hq, wl.T, wl.d), generator=gen, device=dev)
    for b in range(wl.B):
        for h in range(wl.Hkv):
            lab = torch.from_numpy(draw.labels[b, cluster_graph(wl, h), wl.S:].astype(np.int64)).to(dev)
            centre = draw.mu[b, h].index_select(0, lab)                       # [T - S, d]
            q[b, h * gq:(h + 1) * gq, wl.S:] += 0.5 * centre[None]
    return q.to(torch_dtype(wl.dtype)).contiguous()
