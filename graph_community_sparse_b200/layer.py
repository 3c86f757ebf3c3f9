"""Buffers and call sequence for one layer's CommunityKV decode state.

``LayerState`` owns (through PyTorch) the graph arrays, the selection and the
workspace for one KV cache, and issues the four library calls in decode
order.  It computes nothing itself.
"""
from __future__ import annotations

import contextlib
from typing import Optional

import torch

from . import (ASSIGN_SCORE, ASSIGN_VOTE, PER_GROUP, PER_HEAD, Graph, Selection, cache_desc, ckv_append_assign, ckv_assign_update,
               ckv_sparse_decode_append,
               ckv_build_centroids, ckv_dense_decode, ckv_score_select, ckv_sparse_decode,
               ckv_workspace_size, new_graph, new_selection, new_workspace, NEIGHBOURS)


@contextlib.contextmanager
def _range(name: str):
    """An NVTX range around one library call, so that a profiler's timeline
    names the step's parts; a no-op when no profiler is attached."""
    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


class LayerState:
    """K, V: [B, Hkv, T_cap, d] device tensors (bf16 or fp32), read in place.

    mode: "group" (one graph per KV group) or "head" (one graph per query head).
    tok_cap defaults to T_cap, which can never overflow.
    rule: how a new token picks among its neighbours' communities, "score"
    (best k . c) or "vote" (most neighbours, then the score).
    """

    def __init__(self, K: torch.Tensor, V: torch.Tensor, Hq: int, mode: str, S: int, Cmax: int,
                 max_tail: int, tok_cap: Optional[int] = None, rule: str = "score"):
        if rule not in ("score", "vote"):
            raise ValueError(f"unknown assignment rule {rule!r}")
        self.K, self.V = K, V
        self.cache = cache_desc(K, V, Hq)
        self.mode = PER_HEAD if mode == "head" else PER_GROUP
        self.graph: Graph = new_graph(self.cache, self.mode, S, Cmax, max_tail, device=K.device,
                                      rule=ASSIGN_VOTE if rule == "vote" else ASSIGN_SCORE)
        self.sel: Selection = new_selection(self.cache, self.graph, tok_cap or self.cache.T_cap,
                                            device=K.device)
        self.ws = new_workspace(ckv_workspace_size(self.cache, self.graph, self.sel), device=K.device)
        B, Hq_, d = self.cache.B, Hq, self.cache.d
        # the step's results share one allocation (out, then nbr8, then
        # assigned; all 4-byte types), so a caller reads them back with one copy
        n_out, U = B * Hq_ * d, self.graph.U
        self.results = torch.full((n_out + U * NEIGHBOURS + U,), -1, dtype=torch.int32, device=K.device)
        self.out = self.results[:n_out].view(torch.float32).view(B, Hq_, d)
        self.nbr8 = self.results[n_out: n_out + U * NEIGHBOURS].view(U, NEIGHBOURS)
        self.assigned = self.results[n_out + U * NEIGHBOURS:]
        self.T = 0

    @property
    def U(self) -> int:
        return self.graph.U

    def build(self, labels: torch.Tensor, T: int, stream=None) -> None:
        """labels: int32 [U, >=T] on the device."""
        with _range("ckv_build_centroids"):
            ckv_build_centroids(self.cache, labels, T, self.graph, self.ws, stream)
        self.T = T

    def select(self, q: torch.Tensor, budget: int, stream=None) -> None:
        with _range("ckv_score_select"):
            ckv_score_select(self.cache, self.graph, q, budget, self.sel, self.ws, stream)

    def attend(self, q: torch.Tensor, want_nbr: bool = True, stream=None) -> torch.Tensor:
        with _range("ckv_sparse_decode"):
            ckv_sparse_decode(self.cache, q, self.graph, self.sel, self.out,
                              self.nbr8 if want_nbr else None, self.ws, stream)
        return self.out

    def decode(self, q: torch.Tensor, budget: int, want_nbr: bool = True, stream=None) -> torch.Tensor:
        self.select(q, budget, stream)
        return self.attend(q, want_nbr, stream)

    def attend_append(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> torch.Tensor:
        """attend (neighbours into nbr8) and append in one call: the update
        runs inside the attention's merge kernel."""
        pos = self.T
        with _range("ckv_sparse_decode_append"):
            ckv_sparse_decode_append(self.cache, q, self.graph, self.sel, self.out, self.nbr8, pos,
                                     k_new.contiguous(), v_new.contiguous(), self.assigned, self.ws, stream)
        self.T += 1
        return self.out

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> torch.Tensor:
        """Write the new token's K/V rows ([B, Hkv, d]) at position T and let
        it join a community: one library call (ckv_append_assign)."""
        pos = self.T
        with _range("ckv_append_assign"):
            ckv_append_assign(self.cache, self.graph, pos, k_new.contiguous(), v_new.contiguous(), self.nbr8,
                              self.assigned, stream)
        self.T += 1
        return self.assigned

    def append_external(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> torch.Tensor:
        """Same result for a caller that writes the cache itself: the rows are
        copied with PyTorch, then ckv_assign_update reads the key from K."""
        pos = self.T
        self.K[:, :, pos].copy_(k_new)
        self.V[:, :, pos].copy_(v_new)
        with _range("ckv_assign_update"):
            ckv_assign_update(self.cache, self.graph, pos, self.nbr8, self.assigned, stream)
        self.T += 1
        return self.assigned

    def dense(self, q: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        out = torch.empty_like(self.out) if out is None else out
        with _range("ckv_dense_decode"):
            ckv_dense_decode(self.cache, q, self.T, out, self.ws, stream)
        return out
