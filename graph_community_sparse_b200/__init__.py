"""Python binding of libckv, the CommunityKV decode hot path for B200.

Argument marshalling only: every function passes raw device pointers, sizes
and the current CUDA stream to the C entry point of the same name in
``libckv.so`` (declared in include/ckv.h) and raises ``CKVError`` on a
non-zero status.  PyTorch provides device memory and streams; no computation
of the path happens here.  Importing the package fails loudly when the
library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "CKVError", "lib", "LIB_PATH", "CacheDesc", "GraphDesc", "SelectionDesc",
    "Graph", "Selection", "cache_desc", "new_graph", "new_selection", "new_workspace",
    "ckv_workspace_size", "ckv_build_centroids", "ckv_score_select", "ckv_sparse_decode",
    "ckv_sparse_decode_noalloc", "NOALLOC_SCRATCH_BYTES", "ckv_assign_update", "ckv_append_assign",
    "ckv_sparse_decode_append", "ckv_get_device_error", "ckv_kernel_timing", "ckv_kernel_times",
    "KERNEL_KINDS",
    "ckv_dense_decode", "ckv_status_string", "ckv_last_error",
    "ckv_abi_version", "ckv_debug_build", "load_debug_library", "DEBUG_LIB_PATH",
    "ckv_edges_workspace_size", "ckv_build_edges", "Edges", "new_edges", "DEVERR_EDGE_CAP",
    "EXPORTED", "DTYPE_F32", "DTYPE_BF16", "PER_GROUP", "PER_HEAD",
    "ASSIGN_SCORE", "ASSIGN_VOTE",
    "DEVERR_SINK_LABEL", "DEVERR_LABEL_RANGE", "DEVERR_TAIL_FULL", "DEVERR_TOKEN_CAP", "DEVERR_INDEX",
    "NEIGHBOURS",
]

# the in-tree build, always: no environment variable selects another library
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libckv.so")
# the same library built with device-side index checks (build.py --debug); it
# is loaded only on request (load_debug_library)
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libckv_debug.so")

DTYPE_F32, DTYPE_BF16 = 0, 1
PER_GROUP, PER_HEAD = 0, 1
ASSIGN_SCORE, ASSIGN_VOTE = 0, 1
DEVERR_SINK_LABEL, DEVERR_LABEL_RANGE, DEVERR_TAIL_FULL, DEVERR_TOKEN_CAP, DEVERR_INDEX = 1, 2, 4, 8, 16
DEVERR_EDGE_CAP = 32
NEIGHBOURS = 8
KERNEL_KINDS = ("build", "score", "select", "attention", "merge", "update", "edges")
EXPORTED = ("ckv_workspace_size", "ckv_build_centroids", "ckv_score_select", "ckv_sparse_decode",
            "ckv_sparse_decode_noalloc", "ckv_assign_update", "ckv_append_assign", "ckv_sparse_decode_append",
            "ckv_get_device_error", "ckv_kernel_timing", "ckv_kernel_times",
            "ckv_dense_decode",
            "ckv_edges_workspace_size", "ckv_build_edges",
            "ckv_status_string", "ckv_last_error", "ckv_abi_version", "ckv_debug_build")
NOALLOC_SCRATCH_BYTES = 32 << 20


class CKVError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {ckv_status_string(status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libckv.so not built at {LIB_PATH}; run `python graph_community_sparse_b200/build.py`")
lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _p, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t


class CacheDesc(ctypes.Structure):
    _fields_ = [("dtype", _i32), ("B", _i32), ("Hkv", _i32), ("Hq", _i32), ("d", _i32),
                ("T_cap", _i32), ("k", _p), ("v", _p), ("stride_b", _i64), ("stride_h", _i64),
                ("stride_t", _i64)]


class GraphDesc(ctypes.Structure):
    _fields_ = [("mode", _i32), ("S", _i32), ("Cmax", _i32), ("max_tail", _i32), ("T_cap", _i32),
                ("assign_rule", _i32), ("comm_of", _p), ("offs", _p), ("tok", _p), ("cnt", _p), ("cent", _p), ("cent_q", _p), ("cent_qs", _p),
                ("num_comm", _p), ("tail_tok", _p), ("tail_comm", _p), ("tail_len", _p),
                ("dev_err", _p)]


class SelectionDesc(ctypes.Structure):
    _fields_ = [("tok_cap", _i32), ("sel_comm", _p), ("n_sel", _p), ("sel_tok", _p), ("n_tok", _p),
                ("tok_prefix", _p), ("tail_sel", _p), ("unit_prefix", _p)]


_P = ctypes.POINTER


def _declare(lib_: ctypes.CDLL) -> ctypes.CDLL:
    """Argument and result types of every entry point of a loaded libckv."""
    lib_.ckv_workspace_size.argtypes = [_P(CacheDesc), _P(GraphDesc), _P(SelectionDesc), _P(_sz)]
    lib_.ckv_build_centroids.argtypes = [_P(CacheDesc), _p, _i64, _i32, _P(GraphDesc), _p, _sz, _p]
    lib_.ckv_score_select.argtypes = [_P(CacheDesc), _P(GraphDesc), _p, _i32, _P(SelectionDesc), _p, _sz, _p]
    lib_.ckv_sparse_decode.argtypes = [_P(CacheDesc), _p, _P(GraphDesc), _P(SelectionDesc), _p, _p, _p, _sz, _p]
    lib_.ckv_sparse_decode_noalloc.argtypes = [_P(CacheDesc), _p, _P(GraphDesc), _P(SelectionDesc), _p, _p, _p]
    lib_.ckv_assign_update.argtypes = [_P(CacheDesc), _P(GraphDesc), _i32, _p, _p, _p]
    lib_.ckv_append_assign.argtypes = [_P(CacheDesc), _P(GraphDesc), _i32, _p, _p, _p, _p, _p]
    lib_.ckv_sparse_decode_append.argtypes = [_P(CacheDesc), _p, _P(GraphDesc), _P(SelectionDesc), _p, _p, _i32,
                                              _p, _p, _p, _p, _sz, _p]
    lib_.ckv_dense_decode.argtypes = [_P(CacheDesc), _p, _i32, _p, _p, _sz, _p]
    lib_.ckv_edges_workspace_size.argtypes = [_P(CacheDesc), _i32, _i32, _i32, _P(_sz)]
    lib_.ckv_build_edges.argtypes = [_P(CacheDesc), _i32, _i32, _p, _i32, _p, _p, _p, _p, _p, _p, _i32, _p, _p, _sz,
                                     _p]
    lib_.ckv_get_device_error.argtypes = [_P(GraphDesc), _p, _P(ctypes.c_int32), _i32]
    lib_.ckv_kernel_timing.argtypes = [_i32]
    lib_.ckv_kernel_times.argtypes = [_P(ctypes.c_float), _P(ctypes.c_int32), _i32]
    for f in ("ckv_workspace_size", "ckv_build_centroids", "ckv_score_select", "ckv_sparse_decode",
              "ckv_sparse_decode_noalloc", "ckv_assign_update", "ckv_append_assign", "ckv_sparse_decode_append",
              "ckv_dense_decode", "ckv_get_device_error", "ckv_kernel_timing", "ckv_kernel_times",
              "ckv_edges_workspace_size", "ckv_build_edges"):
        getattr(lib_, f).restype = ctypes.c_int
    lib_.ckv_status_string.argtypes = [ctypes.c_int]
    lib_.ckv_status_string.restype = ctypes.c_char_p
    lib_.ckv_last_error.argtypes = []
    lib_.ckv_last_error.restype = ctypes.c_char_p
    lib_.ckv_abi_version.argtypes = []
    lib_.ckv_abi_version.restype = ctypes.c_int32
    lib_.ckv_debug_build.argtypes = []
    lib_.ckv_debug_build.restype = ctypes.c_int32
    return lib_


_declare(lib)
_debug_lib: Optional[ctypes.CDLL] = None


def load_debug_library() -> ctypes.CDLL:
    """The debug build of the library (libckv_debug.so: every index a
    caller's array feeds to a kernel is checked on the device), loaded on
    first use, with the same entry points as `lib`.  Raises ImportError when
    it has not been built (build.py --debug)."""
    global _debug_lib
    if _debug_lib is None:
        if not os.path.exists(DEBUG_LIB_PATH):
            raise ImportError(f"libckv_debug.so not built at {DEBUG_LIB_PATH}; run "
                              "`python graph_community_sparse_b200/build.py --debug`")
        _debug_lib = _declare(ctypes.CDLL(DEBUG_LIB_PATH))
    return _debug_lib


def ckv_debug_build() -> int:
    return int(lib.ckv_debug_build())


def ckv_status_string(status: int) -> str:
    return lib.ckv_status_string(int(status)).decode()


def ckv_last_error() -> str:
    return lib.ckv_last_error().decode()


def ckv_abi_version() -> int:
    return int(lib.ckv_abi_version())


def _check(status: int, where: str) -> None:
    if status != 0:
        raise CKVError(status, where, ckv_last_error())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ----------------------------------------------------------------------------
# descriptors and buffers (device memory comes from PyTorch)
# ----------------------------------------------------------------------------

def cache_desc(K: torch.Tensor, V: torch.Tensor, Hq: int) -> CacheDesc:
    """Describe a [B, Hkv, T_cap, d] K/V cache pair (same shape and strides)."""
    if K.shape != V.shape or K.stride() != V.stride() or K.dtype != V.dtype:
        raise ValueError("K and V must share shape, strides and dtype")
    if K.dim() != 4 or K.stride(3) != 1:
        raise ValueError("K must be [B, Hkv, T_cap, d] with contiguous rows")
    dt = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(K.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {K.dtype}")
    B, Hkv, T_cap, d = K.shape
    return CacheDesc(dt, B, Hkv, Hq, d, T_cap, K.data_ptr(), V.data_ptr(),
                     K.stride(0), K.stride(1), K.stride(2))


@dataclass
class Graph:
    desc: GraphDesc
    comm_of: torch.Tensor
    offs: torch.Tensor
    tok: torch.Tensor
    cnt: torch.Tensor
    cent: torch.Tensor
    cent_q: torch.Tensor
    cent_qs: torch.Tensor
    num_comm: torch.Tensor
    tail_tok: torch.Tensor
    tail_comm: torch.Tensor
    tail_len: torch.Tensor
    dev_err: torch.Tensor

    @property
    def U(self) -> int:
        return self.num_comm.shape[0]


@dataclass
class Selection:
    desc: SelectionDesc
    sel_comm: torch.Tensor
    n_sel: torch.Tensor
    sel_tok: torch.Tensor
    n_tok: torch.Tensor
    tok_prefix: torch.Tensor
    tail_sel: torch.Tensor
    unit_prefix: torch.Tensor


def new_graph(cache: CacheDesc, mode: int, S: int, Cmax: int, max_tail: int, device="cuda",
              rule: int = ASSIGN_SCORE) -> Graph:
    G = cache.Hq if mode == PER_HEAD else cache.Hkv
    U = cache.B * G
    i32 = dict(dtype=torch.int32, device=device)
    t = dict(
        comm_of=torch.full((U, cache.T_cap), -1, **i32),
        offs=torch.zeros((U, Cmax + 1), **i32),
        tok=torch.zeros((U, cache.T_cap), **i32),
        cnt=torch.zeros((U, Cmax), **i32),
        cent=torch.zeros((U, Cmax, cache.d), dtype=torch.float32, device=device),
        cent_q=torch.zeros((U, Cmax, cache.d), dtype=torch.int8, device=device),
        cent_qs=torch.zeros((U, Cmax), dtype=torch.float32, device=device),
        num_comm=torch.zeros((U,), **i32),
        tail_tok=torch.zeros((U, max(max_tail, 1)), **i32),
        tail_comm=torch.zeros((U, max(max_tail, 1)), **i32),
        tail_len=torch.zeros((U,), **i32),
        dev_err=torch.zeros((1,), **i32),
    )
    desc = GraphDesc(mode, S, Cmax, max_tail, cache.T_cap, rule, *(t[k].data_ptr() for k in (
        "comm_of", "offs", "tok", "cnt", "cent", "cent_q", "cent_qs", "num_comm", "tail_tok", "tail_comm", "tail_len",
        "dev_err")))
    return Graph(desc, **t)


def new_selection(cache: CacheDesc, graph: Graph, tok_cap: int, device="cuda") -> Selection:
    U, Cmax = graph.U, graph.desc.Cmax
    i32 = dict(dtype=torch.int32, device=device)
    t = dict(sel_comm=torch.zeros((U, Cmax), **i32), n_sel=torch.zeros((U,), **i32),
             sel_tok=torch.zeros((U, tok_cap), **i32), n_tok=torch.zeros((U,), **i32),
             tok_prefix=torch.zeros((U, Cmax + 1), **i32),
             tail_sel=torch.zeros((U, max(graph.desc.max_tail, 1)), **i32),
             unit_prefix=torch.zeros((U + 1,), **i32))
    desc = SelectionDesc(tok_cap, *(t[k].data_ptr() for k in ("sel_comm", "n_sel", "sel_tok", "n_tok",
                                                               "tok_prefix", "tail_sel", "unit_prefix")))
    return Selection(desc, **t)


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zeroed (the library needs its first 256 bytes zero before first use
    and leaves them zero); torch's caching allocator hands out 512-byte
    aligned blocks."""
    return torch.zeros((max(int(nbytes), 256),), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------------------
# the entry points
# ----------------------------------------------------------------------------

def ckv_workspace_size(cache: CacheDesc, graph: Optional[Graph] = None,
                       sel: Optional[Selection] = None) -> int:
    out = _sz(0)
    g = ctypes.byref(graph.desc) if graph is not None else None
    s = ctypes.byref(sel.desc) if sel is not None else None
    _check(lib.ckv_workspace_size(ctypes.byref(cache), g, s, ctypes.byref(out)), "ckv_workspace_size")
    return int(out.value)


def ckv_build_centroids(cache: CacheDesc, labels: torch.Tensor, T: int, graph: Graph,
                        ws: torch.Tensor, stream=None) -> None:
    if labels.dtype != torch.int32 or labels.dim() != 2 or labels.stride(1) != 1:
        raise ValueError("labels must be int32 [U, >=T] with contiguous rows")
    _check(lib.ckv_build_centroids(ctypes.byref(cache), labels.data_ptr(), labels.stride(0), T,
                                   ctypes.byref(graph.desc), ws.data_ptr(), ws.numel(), _stream(stream)),
           "ckv_build_centroids")


def ckv_score_select(cache: CacheDesc, graph: Graph, q: torch.Tensor, budget: int, sel: Selection,
                     ws: torch.Tensor, stream=None) -> None:
    _check(lib.ckv_score_select(ctypes.byref(cache), ctypes.byref(graph.desc), q.data_ptr(), budget,
                                ctypes.byref(sel.desc), ws.data_ptr(), ws.numel(), _stream(stream)),
           "ckv_score_select")


def ckv_sparse_decode(cache: CacheDesc, q: torch.Tensor, graph: Graph, sel: Selection, out: torch.Tensor,
                      nbr8: Optional[torch.Tensor], ws: torch.Tensor, stream=None) -> None:
    _check(lib.ckv_sparse_decode(ctypes.byref(cache), q.data_ptr(), ctypes.byref(graph.desc),
                                 ctypes.byref(sel.desc), out.data_ptr(), _ptr(nbr8), ws.data_ptr(),
                                 ws.numel(), _stream(stream)),
           "ckv_sparse_decode")


def ckv_sparse_decode_noalloc(cache: CacheDesc, q: torch.Tensor, graph: Graph, sel: Selection,
                              out: torch.Tensor, nbr8: Optional[torch.Tensor], stream=None) -> None:
    """ckv_sparse_decode for callers that cannot hand over a workspace: the
    scratch is a fixed 32 MiB array inside the library (see include/ckv.h).
    Calls must not overlap on the GPU."""
    _check(lib.ckv_sparse_decode_noalloc(ctypes.byref(cache), q.data_ptr(), ctypes.byref(graph.desc),
                                         ctypes.byref(sel.desc), out.data_ptr(), _ptr(nbr8), _stream(stream)),
           "ckv_sparse_decode_noalloc")


def ckv_assign_update(cache: CacheDesc, graph: Graph, pos: int, nbr8: torch.Tensor,
                      assigned: Optional[torch.Tensor], stream=None) -> None:
    _check(lib.ckv_assign_update(ctypes.byref(cache), ctypes.byref(graph.desc), pos, nbr8.data_ptr(),
                                 _ptr(assigned), _stream(stream)),
           "ckv_assign_update")


def _check_rows(cache: CacheDesc, **rows) -> None:
    shape = (cache.B, cache.Hkv, cache.d)
    for name, t in rows.items():
        if tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {shape} tensor, got {tuple(t.shape)}")


def ckv_sparse_decode_append(cache: CacheDesc, q: torch.Tensor, graph: Graph, sel: Selection, out: torch.Tensor,
                             nbr8: Optional[torch.Tensor], pos: int, k_new: torch.Tensor, v_new: torch.Tensor,
                             assigned: Optional[torch.Tensor], ws: torch.Tensor, stream=None) -> None:
    """ckv_sparse_decode + ckv_append_assign in one call (the update runs in
    the attention's merge kernel)."""
    _check_rows(cache, k_new=k_new, v_new=v_new)
    _check(lib.ckv_sparse_decode_append(ctypes.byref(cache), q.data_ptr(), ctypes.byref(graph.desc),
                                        ctypes.byref(sel.desc), out.data_ptr(), _ptr(nbr8), pos, k_new.data_ptr(),
                                        v_new.data_ptr(), _ptr(assigned), ws.data_ptr(), ws.numel(),
                                        _stream(stream)),
           "ckv_sparse_decode_append")


def ckv_kernel_timing(enable: bool) -> None:
    """Bracket every later launch with CUDA events (diagnostic; see ckv.h)."""
    _check(lib.ckv_kernel_timing(int(bool(enable))), "ckv_kernel_timing")


def ckv_kernel_times() -> dict:
    """{kind: (total ms, launches)} of the launches timed since the last read."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_int32 * n)()
    _check(lib.ckv_kernel_times(ms, cnt, n), "ckv_kernel_times")
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}


def ckv_get_device_error(graph: Graph, reset: bool = False, stream=None) -> int:
    """The graph's device error word (OR of DEVERR_* bits) once the stream's
    queued work is done; reset=True zeroes it afterwards."""
    code = ctypes.c_int32(0)
    _check(lib.ckv_get_device_error(ctypes.byref(graph.desc), _stream(stream), ctypes.byref(code), int(reset)),
           "ckv_get_device_error")
    return int(code.value)


def ckv_append_assign(cache: CacheDesc, graph: Graph, pos: int, k_new: torch.Tensor, v_new: torch.Tensor,
                      nbr8: torch.Tensor, assigned: Optional[torch.Tensor], stream=None) -> None:
    """k_new, v_new: [B, Hkv, d] contiguous in the cache dtype; written to
    row ``pos`` of K and V by the library, then the update runs."""
    _check_rows(cache, k_new=k_new, v_new=v_new)
    _check(lib.ckv_append_assign(ctypes.byref(cache), ctypes.byref(graph.desc), pos, k_new.data_ptr(),
                                 v_new.data_ptr(), nbr8.data_ptr(), _ptr(assigned), _stream(stream)),
           "ckv_append_assign")


def ckv_dense_decode(cache: CacheDesc, q: torch.Tensor, T: int, out: torch.Tensor, ws: torch.Tensor,
                     stream=None) -> None:
    _check(lib.ckv_dense_decode(ctypes.byref(cache), q.data_ptr(), T, out.data_ptr(), ws.data_ptr(),
                                ws.numel(), _stream(stream)),
           "ckv_dense_decode")


# ----------------------------------------------------------------------------
# the prefill token graph
# ----------------------------------------------------------------------------

@dataclass
class Edges:
    """Outputs of ckv_build_edges for U graph units of a T-token prefill."""
    nbr: torch.Tensor      # int32 [U, T, 8] direct-edge key positions, best first, -1 padded
    lam: torch.Tensor      # fp32 [U, T, 8] their graph logits
    co_src: torch.Tensor   # int32 [U, pair_cap]
    co_dst: torch.Tensor   # int32 [U, pair_cap]
    co_w: torch.Tensor     # int32 [U, pair_cap]
    co_n: torch.Tensor     # int32 [U]
    dev_err: torch.Tensor  # int32 [1]
    ws: torch.Tensor

    def pairs(self, u: int):
        """Unit u's co-attention edges as (src, dst, weight) rows, sorted."""
        n = min(int(self.co_n[u].item()), self.co_src.shape[1])
        t = torch.stack([self.co_src[u, :n], self.co_dst[u, :n], self.co_w[u, :n]], dim=1)
        if n == 0:
            return t
        order = torch.argsort(t[:, 0].long() * (1 << 31) + t[:, 1].long())
        return t[order]


def ckv_edges_workspace_size(cache: CacheDesc, mode: int, S: int, T: int) -> int:
    out = _sz(0)
    _check(lib.ckv_edges_workspace_size(ctypes.byref(cache), mode, S, T, ctypes.byref(out)),
           "ckv_edges_workspace_size")
    return int(out.value)


def new_edges(cache: CacheDesc, mode: int, S: int, T: int, pair_cap: Optional[int] = None, device="cuda") -> Edges:
    """Buffers for ckv_build_edges; pair_cap defaults to 28 (T - S), which can
    never overflow."""
    U = cache.B * (cache.Hq if mode == PER_HEAD else cache.Hkv)
    cap = max(1, 28 * max(T - S, 0)) if pair_cap is None else pair_cap
    i32 = dict(dtype=torch.int32, device=device)
    return Edges(nbr=torch.empty((U, T, NEIGHBOURS), **i32),
                 lam=torch.empty((U, T, NEIGHBOURS), dtype=torch.float32, device=device),
                 co_src=torch.empty((U, cap), **i32), co_dst=torch.empty((U, cap), **i32),
                 co_w=torch.empty((U, cap), **i32), co_n=torch.empty((U,), **i32),
                 dev_err=torch.zeros((1,), **i32),
                 ws=torch.empty((max(ckv_edges_workspace_size(cache, mode, S, T), 256),), dtype=torch.uint8,
                                device=device))


def ckv_build_edges(cache: CacheDesc, mode: int, S: int, q_prefill: torch.Tensor, T: int, edges: Edges,
                    stream=None) -> None:
    """q_prefill: [B, Hq, >=T, d] bf16, contiguous rows; fills `edges`."""
    if q_prefill.dtype != torch.bfloat16 or q_prefill.dim() != 4 or not q_prefill.is_contiguous():
        raise ValueError("q_prefill must be a contiguous bf16 [B, Hq, T, d] tensor")
    if q_prefill.shape[2] != T:
        raise ValueError("q_prefill's third dimension must be T")
    _check(lib.ckv_build_edges(ctypes.byref(cache), mode, S, q_prefill.data_ptr(), T, edges.nbr.data_ptr(),
                               edges.lam.data_ptr(), edges.co_src.data_ptr(), edges.co_dst.data_ptr(),
                               edges.co_w.data_ptr(), edges.co_n.data_ptr(), edges.co_src.shape[1],
                               edges.dev_err.data_ptr(), edges.ws.data_ptr(), edges.ws.numel(), _stream(stream)),
           "ckv_build_edges")
