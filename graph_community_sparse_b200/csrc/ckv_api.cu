// Host side of the libckv C ABI: argument checks, workspace sizing, dispatch.
// Every check runs before any CUDA call, so a rejected call never touches the
// device.  See include/ckv.h for the contract of each entry point.
#include <stdarg.h>
#include <stdio.h>

#include <string>

#include "ckv_assign.cuh"
#include "ckv_internal.cuh"

namespace {

thread_local std::string g_last_error;

ckv_status fail(ckv_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

ckv_status ok() {
    g_last_error.clear();
    return CKV_OK;
}

ckv_status cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return ok();
    return fail(CKV_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dtype) { return dtype == CKV_DTYPE_BF16 ? 2 : 4; }

ckv_status check_cache(const ckv_cache_desc* c, bool need_kv) {
    if (!c) return fail(CKV_ERR_INVALID_ARG, "cache descriptor is NULL");
    if (c->dtype != CKV_DTYPE_F32 && c->dtype != CKV_DTYPE_BF16)
        return fail(CKV_ERR_UNSUPPORTED, "dtype %d is not CKV_DTYPE_F32 or CKV_DTYPE_BF16", c->dtype);
    if (c->B < 1 || c->Hkv < 1 || c->Hq < 1 || c->T_cap < 1)
        return fail(CKV_ERR_INVALID_ARG, "B, Hkv, Hq and T_cap must be >= 1");
    if (c->Hq % c->Hkv != 0) return fail(CKV_ERR_INVALID_ARG, "Hq %% Hkv != 0");
    const int gq = c->Hq / c->Hkv;
    if (gq != 1 && gq != 2 && gq != 4 && gq != 8)
        return fail(CKV_ERR_UNSUPPORTED, "Hq/Hkv = %d not in {1,2,4,8}", gq);
    if (c->d != 64 && c->d != 128) return fail(CKV_ERR_UNSUPPORTED, "d = %d not in {64,128}", c->d);
    if (need_kv) {
        if (!c->k || !c->v) return fail(CKV_ERR_INVALID_ARG, "K or V pointer is NULL");
        if (c->stride_t < c->d || c->stride_h < 1 || c->stride_b < 1)
            return fail(CKV_ERR_INVALID_ARG, "strides must be positive and stride_t >= d");
        const int64_t es = elem_size(c->dtype);
        if (!aligned16(c->k) || !aligned16(c->v) || (c->stride_t * es) % 16 || (c->stride_h * es) % 16 ||
            (c->stride_b * es) % 16)
            return fail(CKV_ERR_MISALIGNED, "K/V base pointers and byte strides must be multiples of 16");
    }
    return CKV_OK;
}

int graphs_per_seq(const ckv_cache_desc* c, const ckv_graph_desc* g) {
    return g->mode == CKV_GRAPH_PER_HEAD ? c->Hq : c->Hkv;
}

ckv_status check_graph(const ckv_cache_desc* c, const ckv_graph_desc* g) {
    if (!g) return fail(CKV_ERR_INVALID_ARG, "graph descriptor is NULL");
    if (g->mode != CKV_GRAPH_PER_GROUP && g->mode != CKV_GRAPH_PER_HEAD)
        return fail(CKV_ERR_INVALID_ARG, "graph mode %d unknown", g->mode);
    if (g->S < 0) return fail(CKV_ERR_INVALID_ARG, "S < 0");
    if (g->assign_rule != CKV_ASSIGN_SCORE && g->assign_rule != CKV_ASSIGN_VOTE)
        return fail(CKV_ERR_INVALID_ARG, "assign rule %d unknown", g->assign_rule);
    if (g->Cmax < 1 || g->Cmax > ckv::MAX_CMAX)
        return fail(CKV_ERR_UNSUPPORTED, "Cmax = %d outside [1, %d]", g->Cmax, ckv::MAX_CMAX);
    if (g->max_tail < 0) return fail(CKV_ERR_INVALID_ARG, "max_tail < 0");
    if (g->T_cap != c->T_cap) return fail(CKV_ERR_INVALID_ARG, "graph T_cap %d != cache T_cap %d", g->T_cap, c->T_cap);
    if (g->S > g->T_cap) return fail(CKV_ERR_CAPACITY, "S > T_cap");
    const int64_t U = (int64_t)c->B * graphs_per_seq(c, g);
    if (U > ckv::MAX_UNITS) return fail(CKV_ERR_UNSUPPORTED, "B*G = %lld above %d", (long long)U, ckv::MAX_UNITS);
    if (!g->comm_of || !g->offs || !g->tok || !g->cnt || !g->cent || !g->cent_q || !g->cent_qs || !g->num_comm ||
        !g->tail_len ||
        !g->dev_err || (g->max_tail > 0 && (!g->tail_tok || !g->tail_comm)))
        return fail(CKV_ERR_INVALID_ARG, "a graph array pointer is NULL");
    if (!aligned16(g->cent) || !aligned16(g->cent_q) || !aligned16(g->cent_qs))
        return fail(CKV_ERR_MISALIGNED, "cent, cent_q and cent_qs must be 16-byte aligned");
    if (U * (int64_t)g->T_cap > (int64_t)1 << 31 || U * (int64_t)g->Cmax * c->d > (int64_t)1 << 40)
        return fail(CKV_ERR_UNSUPPORTED, "graph arrays too large");
    return CKV_OK;
}

ckv_status check_sel(const ckv_graph_desc* g, const ckv_selection_desc* s, int64_t U) {
    if (!s) return fail(CKV_ERR_INVALID_ARG, "selection descriptor is NULL");
    if (!s->sel_comm || !s->n_sel || !s->sel_tok || !s->n_tok || !s->tok_prefix || !s->tail_sel || !s->unit_prefix)
        return fail(CKV_ERR_INVALID_ARG, "a selection array pointer is NULL");
    if (s->tok_cap < 1 || s->tok_cap < g->S) return fail(CKV_ERR_INVALID_ARG, "tok_cap must be >= max(S, 1)");
    if (U * (int64_t)s->tok_cap > (int64_t)1 << 30)
        return fail(CKV_ERR_UNSUPPORTED, "B*G*tok_cap above 2^30");
    return CKV_OK;
}

ckv_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (need == 0) return CKV_OK;
    if (!ws) return fail(CKV_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(CKV_ERR_WORKSPACE, "workspace not 256-byte aligned");
    if (ws_bytes < need) return fail(CKV_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    return CKV_OK;
}

ckv::CacheView cache_view(const ckv_cache_desc* c) {
    ckv::CacheView v;
    v.k = c->k;
    v.v = c->v;
    v.sb = c->stride_b;
    v.sh = c->stride_h;
    v.st = c->stride_t;
    v.B = c->B;
    v.Hkv = c->Hkv;
    v.Hq = c->Hq;
    v.d = c->d;
    v.T_cap = c->T_cap;
    v.dtype = c->dtype;
    return v;
}

ckv::GraphView graph_view(const ckv_cache_desc* c, const ckv_graph_desc* g) {
    ckv::GraphView v;
    v.mode = g->mode;
    v.S = g->S;
    v.Cmax = g->Cmax;
    v.max_tail = g->max_tail;
    v.T_cap = g->T_cap;
    v.rule = g->assign_rule;
    v.G = graphs_per_seq(c, g);
    v.gq = g->mode == CKV_GRAPH_PER_HEAD ? 1 : c->Hq / c->Hkv;
    v.comm_of = g->comm_of;
    v.offs = g->offs;
    v.tok = g->tok;
    v.cnt = g->cnt;
    v.cent = g->cent;
    v.cent_q = g->cent_q;
    v.cent_qs = g->cent_qs;
    v.num_comm = g->num_comm;
    v.tail_tok = g->tail_tok;
    v.tail_comm = g->tail_comm;
    v.tail_len = g->tail_len;
    v.dev_err = g->dev_err;
    return v;
}

ckv::SelView sel_view(const ckv_selection_desc* s) {
    ckv::SelView v;
    v.tok_cap = s->tok_cap;
    v.sel_comm = s->sel_comm;
    v.n_sel = s->n_sel;
    v.sel_tok = s->sel_tok;
    v.n_tok = s->n_tok;
    v.unit_prefix = s->unit_prefix;
    v.tok_prefix = s->tok_prefix;
    v.tail_sel = s->tail_sel;
    return v;
}

#define CKV_TRY(expr)                      \
    do {                                   \
        ckv_status _s = (expr);            \
        if (_s != CKV_OK) return _s;       \
    } while (0)

}  // namespace

extern "C" {

int32_t ckv_abi_version(void) { return CKV_ABI_VERSION; }

int32_t ckv_debug_build(void) { return ckv::kDebugChecks ? 1 : 0; }

static_assert(ckv::KK_COUNT == CKV_KERNEL_KINDS && ckv::KK_ATTENTION == CKV_KERNEL_ATTENTION &&
                  ckv::KK_UPDATE == CKV_KERNEL_UPDATE && ckv::KK_EDGES == CKV_KERNEL_EDGES,
              "kernel kinds match the header");

ckv_status ckv_kernel_timing(int32_t enable) {
    ckv::timing_set(enable != 0);
    return ok();
}

ckv_status ckv_kernel_times(float* total_ms, int32_t* launches, int32_t n) {
    if (!total_ms || !launches) return fail(CKV_ERR_INVALID_ARG, "total_ms or launches is NULL");
    if (n < CKV_KERNEL_KINDS) return fail(CKV_ERR_INVALID_ARG, "n = %d < %d kernel kinds", n, CKV_KERNEL_KINDS);
    return cuda_status(ckv::timing_read(total_ms, launches), "ckv_kernel_times");
}

ckv_status ckv_get_device_error(const ckv_graph_desc* graph, ckv_stream_t stream, int32_t* code, int32_t reset) {
    if (!graph || !graph->dev_err) return fail(CKV_ERR_INVALID_ARG, "graph descriptor or its dev_err is NULL");
    if (!code) return fail(CKV_ERR_INVALID_ARG, "code is NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, graph->dev_err, sizeof(word), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && reset && word != 0) e = cudaMemsetAsync(graph->dev_err, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return cuda_status(e, "ckv_get_device_error");
    *code = word;
    return ok();
}

const char* ckv_status_string(ckv_status s) {
    switch (s) {
        case CKV_OK: return "CKV_OK";
        case CKV_ERR_INVALID_ARG: return "CKV_ERR_INVALID_ARG";
        case CKV_ERR_MISALIGNED: return "CKV_ERR_MISALIGNED";
        case CKV_ERR_UNSUPPORTED: return "CKV_ERR_UNSUPPORTED";
        case CKV_ERR_CAPACITY: return "CKV_ERR_CAPACITY";
        case CKV_ERR_WORKSPACE: return "CKV_ERR_WORKSPACE";
        case CKV_ERR_CUDA: return "CKV_ERR_CUDA";
    }
    return "CKV_ERR_UNKNOWN";
}

const char* ckv_last_error(void) { return g_last_error.c_str(); }

ckv_status ckv_workspace_size(const ckv_cache_desc* cache, const ckv_graph_desc* graph,
                              const ckv_selection_desc* sel, size_t* bytes) {
    if (!bytes) return fail(CKV_ERR_INVALID_ARG, "bytes is NULL");
    CKV_TRY(check_cache(cache, false));
    const int gq_dense = cache->Hq / cache->Hkv;
    size_t need = ckv::decode_ws_bytes(cache->B * cache->Hkv, gq_dense, cache->d, 0);
    if (graph) {
        CKV_TRY(check_graph(cache, graph));
        const int U = cache->B * graphs_per_seq(cache, graph);
        const int gq = graph->mode == CKV_GRAPH_PER_HEAD ? 1 : gq_dense;
        const size_t a = ckv::build_ws_bytes(U, graph->Cmax, graph->T_cap);
        const size_t b = ckv::select_ws_bytes(U, graph->Cmax);
        const size_t c = ckv::decode_ws_bytes(U, gq, cache->d, sel ? sel->tok_cap : graph->T_cap);
        need = need > a ? need : a;
        need = need > b ? need : b;
        need = need > c ? need : c;
    }
    *bytes = ckv::ws_head_bytes(cache->B, cache->Hq) + need;
    return ok();
}

ckv_status ckv_build_centroids(const ckv_cache_desc* cache, const int32_t* labels, int64_t labels_stride,
                               int32_t T, const ckv_graph_desc* graph, void* ws, size_t ws_bytes,
                               ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    CKV_TRY(check_graph(cache, graph));
    if (!labels) return fail(CKV_ERR_INVALID_ARG, "labels is NULL");
    if (T < graph->S) return fail(CKV_ERR_INVALID_ARG, "T = %d < S = %d", T, graph->S);
    if (T > cache->T_cap) return fail(CKV_ERR_CAPACITY, "T = %d > T_cap = %d", T, cache->T_cap);
    if (labels_stride < T) return fail(CKV_ERR_INVALID_ARG, "labels_stride < T");
    const int U = cache->B * graphs_per_seq(cache, graph);
    const size_t head = ckv::ws_head_bytes(cache->B, cache->Hq);
    CKV_TRY(check_ws(ws, ws_bytes, head + ckv::build_ws_bytes(U, graph->Cmax, graph->T_cap)));
    return cuda_status(ckv::launch_build(cache_view(cache), graph_view(cache, graph), labels, labels_stride, T,
                                         static_cast<char*>(ws) + head,
                                         reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_build_centroids");
}

ckv_status ckv_score_select(const ckv_cache_desc* cache, const ckv_graph_desc* graph, const void* q,
                            int32_t budget, const ckv_selection_desc* sel, void* ws, size_t ws_bytes,
                            ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, false));
    CKV_TRY(check_graph(cache, graph));
    const int64_t U = (int64_t)cache->B * graphs_per_seq(cache, graph);
    CKV_TRY(check_sel(graph, sel, U));
    if (!q) return fail(CKV_ERR_INVALID_ARG, "q is NULL");
    if (!aligned16(q)) return fail(CKV_ERR_MISALIGNED, "q must be 16-byte aligned");
    if (budget < 0) return fail(CKV_ERR_INVALID_ARG, "budget < 0");
    CKV_TRY(check_ws(ws, ws_bytes,
                     ckv::ws_head_bytes(cache->B, cache->Hq) + ckv::select_ws_bytes((int)U, graph->Cmax)));
    return cuda_status(ckv::launch_score_select(cache_view(cache), graph_view(cache, graph), q, budget,
                                                sel_view(sel), ws, reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_score_select");
}

ckv_status ckv_sparse_decode(const ckv_cache_desc* cache, const void* q, const ckv_graph_desc* graph,
                             const ckv_selection_desc* sel, float* out, int32_t* nbr8, void* ws,
                             size_t ws_bytes, ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    CKV_TRY(check_graph(cache, graph));
    const int64_t U = (int64_t)cache->B * graphs_per_seq(cache, graph);
    CKV_TRY(check_sel(graph, sel, U));
    if (!q || !out) return fail(CKV_ERR_INVALID_ARG, "q or out is NULL");
    if (!aligned16(q) || !aligned16(out)) return fail(CKV_ERR_MISALIGNED, "q and out must be 16-byte aligned");
    const int gq = graph->mode == CKV_GRAPH_PER_HEAD ? 1 : cache->Hq / cache->Hkv;
    CKV_TRY(check_ws(ws, ws_bytes,
                     ckv::ws_head_bytes(cache->B, cache->Hq) + ckv::decode_ws_bytes((int)U, gq, cache->d, sel->tok_cap)));
    return cuda_status(ckv::launch_sparse_decode(cache_view(cache), graph_view(cache, graph), sel_view(sel), q,
                                                 out, nbr8, ws, nullptr, reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_sparse_decode");
}

// Same validation and kernels as ckv_sparse_decode; the scratch is the
// library's fixed array instead of a caller workspace, so nothing is
// allocated.  Sizes whose scratch would not fit are refused up front.
ckv_status ckv_sparse_decode_noalloc(const ckv_cache_desc* cache, const void* q, const ckv_graph_desc* graph,
                                     const ckv_selection_desc* sel, float* out, int32_t* nbr8,
                                     ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    CKV_TRY(check_graph(cache, graph));
    const int64_t U = (int64_t)cache->B * graphs_per_seq(cache, graph);
    CKV_TRY(check_sel(graph, sel, U));
    if (!q || !out) return fail(CKV_ERR_INVALID_ARG, "q or out is NULL");
    if (!aligned16(q) || !aligned16(out)) return fail(CKV_ERR_MISALIGNED, "q and out must be 16-byte aligned");
    const int gq = graph->mode == CKV_GRAPH_PER_HEAD ? 1 : cache->Hq / cache->Hkv;
    const size_t need = ckv::ws_head_bytes(cache->B, cache->Hq) + ckv::decode_ws_bytes((int)U, gq, cache->d, sel->tok_cap);
    if (need > CKV_NOALLOC_SCRATCH_BYTES)
        return fail(CKV_ERR_UNSUPPORTED,
                    "ckv_sparse_decode_noalloc: these shapes need %zu bytes of scratch, above the library's "
                    "fixed %zu; use ckv_sparse_decode with a workspace",
                    need, (size_t)CKV_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    size_t have = 0;
    cudaError_t e = ckv::static_decode_scratch(&scratch, &have);
    if (e != cudaSuccess) return cuda_status(e, "ckv_sparse_decode_noalloc: scratch address lookup");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    e = ckv::launch_sparse_decode(cache_view(cache), graph_view(cache, graph), sel_view(sel), q, out, nbr8, scratch,
                                  nullptr, st);
    if (e != cudaSuccess) {
        // a kernel enqueued before the failed launch may leave the head's
        // counters nonzero; zero them so later calls start clean
        (void)cudaMemsetAsync(scratch, 0, ckv::ws_head_bytes(cache->B, cache->Hq), st);
    }
    return cuda_status(e, "ckv_sparse_decode_noalloc");
}

ckv_status ckv_assign_update(const ckv_cache_desc* cache, const ckv_graph_desc* graph, int32_t pos,
                             const int32_t* nbr8, int32_t* assigned, ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    CKV_TRY(check_graph(cache, graph));
    if (!nbr8) return fail(CKV_ERR_INVALID_ARG, "nbr8 is NULL");
    if (pos < 0 || pos >= cache->T_cap) return fail(CKV_ERR_CAPACITY, "pos = %d outside [0, T_cap)", pos);
    return cuda_status(ckv::launch_assign_update(cache_view(cache), graph_view(cache, graph), pos, nullptr,
                                                 nullptr, nbr8, assigned, reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_assign_update");
}

ckv_status ckv_append_assign(const ckv_cache_desc* cache, const ckv_graph_desc* graph, int32_t pos,
                             const void* k_new, const void* v_new, const int32_t* nbr8, int32_t* assigned,
                             ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    CKV_TRY(check_graph(cache, graph));
    if (!nbr8) return fail(CKV_ERR_INVALID_ARG, "nbr8 is NULL");
    if (!k_new || !v_new) return fail(CKV_ERR_INVALID_ARG, "k_new or v_new is NULL");
    if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15)
        return fail(CKV_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
    if (pos < 0 || pos >= cache->T_cap) return fail(CKV_ERR_CAPACITY, "pos = %d outside [0, T_cap)", pos);
    return cuda_status(ckv::launch_assign_update(cache_view(cache), graph_view(cache, graph), pos, k_new, v_new,
                                                 nbr8, assigned, reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_append_assign");
}

ckv_status ckv_sparse_decode_append(const ckv_cache_desc* cache, const void* q, const ckv_graph_desc* graph,
                                    const ckv_selection_desc* sel, float* out, int32_t* nbr8, int32_t pos,
                                    const void* k_new, const void* v_new, int32_t* assigned, void* ws,
                                    size_t ws_bytes, ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    CKV_TRY(check_graph(cache, graph));
    const int64_t U = (int64_t)cache->B * graphs_per_seq(cache, graph);
    CKV_TRY(check_sel(graph, sel, U));
    if (!q || !out) return fail(CKV_ERR_INVALID_ARG, "q or out is NULL");
    if (!aligned16(q) || !aligned16(out)) return fail(CKV_ERR_MISALIGNED, "q and out must be 16-byte aligned");
    if (!k_new || !v_new) return fail(CKV_ERR_INVALID_ARG, "k_new or v_new is NULL");
    if (!aligned16(k_new) || !aligned16(v_new))
        return fail(CKV_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
    if (pos < 0 || pos >= cache->T_cap) return fail(CKV_ERR_CAPACITY, "pos = %d outside [0, T_cap)", pos);
    const int gq = graph->mode == CKV_GRAPH_PER_HEAD ? 1 : cache->Hq / cache->Hkv;
    CKV_TRY(check_ws(ws, ws_bytes,
                     ckv::ws_head_bytes(cache->B, cache->Hq) + ckv::decode_ws_bytes((int)U, gq, cache->d, sel->tok_cap)));
    const ckv::CacheView cv = cache_view(cache);
    const ckv::GraphView gv = graph_view(cache, graph);
    const ckv::AssignParams ap = ckv::make_assign_params(cv, gv, pos, k_new, v_new, nullptr, assigned);
    return cuda_status(ckv::launch_sparse_decode(cv, gv, sel_view(sel), q, out, nbr8, ws, &ap,
                                                 reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_sparse_decode_append");
}

ckv_status ckv_edges_workspace_size(const ckv_cache_desc* cache, int32_t mode, int32_t S, int32_t T, size_t* bytes) {
    if (!bytes) return fail(CKV_ERR_INVALID_ARG, "bytes is NULL");
    CKV_TRY(check_cache(cache, false));
    if (mode != CKV_GRAPH_PER_GROUP && mode != CKV_GRAPH_PER_HEAD)
        return fail(CKV_ERR_INVALID_ARG, "graph mode %d unknown", mode);
    if (S < 0 || T < S || T > cache->T_cap) return fail(CKV_ERR_INVALID_ARG, "need 0 <= S <= T <= T_cap");
    const int U = cache->B * (mode == CKV_GRAPH_PER_HEAD ? cache->Hq : cache->Hkv);
    *bytes = ckv::edges_ws_bytes(U, T, S);
    return ok();
}

ckv_status ckv_build_edges(const ckv_cache_desc* cache, int32_t mode, int32_t S, const void* q_prefill, int32_t T,
                           int32_t* nbr, float* lam, int32_t* co_src, int32_t* co_dst, int32_t* co_w, int32_t* co_n,
                           int32_t pair_cap, int32_t* dev_err, void* ws, size_t ws_bytes, ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    if (cache->dtype != CKV_DTYPE_BF16) return fail(CKV_ERR_UNSUPPORTED, "ckv_build_edges takes bf16 caches only");
    if (mode != CKV_GRAPH_PER_GROUP && mode != CKV_GRAPH_PER_HEAD)
        return fail(CKV_ERR_INVALID_ARG, "graph mode %d unknown", mode);
    if (S < 0 || T < S) return fail(CKV_ERR_INVALID_ARG, "need 0 <= S <= T");
    if (T > cache->T_cap) return fail(CKV_ERR_CAPACITY, "T = %d > T_cap = %d", T, cache->T_cap);
    if (!q_prefill || !nbr || !co_src || !co_dst || !co_w || !co_n || !dev_err)
        return fail(CKV_ERR_INVALID_ARG, "an output or input pointer is NULL");
    if (!aligned16(q_prefill)) return fail(CKV_ERR_MISALIGNED, "q_prefill must be 16-byte aligned");
    if (pair_cap < 1) return fail(CKV_ERR_INVALID_ARG, "pair_cap < 1");
    const int64_t U = (int64_t)cache->B * (mode == CKV_GRAPH_PER_HEAD ? cache->Hq : cache->Hkv);
    if (U > ckv::MAX_UNITS || U * (int64_t)T * 8 > (int64_t)1 << 31 || U * (int64_t)pair_cap > (int64_t)1 << 31)
        return fail(CKV_ERR_UNSUPPORTED, "edge arrays too large");
    CKV_TRY(check_ws(ws, ws_bytes, ckv::edges_ws_bytes((int)U, T, S)));
    return cuda_status(ckv::launch_build_edges(cache_view(cache), mode, S, q_prefill, T, nbr, lam, co_src, co_dst, co_w,
                                               co_n, pair_cap, dev_err, ws, reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_build_edges");
}

ckv_status ckv_dense_decode(const ckv_cache_desc* cache, const void* q, int32_t T, float* out, void* ws,
                            size_t ws_bytes, ckv_stream_t stream) {
    CKV_TRY(check_cache(cache, true));
    if (!q || !out) return fail(CKV_ERR_INVALID_ARG, "q or out is NULL");
    if (!aligned16(q) || !aligned16(out)) return fail(CKV_ERR_MISALIGNED, "q and out must be 16-byte aligned");
    if (T < 1 || T > cache->T_cap) return fail(CKV_ERR_CAPACITY, "T = %d outside [1, T_cap]", T);
    const int64_t U = (int64_t)cache->B * cache->Hkv;
    if (U * T > (int64_t)1 << 30) return fail(CKV_ERR_UNSUPPORTED, "B*Hkv*T above 2^30");
    CKV_TRY(check_ws(ws, ws_bytes,
                     ckv::ws_head_bytes(cache->B, cache->Hq) + ckv::decode_ws_bytes((int)U, cache->Hq / cache->Hkv, cache->d, 0)));
    return cuda_status(ckv::launch_dense_decode(cache_view(cache), q, T, out, ws,
                                                reinterpret_cast<cudaStream_t>(stream)),
                       "ckv_dense_decode");
}

}  // extern "C"
