// Local community update for a newly generated token, sm_100a.
//
// A new token never triggers a global re-partition: it is attached to one of
// the neighbouring communities and only that community's centre changes, at a
// cost set by the head dimension rather than the context length (CommunityKV,
// rit.work summary, section "A graph of tokens replaces re-clustering",
// paragraph 6; the abstract describes the rule as constant-time).
//
// One warp per graph unit: the candidate communities are those of the 8
// neighbour positions found by the attention kernel; each distinct candidate
// costs one d-long dot product with the new key; the winner's centre moves
// by (k - c)/(n + 1) and its count grows by one.  O(8 d) work per graph.
#include <math.h>

#include "ckv_internal.cuh"

namespace ckv {

struct AssignParams {
    const void* k;
    int64_t sb, sh, st;
    int U, G, Hq, Hkv, per_head, Cmax, T_cap, max_tail, pos;
    float inv_sqrt_d;
    const int32_t* nbr8;
    int32_t* comm_of;
    int32_t* cnt;
    float* cent;
    int32_t* tail_tok;
    int32_t* tail_comm;
    int32_t* tail_len;
    int32_t* dev_err;
    int32_t* assigned;
};

template <typename T, int D>
__global__ void __launch_bounds__(128) assign_kernel(AssignParams p) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const int u = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (u >= p.U) return;
    const int b = u / p.G, g = u - b * p.G;
    const int kvh = p.per_head ? g / (p.Hq / p.Hkv) : g;
    const T* krow = static_cast<const T*>(p.k) + b * p.sb + kvh * p.sh + (int64_t)p.pos * p.st + lane * E;
    float kx[E];
#pragma unroll
    for (int e = 0; e < E; ++e) kx[e] = to_f32(krow[e]);

    int cand = -1;
    if (lane < CKV_NEIGHBOURS) {
        const int np = p.nbr8[(size_t)u * CKV_NEIGHBOURS + lane];
        if (np >= 0 && np < p.T_cap) {
            const int c = p.comm_of[(size_t)u * p.T_cap + np];
            if (c >= 0 && c < p.Cmax) cand = c;
        }
    }
    int best = -1;
    float best_s = -INFINITY;
    for (int i = 0; i < CKV_NEIGHBOURS; ++i) {
        const int ci = __shfl_sync(FULL, cand, i);
        if (ci < 0) continue;
        if (__ballot_sync(FULL, lane < i && cand == ci)) continue;  // seen already
        const float* cr = p.cent + ((size_t)u * p.Cmax + ci) * D + lane * E;
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) a = fmaf(kx[e], cr[e], a);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
        const float s = a * p.inv_sqrt_d;
        if (best < 0 || s > best_s || (s == best_s && ci < best)) {
            best = ci;
            best_s = s;
        }
    }
    int32_t* cpos = p.comm_of + (size_t)u * p.T_cap + p.pos;
    if (best < 0) {
        if (lane == 0) {
            *cpos = -1;
            if (p.assigned) p.assigned[u] = -1;
        }
        return;
    }
    int tl = 0;
    if (lane == 0) tl = p.tail_len[u];
    tl = __shfl_sync(FULL, tl, 0);
    if (tl >= p.max_tail) {
        if (lane == 0) {
            *cpos = -1;
            atomicOr(p.dev_err, CKV_DEVERR_TAIL_FULL);
            if (p.assigned) p.assigned[u] = -1;
        }
        return;
    }
    int n = 0;
    if (lane == 0) n = p.cnt[(size_t)u * p.Cmax + best];
    n = __shfl_sync(FULL, n, 0);
    float* cr = p.cent + ((size_t)u * p.Cmax + best) * D + lane * E;
    const float denom = (float)(n + 1);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float c0 = cr[e];
        cr[e] = c0 + (kx[e] - c0) / denom;
    }
    if (lane == 0) {
        p.cnt[(size_t)u * p.Cmax + best] = n + 1;
        *cpos = best;
        p.tail_tok[(size_t)u * p.max_tail + tl] = p.pos;
        p.tail_comm[(size_t)u * p.max_tail + tl] = best;
        p.tail_len[u] = tl + 1;
        if (p.assigned) p.assigned[u] = best;
    }
}

cudaError_t launch_assign_update(const CacheView& c, const GraphView& g, int pos, const int32_t* nbr8,
                                 int32_t* assigned, cudaStream_t st) {
    AssignParams p{};
    p.k = c.k;
    p.sb = c.sb;
    p.sh = c.sh;
    p.st = c.st;
    p.U = c.B * g.G;
    p.G = g.G;
    p.Hq = c.Hq;
    p.Hkv = c.Hkv;
    p.per_head = g.mode == CKV_GRAPH_PER_HEAD;
    p.Cmax = g.Cmax;
    p.T_cap = g.T_cap;
    p.max_tail = g.max_tail;
    p.pos = pos;
    p.inv_sqrt_d = 1.0f / sqrtf((float)c.d);
    p.nbr8 = nbr8;
    p.comm_of = g.comm_of;
    p.cnt = g.cnt;
    p.cent = g.cent;
    p.tail_tok = g.tail_tok;
    p.tail_comm = g.tail_comm;
    p.tail_len = g.tail_len;
    p.dev_err = g.dev_err;
    p.assigned = assigned;
    const int blocks = (p.U + 3) / 4;
    if (c.dtype == CKV_DTYPE_BF16) {
        if (c.d == 128) assign_kernel<__nv_bfloat16, 128><<<blocks, 128, 0, st>>>(p);
        else assign_kernel<__nv_bfloat16, 64><<<blocks, 128, 0, st>>>(p);
    } else {
        if (c.d == 128) assign_kernel<float, 128><<<blocks, 128, 0, st>>>(p);
        else assign_kernel<float, 64><<<blocks, 128, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace ckv
