// Local community update for one graph unit (device code shared by the
// stand-alone update kernel and the attention merge kernel).
//
// A new token never triggers a global re-partition: it is attached to one of
// the neighbouring communities and only that community's centre changes, at a
// cost set by the head dimension rather than the context length (CommunityKV,
// rit.work summary, section "A graph of tokens replaces re-clustering",
// paragraph 6; the abstract describes the rule as constant-time).
//
// The candidate communities are those of the 8 neighbour positions found by
// the attention; each distinct candidate costs one d-long dot product with
// the new key; the winner (largest k . c / sqrt(d), ties to the lower id; or,
// under the vote rule, the candidate named by the most neighbours, the score
// and then the id breaking ties) moves its centre by (k - c)/(n + 1), its count grows by one and (pos, c)
// joins the unit's tail.  O(8 d) work per graph.
#pragma once

#include "ckv_internal.cuh"

namespace ckv {

struct AssignParams {
    const void* k;      // new key rows: the cache at pos, or the caller's k_new
    int64_t sb, sh;     // element strides of k between sequences / KV heads
    // fused append: copy the caller's rows into the cache at pos
    const void* k_new;
    const void* v_new;
    void* k_dst;        // K row (b = 0, kv head 0) at pos; NULL: no append
    void* v_dst;
    int64_t csb, csh;   // cache element strides between sequences / KV heads
    int row_vec;        // 16-byte vectors per row
    int U, G, Hq, Hkv, d, per_head, Cmax, T_cap, max_tail, pos;
    int vote;           // CKV_ASSIGN_VOTE: most neighbours first, the score breaks ties
    float inv_sqrt_d;
    const int32_t* nbr8;
    int32_t* comm_of;
    int32_t* cnt;
    float* cent;
    int8_t* cent_q;
    float* cent_qs;
    int32_t* tail_tok;
    int32_t* tail_comm;
    int32_t* tail_len;
    int32_t* dev_err;
    int32_t* assigned;
};

// Fills the fields that come from the cache, the graph and the call.
// k_new/v_new NULL: the new key is read from the cache at pos; otherwise it
// comes from k_new and both rows are first written to the cache at pos.
inline AssignParams make_assign_params(const CacheView& c, const GraphView& g, int pos, const void* k_new,
                                       const void* v_new, const int32_t* nbr8, int32_t* assigned) {
    AssignParams p{};
    const size_t esz = c.dtype == CKV_DTYPE_BF16 ? 2 : 4;
    if (k_new) {
        p.k = k_new;
        p.sb = (int64_t)c.Hkv * c.d;
        p.sh = c.d;
        p.k_new = k_new;
        p.v_new = v_new;
        p.k_dst = const_cast<char*>(static_cast<const char*>(c.k)) + (size_t)pos * c.st * esz;
        p.v_dst = const_cast<char*>(static_cast<const char*>(c.v)) + (size_t)pos * c.st * esz;
    } else {
        p.k = static_cast<const char*>(c.k) + (size_t)pos * c.st * esz;
        p.sb = c.sb;
        p.sh = c.sh;
    }
    p.csb = c.sb;
    p.csh = c.sh;
    p.row_vec = (int)(c.d * esz / 16);
    p.U = c.B * g.G;
    p.G = g.G;
    p.Hq = c.Hq;
    p.Hkv = c.Hkv;
    p.d = c.d;
    p.per_head = g.mode == CKV_GRAPH_PER_HEAD;
    p.Cmax = g.Cmax;
    p.T_cap = g.T_cap;
    p.max_tail = g.max_tail;
    p.pos = pos;
    p.vote = g.rule == CKV_ASSIGN_VOTE;
    p.inv_sqrt_d = 1.0f / sqrtf((float)c.d);
    p.nbr8 = nbr8;
    p.comm_of = g.comm_of;
    p.cnt = g.cnt;
    p.cent = g.cent;
    p.cent_q = g.cent_q;
    p.cent_qs = g.cent_qs;
    p.tail_tok = g.tail_tok;
    p.tail_comm = g.tail_comm;
    p.tail_len = g.tail_len;
    p.dev_err = g.dev_err;
    p.assigned = assigned;
    return p;
}

// Shared-memory scratch of one unit's update (the caller provides it: the
// stand-alone kernel as a shared variable, the attention's merging warp in
// its own staging ring, which is idle by then).
template <int D>
struct AssignScratch {
    int cand[CKV_NEIGHBOURS];
    float score[CKV_NEIGHBOURS];
    int cnt[CKV_NEIGHBOURS];
    int tl;
    int pad[3];
    float row[CKV_NEIGHBOURS][D];  // candidate centres, reused by the update
};

// Fused append: the first graph of each (sequence, KV head) copies the
// caller's new K and V rows into the cache at pos (threads t of nthr, one
// 16-byte vector each per step).
__device__ __forceinline__ void append_rows(const AssignParams& p, int u, int t, int nthr) {
    if (!p.k_dst) return;
    const int b = u / p.G, g = u - b * p.G;
    const int gq = p.Hq / p.Hkv;
    if (p.per_head && g % gq != 0) return;
    const int kvh = p.per_head ? g / gq : g;
    const uint4* ks = static_cast<const uint4*>(p.k_new) + ((size_t)b * p.Hkv + kvh) * p.row_vec;
    const uint4* vs = static_cast<const uint4*>(p.v_new) + ((size_t)b * p.Hkv + kvh) * p.row_vec;
    const size_t eoff = (size_t)(b * p.csb + kvh * p.csh);  // elements
    const size_t esz = p.row_vec * 16 / (size_t)p.d;
    uint4* kd = reinterpret_cast<uint4*>(static_cast<char*>(p.k_dst) + eoff * esz);
    uint4* vd = reinterpret_cast<uint4*>(static_cast<char*>(p.v_dst) + eoff * esz);
    for (int i = t; i < p.row_vec; i += nthr) {
        kd[i] = ks[i];
        vd[i] = vs[i];
    }
}

// The update of unit u by NW warps (thread index tid in [0, 32 NW)), given
// the unit's 8 neighbour positions (-1: none) in nbrpos, readable by all of
// them.  sync() is a barrier over exactly these NW warps.  Warp w scores
// candidates w, w + NW, ... with all of their centres requested before any
// is used; warp 0 picks the winner and moves its centre.  APPEND: the last
// warp also writes the new K/V rows (append_rows; the attention's merge
// kernel does that itself, off the update's path).
template <typename T, int D, int NW, bool APPEND, typename Sync>
__device__ __forceinline__ void assign_unit(const AssignParams& p, int u, const int* nbrpos, int tid,
                                            AssignScratch<D>& sc, Sync sync) {
    constexpr int E = D / 32;
    constexpr int PER = CKV_NEIGHBOURS / NW;  // candidates per warp
    static_assert(E == 2 || E == 4, "d is 64 or 128");
    static_assert(CKV_NEIGHBOURS % NW == 0, "whole candidates per warp");
    const int lane = tid & 31, warp = NW == 1 ? 0 : tid >> 5;
    const int b = u / p.G, g = u - b * p.G;
    const int gq = p.Hq / p.Hkv;
    const int kvh = p.per_head ? g / gq : g;
    if (APPEND && warp == NW - 1) append_rows(p, u, lane, 32);
    if (tid < CKV_NEIGHBOURS) {
        int c = -1;
        const int np = nbrpos[tid];
        if (np >= 0 && np < p.T_cap) {
            const int cc = p.comm_of[(size_t)u * p.T_cap + np];
            if (cc >= 0 && cc < p.Cmax) c = cc;
        }
        sc.cand[tid] = c;
    }
    if (tid == 0) sc.tl = p.tail_len[u];
    const T* krow = static_cast<const T*>(p.k) + b * p.sb + kvh * p.sh + lane * E;
    float kx[E];
#pragma unroll
    for (int e = 0; e < E; ++e) kx[e] = to_f32(krow[e]);
    sync();

    // this warp's candidates (-inf when absent or a repeat): rows first
    bool use[PER];
    int ci[PER];
    float row[PER][E];
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        const int i = warp + r * NW;
        ci[r] = sc.cand[i];
        use[r] = ci[r] >= 0;
        for (int j = 0; j < i; ++j) use[r] = use[r] && sc.cand[j] != ci[r];
        const float* cr = p.cent + ((size_t)u * p.Cmax + max(ci[r], 0)) * D + lane * E;
        if (use[r]) {
            if constexpr (E == 4) {
                const float4 v = *reinterpret_cast<const float4*>(cr);
                row[r][0] = v.x; row[r][1] = v.y; row[r][2] = v.z; row[r][3] = v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2*>(cr);
                row[r][0] = v.x; row[r][1] = v.y;
            }
            if (lane == 0) sc.cnt[i] = p.cnt[(size_t)u * p.Cmax + ci[r]];
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) row[r][e] = 0.f;
        }
    }
#pragma unroll
    for (int r = 0; r < PER; ++r) {
        const int i = warp + r * NW;
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            sc.row[i][lane * E + e] = row[r][e];
            a = fmaf(kx[e], row[r][e], a);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
        if (lane == 0) sc.score[i] = use[r] ? a * p.inv_sqrt_d : -INFINITY;
    }
    sync();
    if (warp != 0) return;  // warp 0 picks the winner and updates its row
    // Lane i < 8 holds slot i.  Each distinct candidate carries its score at
    // its first slot; the winner is the largest (votes, score, -id), votes
    // (the slots naming the community) counting only under the vote rule:
    // one 64-bit key per lane, reduced over the warp.  The slot rides in the
    // low bits below the id, which is unique among the keys.
    unsigned long long key = 0ull;  // 0: no candidate
    if (lane < CKV_NEIGHBOURS) {
        const int c = sc.cand[lane];
        const float s = sc.score[lane];
        const unsigned same = __match_any_sync(0xffu, c);  // lanes 0..7 naming the same community
        if (c >= 0 && s != -INFINITY) {
            const unsigned v = p.vote ? (unsigned)__popc(same) : 0u;
            unsigned bits = __float_as_uint(s + 0.0f);  // -0 ranks as +0
            bits = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
            key = ((unsigned long long)v << 60) | ((unsigned long long)bits << 16) |
                  ((unsigned long long)(MAX_CMAX - 1 - c) << 3) | (unsigned long long)lane;
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const unsigned long long k2 = __shfl_xor_sync(FULL, key, o);
        key = k2 > key ? k2 : key;
    }
    int best = key ? MAX_CMAX - 1 - (int)((key >> 3) & 0x1fffu) : -1;
    const int bi = (int)(key & 7u);
    const int tl = sc.tl;
    if (best >= 0 && tl >= p.max_tail) {
        if (lane == 0) atomicOr(p.dev_err, CKV_DEVERR_TAIL_FULL);
        best = -1;
    }
    if (best >= 0 && tl < 0) {  // a corrupted tail length: never written through
        if (lane == 0 && kDebugChecks) atomicOr(p.dev_err, CKV_DEVERR_INDEX);
        best = -1;
    }
    const int n = best >= 0 ? sc.cnt[bi] : 0;  // written by the candidate's warp above
    if (lane == 0) {
        int32_t* cpos = p.comm_of + (size_t)u * p.T_cap + p.pos;
        if (best < 0) {
            *cpos = -1;
            if (p.assigned) p.assigned[u] = -1;
        } else {
            p.cnt[(size_t)u * p.Cmax + best] = n + 1;
            *cpos = best;
            p.tail_tok[(size_t)u * p.max_tail + tl] = p.pos;
            p.tail_comm[(size_t)u * p.max_tail + tl] = best;
            p.tail_len[u] = tl + 1;
            if (p.assigned) p.assigned[u] = best;
        }
    }
    if (best < 0) return;
    // running mean: c <- c + (k - c) / (n + 1) (as (k - c) * (1/(n + 1)) + c,
    // one rounding more than a division), from the copy of the centre
    // taken while scoring
    const size_t rowi = (size_t)u * p.Cmax + best;
    float* cr = p.cent + rowi * D + lane * E;
    const float* c0r = sc.row[bi] + lane * E;
    const float inv_n1 = __frcp_rn((float)(n + 1));  // one reciprocal, then products
    float c1[E], amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float c0 = c0r[e];
        c1[e] = fmaf(kx[e] - c0, inv_n1, c0);
        cr[e] = c1[e];
        amax = fmaxf(amax, fabsf(c1[e]));
    }
    // the int8 scoring copy follows the centre: new scale, new codes
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
    const float scl = q8_scale(amax), rc = q8_recip(amax);
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) packed |= (uint32_t)(q8_code(c1[e], rc) & 0xff) << (8 * e);
    int8_t* qr = p.cent_q + rowi * D + lane * E;
    if constexpr (E == 4) *reinterpret_cast<uint32_t*>(qr) = packed;
    else *reinterpret_cast<uint16_t*>(qr) = (uint16_t)packed;
    if (lane == 0) p.cent_qs[rowi] = scl;
}

}  // namespace ckv
