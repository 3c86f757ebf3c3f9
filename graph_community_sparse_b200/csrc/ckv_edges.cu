// The prefill token graph for sm_100a: direct and co-attention edges.
//
// CommunityKV builds its graph during the prefill pass from the attention
// scores the model computes anyway: nodes are tokens, a query that pays a key
// much attention links the two (direct edges), keys that are attended
// together are linked too (co-attention edges), and the first tokens, which
// attract attention whatever their meaning, are kept out of the graph
// (rit.work summary, section "A graph of tokens replaces re-clustering",
// paragraph 3).  The partition of this graph (Leiden) is not computed here.
//
// Reading used (the pages give no thresholds): the direct edges of query i
// are the 8 key positions j in [S, i) with the largest graph logit
// lambda_ij = max over the graph's query heads of q_{h,i} . k_j / sqrt(d),
// ties to the lower position -- the rule of the decode-time neighbours; the
// co-attention edges are the key pairs j < l found together in one query's
// direct edges, weighted by the number of such queries.
//
//  edges_direct_kernel: the causal Q K^T of every graph unit on the tensor
//    cores (mma.sync m16n8k16, bf16 in, fp32 accumulate), a dense
//    contraction: a warp's 16 A rows are 16/GQ queries x the GQ heads of the
//    graph, placed so that an accumulator thread's two rows (g, g + 8) are
//    two heads of one query: the max over heads is one comparison in the
//    thread plus a shuffle per further pair.  With several heads a warp
//    holds two such 16-row tiles, so each K fragment feeds two products.  The block's 4 warps share
//    32-key K tiles staged by cp.async into padded rows and read as B
//    fragments by ldmatrix.  Each lane keeps a running top-8 (logit,
//    position) list for its share of its query's keys; after every tile the
//    lists of a query share the largest of their 8th logits as a pruning
//    cut (a lower bound of the query's 8th best); insertions run in a
//    warp-uniform branch taken only when some lane has one, so most tiles
//    cost the products, the max and one comparison per value.  At the end the lists of each query are merged
//    by the lanes that share it, pairwise over shuffles.
//  edges_pairs_kernel: one thread per query adds the 28 pairs of its list to
//    the unit's open-addressing hash table (64-bit keys, integer counts by
//    atomics: the multiset is exact whatever the order).
//  edges_compact_kernel: the occupied slots become the unit's (src, dst,
//    weight) list (unordered), warp-aggregated appends.
#include <math.h>
#include <type_traits>

#include "ckv_internal.cuh"

namespace ckv {

constexpr int ED_WARPS = 4;
constexpr int ED_KT = 32;                 // keys per K tile
constexpr int ED_RT = 2;                  // 16-row A tiles per warp (several heads per graph)
constexpr unsigned long long ED_EMPTY = ~0ull;

struct EdgesParams {
    const __nv_bfloat16* k;     // cache K
    int64_t sb, sh, st;
    const __nv_bfloat16* q;     // prefill queries [B, Hq, T, d]
    int B, Hq, Hkv, G, per_head, S, T, T_cap;
    float inv_sqrt_d;
    int32_t* nbr;               // [U, T, 8]
    float* lam;                 // [U, T, 8] or NULL
    unsigned long long* hkey;   // [U, hcap]
    int32_t* hcnt;              // [U, hcap]
    int hcap_log2;
    int32_t* co_src;
    int32_t* co_dst;
    int32_t* co_w;
    int32_t* co_n;              // [U]
    int pair_cap;
    int32_t* dev_err;
};

// Order-preserving key of (logit, position): larger is better, equal logits
// rank the lower position first; 0 is below every real key.
__device__ __forceinline__ unsigned long long edge_key(float lam, int pos) {
    unsigned b = __float_as_uint(lam + 0.0f);  // -0 ranks as +0
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)b << 32) | (unsigned)(0x7fffffff - pos);
}
__device__ __forceinline__ int edge_pos(unsigned long long k) { return 0x7fffffff - (int)(unsigned)(k & 0xffffffffu); }
__device__ __forceinline__ float edge_lam(unsigned long long k) {
    unsigned b = (unsigned)(k >> 32);
    b = (b & 0x80000000u) ? (b & 0x7fffffffu) : ~b;
    return __uint_as_float(b);
}

// Keep `list` (8 keys, best first) the 8 best of itself and `key`.
__device__ __forceinline__ void top8_insert(unsigned long long (&list)[8], unsigned long long key) {
    if (key <= list[7]) return;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const bool gt = key > list[s];
        const unsigned long long cur = list[s];
        list[s] = gt ? key : cur;
        key = gt ? cur : key;
    }
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
struct EdGeom {
    static constexpr int KS = D / 16;        // k-steps
    static constexpr int ROW = D * 2 + 16;   // padded bytes per staged key row (conflict-free 32-bit reads)
    static constexpr int TILE = ED_KT * ROW;
    static constexpr int CH = D / 8;         // 16-byte chunks per row
};

// ldmatrix of four 8x8 b16 matrices (the B fragments of two k-steps)
__device__ __forceinline__ void ed_ldsm_x4(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// A running top-8 list with the logit of its 8th entry (-inf while it is not
// full): a logit below it cannot enter, so most values cost one comparison.
struct Top8 {
    unsigned long long key[8];
    float th;   // this list's 8th logit
    float cut;  // a logit below which no key can be in the query's top 8:
                // the largest 8th logit among the lists sharing the query
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int s = 0; s < 8; ++s) key[s] = 0ull;
        th = cut = -INFINITY;
    }
    // may (lam, pos) enter?  (a logit equal to the cut needs the key)
    __device__ __forceinline__ bool wants(float lam) const { return lam >= cut; }
    __device__ __forceinline__ void insert(float lam, int pos) {
        top8_insert(key, edge_key(lam, pos));
        th = key[7] ? edge_lam(key[7]) : -INFINITY;
        cut = fmaxf(cut, th);
    }
};

// Rows of the A operand: with one head per graph the 16 rows are 16
// queries; otherwise rows g and g + 8 (the two rows of one accumulator
// thread) are two heads of one query, so the max over heads starts inside
// the thread, and the GQ / 2 row pairs of a query sit in lanes that differ in
// lane bits 2 .. LG.
template <int GQ>
struct EdRows {
    static constexpr int LG = GQ == 1 ? 0 : GQ == 2 ? 1 : GQ == 4 ? 2 : 3;
    static constexpr int RT = GQ == 1 ? 1 : ED_RT;      // A row tiles per warp
    static constexpr int QPW0 = 16 / GQ;                // queries per row tile
    static constexpr int QPW = RT * QPW0;               // queries per warp
    static constexpr int NSH = GQ == 1 ? 1 : GQ / 2;    // lanes sharing a query's columns
    static constexpr int MLEN = GQ == 1 ? 32 : 16 * GQ; // list entries merged per query
    __device__ static int query(int r) { return GQ == 1 ? r : (r & 7) >> (LG - 1); }
    __device__ static int head(int r) { return GQ == 1 ? 0 : (((r & 7) & (NSH - 1)) << 1) | (r >> 3); }
};

template <int D, int GQ>
__global__ void __launch_bounds__(ED_WARPS * 32) edges_direct_kernel(const __grid_constant__ EdgesParams p) {
    using EG = EdGeom<D>;
    using ER = EdRows<GQ>;
    constexpr int QPW = ER::QPW;
    constexpr int QB = ED_WARPS * QPW;       // queries per block
    constexpr int LG = ER::LG, NSH = ER::NSH;
    // the two K tiles, and after the last tile the lists to merge
    constexpr int SK_BYTES = 2 * EG::TILE;
    constexpr int SM_BYTES = ED_WARPS * QPW * ER::MLEN * 8;
    __shared__ __align__(16) unsigned char s_raw[SK_BYTES > SM_BYTES ? SK_BYTES : SM_BYTES];
    unsigned char (*s_k)[EG::TILE] = reinterpret_cast<unsigned char (*)[EG::TILE]>(s_raw);
    unsigned long long (*s_m)[QPW][ER::MLEN] = reinterpret_cast<unsigned long long (*)[QPW][ER::MLEN]>(s_raw);
    pdl_wait();
    const int u = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int b = u / p.G, gg = u - b * p.G;
    const int gq = p.Hq / p.Hkv;
    const int kvh = p.per_head ? gg / gq : gg;
    const int h0 = p.per_head ? gg : gg * GQ;
    const int i_blk = p.S + blockIdx.x * QB;               // the block's first query position
    const int i_w = i_blk + warp * QPW;                    // the warp's first query position
    const int j_end = min(i_blk + QB, p.T) - 1;            // keys [S, j_end) reach the block's last query

    // rows of the sinks' outputs: -1 (block 0 of each unit)
    if (blockIdx.x == 0)
        for (int x = tid; x < p.S * 8; x += blockDim.x) {
            p.nbr[((size_t)u * p.T) * 8 + x] = -1;
            if (p.lam) p.lam[((size_t)u * p.T) * 8 + x] = -INFINITY;
        }

    // A fragments of rows g and g + 8 of each row tile (row tile t holds the
    // warp's queries t QPW0 ..)
    constexpr int RT = ER::RT;
    uint32_t a[RT][EG::KS][4];
#pragma unroll
    for (int t = 0; t < RT; ++t) {
        auto qrow = [&](int r) -> const __nv_bfloat16* {
            const int i = i_w + t * ER::QPW0 + ER::query(r);
            return i < p.T ? p.q + (((size_t)b * p.Hq + h0 + ER::head(r)) * p.T + i) * D : nullptr;
        };
        const __nv_bfloat16* r0 = qrow(g);
        const __nv_bfloat16* r1 = qrow(g + 8);
#pragma unroll
        for (int kk = 0; kk < EG::KS; ++kk) {
            const int c0 = 16 * kk + 2 * tq;
            a[t][kk][0] = r0 ? *reinterpret_cast<const uint32_t*>(r0 + c0) : 0u;
            a[t][kk][1] = r1 ? *reinterpret_cast<const uint32_t*>(r1 + c0) : 0u;
            a[t][kk][2] = r0 ? *reinterpret_cast<const uint32_t*>(r0 + c0 + 8) : 0u;
            a[t][kk][3] = r1 ? *reinterpret_cast<const uint32_t*>(r1 + c0 + 8) : 0u;
        }
    }
    // the lane's lists: one head per graph, queries g (la) and g + 8 (lb);
    // otherwise query g >> (LG - 1) of each row tile (la, and lb for the
    // second), whose keys this lane's sub-index among the NSH lanes sharing
    // them takes a share of
    const int qa = ER::query(g), qb = RT == 2 ? qa + ER::QPW0 : ER::query(g + 8);
    const int ia = i_w + qa, ib = i_w + qb;
    const int sub = g & (NSH - 1);
    Top8 la, lb;
    la.init();
    lb.init();

    const __nv_bfloat16* Kb = p.k + b * p.sb + kvh * p.sh;
    // this thread's 16-byte chunks of a K tile: rows r0 + i RSTEP, chunk c0
    constexpr int NCHT = ED_KT * EG::CH / (ED_WARPS * 32);  // chunks per thread
    constexpr int RSTEP = ED_WARPS * 32 / EG::CH;
    static_assert(NCHT * ED_WARPS * 32 == ED_KT * EG::CH, "whole chunks per thread");
    const int r0 = tid / EG::CH, c0 = tid % EG::CH;
    const __nv_bfloat16* kc = Kb + c0 * 8;
    auto stage = [&](int buf, int j0) {
#pragma unroll
        for (int i = 0; i < NCHT; ++i) {
            const int j = j0 + r0 + i * RSTEP;
            const bool ok = j < j_end;
            cp_async_16(s_k[buf] + (r0 + i * RSTEP) * EG::ROW + c0 * 16, kc + (int64_t)(ok ? j : p.S) * p.st, ok);
        }
        cp_async_commit();
    };
    // ldmatrix lane address inside a tile: matrix lane >> 3 is (k-step 2 kp +
    // (lane >> 4), dims half (lane >> 3) & 1) of key row lane & 7
    const int lm_off = (lane & 7) * EG::ROW + (lane >> 3) * 16;
    constexpr int NT = ED_KT / 8;  // n-tiles of 8 keys per K tile
    // a tile's logits into the lists (MASK: test each key against the query)
    auto epilogue = [&](float (&c)[NT][4], int j0, auto mask_tag, Top8& L, const int iq) {
        constexpr bool MASK = decltype(mask_tag)::value;
        if constexpr (GQ == 1) {
            // rows g and g + 8 are queries qa and qb: keys j0 + 8n + 2tq + e;
            // the insertions run only when some lane has one (a warp-uniform
            // branch: most tiles have none)
            float va[NT][2], vb[NT][2];
            bool any = false;
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int j = j0 + 8 * n + 2 * tq + e;
                    va[n][e] = c[n][e] * p.inv_sqrt_d;
                    vb[n][e] = c[n][e + 2] * p.inv_sqrt_d;
                    any |= ((!MASK || j < ia) && la.wants(va[n][e])) || ((!MASK || j < ib) && lb.wants(vb[n][e]));
                }
            if (__any_sync(FULL, any)) {
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = j0 + 8 * n + 2 * tq + e;
                        if ((!MASK || j < ia) && la.wants(va[n][e])) la.insert(va[n][e], j);
                        if ((!MASK || j < ib) && lb.wants(vb[n][e])) lb.insert(vb[n][e], j);
                    }
            }
        } else if constexpr (NSH == 2) {
            // four heads: the two lanes holding a query's columns split them,
            // this lane keeping column e = sub of each n-tile; each lane maxes
            // its two rows (two heads) for both columns and sends its partner
            // the column the partner keeps
            float v[NT];
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float x0 = fmaxf(c[n][0], c[n][2]), x1 = fmaxf(c[n][1], c[n][3]);
                const float keep = sub ? x1 : x0, give = sub ? x0 : x1;
                v[n] = fmaxf(keep, __shfl_xor_sync(FULL, give, 4)) * p.inv_sqrt_d;
            }
            bool any = false;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int j = j0 + 8 * n + 2 * tq + sub;
                any |= (!MASK || j < iq) && L.wants(v[n]);
            }
            if (__any_sync(FULL, any)) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int j = j0 + 8 * n + 2 * tq + sub;
                    if ((!MASK || j < iq) && L.wants(v[n])) L.insert(v[n], j);
                }
            }
        } else {
            // max over the query's heads: its two rows here, then the NSH
            // lanes holding its other row pairs
            float v[NT][2];
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float x = fmaxf(c[n][e], c[n][e + 2]);
#pragma unroll
                    for (int o = 4; o < (4 << (LG - 1)); o <<= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
                    v[n][e] = x * p.inv_sqrt_d;
                }
            // this lane's share of the query's 2 NT keys here: value 2n + e
            // belongs to the lane whose sub-index is its remainder modulo NSH;
            // the insertions run only when some lane has one
            bool any = false;
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool mine = ((2 * n + e) & (NSH - 1)) == sub;
                    const int j = j0 + 8 * n + 2 * tq + e;
                    any |= mine && (!MASK || j < iq) && L.wants(v[n][e]);
                }
            if (__any_sync(FULL, any)) {
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool mine = ((2 * n + e) & (NSH - 1)) == sub;
                        const int j = j0 + 8 * n + 2 * tq + e;
                        if (mine && (!MASK || j < iq) && L.wants(v[n][e])) L.insert(v[n][e], j);
                    }
            }
        }
    };
    const int ntile = j_end > p.S ? (j_end - p.S + ED_KT - 1) / ED_KT : 0;
    if (ntile > 0) stage(0, p.S);
    for (int t = 0; t < ntile; ++t) {
        const int j0 = p.S + t * ED_KT;
        if (t + 1 < ntile) stage((t + 1) & 1, j0 + ED_KT);
        else cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const unsigned kbase = static_cast<unsigned>(__cvta_generic_to_shared(s_k[t & 1]));
        float c[RT][NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
            for (int t = 0; t < RT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) c[t][n][e] = 0.f;
#pragma unroll
            for (int kp = 0; kp < EG::KS / 2; ++kp) {
                uint32_t b0, b1, b2, b3;
                ed_ldsm_x4(kbase + 8 * n * EG::ROW + lm_off + kp * 64, b0, b1, b2, b3);
#pragma unroll
                for (int t = 0; t < RT; ++t) {
                    mma_bf16(c[t][n], a[t][2 * kp], b0, b1);
                    mma_bf16(c[t][n], a[t][2 * kp + 1], b2, b3);
                }
            }
        }
        // keys of this tile all below the warp's first query: no causal test
        if (j0 + ED_KT <= i_w) {
            epilogue(c[0], j0, std::false_type{}, la, ia);
            if constexpr (RT == 2) epilogue(c[1], j0, std::false_type{}, lb, ib);
        } else {
            epilogue(c[0], j0, std::true_type{}, la, ia);
            if constexpr (RT == 2) epilogue(c[1], j0, std::true_type{}, lb, ib);
        }
        // a query's lists are spread over its 4 column lanes (lane bits 0-1)
        // and, with several heads, its NSH row-pair lanes (bits 2 ..): a list
        // holds 8 keys at or above its 8th logit, so the largest such logit
        // among them bounds the query's 8th best from below and prunes all
        // of them (a list of its own sees only a share of the keys and would
        // admit many more)
        {
            float ca = la.th, cb = lb.th;
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                ca = fmaxf(ca, __shfl_xor_sync(FULL, ca, o));
                if constexpr (GQ == 1) cb = fmaxf(cb, __shfl_xor_sync(FULL, cb, o));
            }
            if constexpr (GQ > 1) {
                if constexpr (RT == 2) {
#pragma unroll
                    for (int o = 1; o < 4; o <<= 1) cb = fmaxf(cb, __shfl_xor_sync(FULL, cb, o));
                }
#pragma unroll
                for (int o = 4; o < 4 * NSH; o <<= 1) {
                    ca = fmaxf(ca, __shfl_xor_sync(FULL, ca, o));
                    if constexpr (RT == 2) cb = fmaxf(cb, __shfl_xor_sync(FULL, cb, o));
                }
            }
            la.cut = fmaxf(la.cut, ca);
            if constexpr (GQ == 1 || RT == 2) lb.cut = fmaxf(lb.cut, cb);
        }
        __syncthreads();  // the tile is read by every warp before it is refilled
    }
    cp_async_wait<0>();
    __syncthreads();  // no warp reads a K tile any more: the lists take its space

    // merge each query's lists (its 4 column lanes x NSH row-pair lanes)
    if constexpr (GQ == 1) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            s_m[warp][qa][tq * 8 + s] = la.key[s];
            s_m[warp][qb][tq * 8 + s] = lb.key[s];
        }
    } else {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            s_m[warp][qa][(tq * NSH + sub) * 8 + s] = la.key[s];
            if constexpr (RT == 2) s_m[warp][qb][(tq * NSH + sub) * 8 + s] = lb.key[s];
        }
    }
    __syncwarp();
    // a query's MLEN / 8 sorted lists, merged by LPQ = 32 / QPW lanes: lane
    // (query lane / LPQ, part lane % LPQ) takes its part's lists in turn, then
    // the parts merge pairwise over shuffles (the best 8 of two sorted lists
    // of 8: the pairwise larger of one list and the other reversed is
    // bitonic, and a 12-exchange network sorts it)
    constexpr int LPQ = 32 / QPW;              // lanes per query
    constexpr int LPL = ER::MLEN / 8 / LPQ;    // lists per lane
    static_assert(LPL >= 1 && LPL * LPQ * 8 == ER::MLEN, "whole lists per lane");
    const int mq = lane / LPQ, mp = lane % LPQ;
    unsigned long long best[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) best[s] = s_m[warp][mq][mp * LPL * 8 + s];
#pragma unroll
    for (int l = 1; l < LPL; ++l)
#pragma unroll
        for (int s = 0; s < 8; ++s) top8_insert(best, s_m[warp][mq][(mp * LPL + l) * 8 + s]);
#pragma unroll
    for (int o = 1; o < LPQ; o <<= 1) {
        unsigned long long other[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) other[s] = __shfl_xor_sync(FULL, best[s], o);
#pragma unroll
        for (int s = 0; s < 8; ++s) best[s] = best[s] > other[7 - s] ? best[s] : other[7 - s];
        // bitonic (rising then falling, or the reverse): sort descending
#pragma unroll
        for (int h = 4; h >= 1; h >>= 1)
#pragma unroll
            for (int s = 0; s < 8; ++s)
                if ((s & h) == 0) {
                    const unsigned long long x = best[s], y = best[s + h];
                    best[s] = x > y ? x : y;
                    best[s + h] = x > y ? y : x;
                }
    }
    if (mp == 0) {
        const int i = i_w + mq;
        if (i < p.T) {
            int32_t* on = p.nbr + ((size_t)u * p.T + i) * 8;
            float* ol = p.lam ? p.lam + ((size_t)u * p.T + i) * 8 : nullptr;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                on[s] = best[s] ? edge_pos(best[s]) : -1;
                if (ol) ol[s] = best[s] ? edge_lam(best[s]) : -INFINITY;
            }
        }
    }
}

__global__ void edges_clear_kernel(EdgesParams p) {
    pdl_wait();
    const size_t n = (size_t)p.B * p.G << p.hcap_log2;
    for (size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (size_t)gridDim.x * blockDim.x) {
        p.hkey[x] = ED_EMPTY;
        p.hcnt[x] = 0;
    }
    for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < p.B * p.G; x += gridDim.x * blockDim.x) p.co_n[x] = 0;
}

// The pairs of query i's list, ascending by position, into unit u's table.
__global__ void __launch_bounds__(256) edges_pairs_kernel(EdgesParams p) {
    pdl_wait();
    const int u = blockIdx.y;
    const int i = p.S + blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= p.T) return;
    const int32_t* in = p.nbr + ((size_t)u * p.T + i) * 8;
    int v[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) v[s] = in[s];
    // ascending by position, -1 (no entry) last
#pragma unroll
    for (int x = 1; x < 8; ++x)
#pragma unroll
        for (int y = x; y > 0; --y) {
            const unsigned a = (unsigned)v[y - 1], c = (unsigned)v[y];  // -1 is the largest unsigned
            const bool sw = c < a;
            v[y - 1] = sw ? (int)c : (int)a;
            v[y] = sw ? (int)a : (int)c;
        }
    const unsigned mask = (1u << p.hcap_log2) - 1u;
    unsigned long long* tk = p.hkey + ((size_t)u << p.hcap_log2);
    int32_t* tc = p.hcnt + ((size_t)u << p.hcap_log2);
    for (int x = 0; x < 8; ++x) {
        if (v[x] < 0) break;
        for (int y = x + 1; y < 8; ++y) {
            if (v[y] < 0) break;
            const unsigned long long key = ((unsigned long long)(unsigned)v[x] << 32) | (unsigned)v[y];
            unsigned h = (unsigned)((key * 0x9E3779B97F4A7C15ull) >> 32) & mask;
            // linear probing; the table is at most half full, so the probe
            // ends long before it could wrap around
            for (unsigned probe = 0; probe <= mask; ++probe) {
                const unsigned long long old = atomicCAS(tk + h, ED_EMPTY, key);
                if (old == ED_EMPTY || old == key) {
                    atomicAdd(tc + h, 1);
                    break;
                }
                h = (h + 1) & mask;
            }
        }
    }
}

// Occupied slots of unit blockIdx.y's table become its (src, dst, weight)
// list, a warp-aggregated append per 32 slots.
__global__ void __launch_bounds__(256) edges_compact_kernel(EdgesParams p) {
    pdl_wait();
    const int u = blockIdx.y, lane = threadIdx.x & 31;
    const int n = 1 << p.hcap_log2;
    const unsigned long long* tk = p.hkey + ((size_t)u << p.hcap_log2);
    const int32_t* tc = p.hcnt + ((size_t)u << p.hcap_log2);
    bool over = false;
    for (int base = blockIdx.x * blockDim.x; base < n; base += gridDim.x * blockDim.x) {
        const int x = base + threadIdx.x;
        unsigned long long key = ED_EMPTY;
        if (x < n) key = tk[x];
        const bool occ = key != ED_EMPTY;
        const unsigned m = __ballot_sync(FULL, occ);
        int first = 0;
        if (lane == 0 && m) first = atomicAdd(p.co_n + u, __popc(m));
        first = __shfl_sync(FULL, first, 0);
        if (occ) {
            const int at = first + __popc(m & ((1u << lane) - 1u));
            if (at < p.pair_cap) {
                const size_t o = (size_t)u * p.pair_cap + at;
                p.co_src[o] = (int32_t)(key >> 32);
                p.co_dst[o] = (int32_t)(key & 0xffffffffu);
                p.co_w[o] = tc[x];
            } else {
                over = true;
            }
        }
    }
    if (over) atomicOr(p.dev_err, CKV_DEVERR_EDGE_CAP);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

int edges_hcap_log2(int T, int S) {
    // 28 pairs per query at most; the table keeps the load factor <= 1/2
    const long long need = 2LL * 28 * (long long)(T - S > 0 ? T - S : 1);
    int l = 6;
    while ((1LL << l) < need) ++l;
    return l;
}

size_t edges_ws_bytes(int U, int T, int S) {
    const size_t cap = (size_t)1 << edges_hcap_log2(T, S);
    return align256((size_t)U * cap * 8) + align256((size_t)U * cap * 4);
}

namespace {
template <int D, int GQ>
cudaError_t launch_direct(const EdgesParams& p, cudaStream_t st) {
    constexpr int QB = ED_WARPS * EdRows<GQ>::QPW;
    const dim3 grid((p.T - p.S + QB - 1) / QB > 0 ? (p.T - p.S + QB - 1) / QB : 1, p.B * p.G);
    return launch_pdl(KK_EDGES, edges_direct_kernel<D, GQ>, grid, dim3(ED_WARPS * 32), 0, st, p);
}
}  // namespace

cudaError_t launch_build_edges(const CacheView& c, int mode, int S, const void* q, int T, int32_t* nbr, float* lam,
                               int32_t* co_src, int32_t* co_dst, int32_t* co_w, int32_t* co_n, int pair_cap,
                               int32_t* dev_err, void* ws, cudaStream_t st) {
    EdgesParams p{};
    p.k = static_cast<const __nv_bfloat16*>(c.k);
    p.sb = c.sb;
    p.sh = c.sh;
    p.st = c.st;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.B = c.B;
    p.Hq = c.Hq;
    p.Hkv = c.Hkv;
    p.per_head = mode == CKV_GRAPH_PER_HEAD;
    p.G = p.per_head ? c.Hq : c.Hkv;
    p.S = S;
    p.T = T;
    p.T_cap = c.T_cap;
    p.inv_sqrt_d = 1.0f / sqrtf((float)c.d);
    p.nbr = nbr;
    p.lam = lam;
    p.hcap_log2 = edges_hcap_log2(T, S);
    const int U = c.B * p.G;
    const size_t cap = (size_t)1 << p.hcap_log2;
    p.hkey = reinterpret_cast<unsigned long long*>(ws);
    p.hcnt = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align256((size_t)U * cap * 8));
    p.co_src = co_src;
    p.co_dst = co_dst;
    p.co_w = co_w;
    p.co_n = co_n;
    p.pair_cap = pair_cap;
    p.dev_err = dev_err;
    const int gq = p.per_head ? 1 : c.Hq / c.Hkv;

    cudaError_t e = launch_pdl(KK_EDGES, edges_clear_kernel, dim3(296), dim3(256), 0, st, p);
    if (e != cudaSuccess) return e;
#define CKV_ED_CASE(DD, GG) \
    if (c.d == DD && gq == GG) e = launch_direct<DD, GG>(p, st); else
    CKV_ED_CASE(128, 1) CKV_ED_CASE(128, 2) CKV_ED_CASE(128, 4) CKV_ED_CASE(128, 8)
    CKV_ED_CASE(64, 1) CKV_ED_CASE(64, 2) CKV_ED_CASE(64, 4) CKV_ED_CASE(64, 8)
    e = cudaErrorInvalidValue;
#undef CKV_ED_CASE
    if (e != cudaSuccess) return e;
    if (T > S) {
        const dim3 pg((T - S + 255) / 256, U);
        e = launch_pdl(KK_EDGES, edges_pairs_kernel, pg, dim3(256), 0, st, p);
        if (e != cudaSuccess) return e;
    }
    const int nchunk = (int)((cap + 255) / 256);
    const dim3 cg(nchunk < 64 ? nchunk : 64, U);
    return launch_pdl(KK_EDGES, edges_compact_kernel, cg, dim3(256), 0, st, p);
}

}  // namespace ckv
