// Indexed sparse decode attention (and the dense comparator) for sm_100a.
//
// CommunityKV runs exact softmax attention over the selected communities
// plus the sink tokens, read straight from the whole cache ("CommunityKV:
// Efficient Long-Context Decoding via Graph Partitioning", rit.work summary,
// section "A graph of tokens replaces re-clustering", paragraphs 4-5).  This
// is a matrix-vector product over gathered rows: bandwidth-bound, so it runs
// on the CUDA cores, not the tensor cores.
//
// Work split (stream-K over warps): the selected tokens of all graph units
// are laid end to end (selection.unit_prefix); warp w of W takes the slice
// [w*per, (w+1)*per) with per = ceil(total/W), whatever units it crosses, so
// every warp reads the same number of K/V rows regardless of how skewed the
// community sizes are.  A warp writes one partial (running max m, sum l,
// unnormalised accumulator) per unit segment into slot w + u, and, when
// neighbours are wanted, each list entry's graph logit;
// which is unique because slices and units are both contiguous and ordered.
// All warps of the persistent grid finish together, so the merge of each
// unit's slots is a second, small kernel launched as a programmatic
// dependent: its launch overlaps the attention kernel's tail and it waits
// (in hardware, griddepcontrol) for that kernel's results; every operand is
// fetched in one round of independent loads.
//
// Inside a warp: each half-warp owns one token row at a time, a lane owns
// D/16 consecutive elements (16 bytes for bf16, d = 128); K and V rows of
// 8 tokens per iteration are staged by cp.async into a per-warp ring of
// Stages<GQ> iterations (2 for one head per graph, where more resident warps
// matter more, 3 otherwise), so loads stay in flight while one is computed.
// Logits of the GQA group's heads are reduced with a value-exchanging
// butterfly; the softmax uses exp2 with log2(e)/sqrt(d) folded into q and a
// lazily raised running max (raised only when a logit exceeds it by more
// than 2^8), which is exact after the final division.
#include <math.h>
#include <type_traits>

#include "ckv_assign.cuh"
#include "ckv_internal.cuh"

namespace ckv {

constexpr int DEC_WARPS = 4;
// Work split of the attention kernel: the first 7/8 of the concatenated token
// lists are cut into one equal slice per warp; the last 1/8 is handed out in
// chunks of at least DYN_CHUNK_MIN tokens (at most NCH_MAX chunks) from an
// atomic ticket, so warps on SMs that run faster (the SMs of a GPC share its
// memory bandwidth unevenly) take more of it and all warps end together.
constexpr int DYN_DEN = 8;
constexpr int MIN_WARP_TOKENS = 64;
constexpr int DYN_CHUNK_MIN = 64;
constexpr int NCH_MAX = 4096;

struct DynSplit {
    int R;      // tokens of the static part, [0, R)
    int per_s;  // static tokens per warp
    int chk;    // dynamic chunk length
    int nch;    // dynamic chunks
};

// dense: static slices only (its units are long, so a dynamic tail would
// multiply the partials each merge block combines)
__host__ __device__ __forceinline__ DynSplit dyn_split(int total, int W, bool dense) {
    DynSplit d;
    const int dyn = dense ? 0 : total / DYN_DEN;
    d.chk = max(DYN_CHUNK_MIN, (dyn + NCH_MAX - 1) / NCH_MAX);
    d.nch = (dyn + d.chk - 1) / d.chk;
    d.R = total - dyn;
    // at least MIN_WARP_TOKENS per warp: small problems use fewer warps, so
    // each unit has fewer partials to merge
    d.per_s = max(MIN_WARP_TOKENS, (d.R + W - 1) / W);
    return d;
}
constexpr int TOK_PER_IT = 8;
constexpr float RESCALE_THRESH = 8.0f;

template <int GQ> struct Stages { static constexpr int v = GQ == 1 ? 2 : 3; };
template <int GQ> struct MinBlocks { static constexpr int v = GQ == 1 ? 6 : (GQ == 2 ? 5 : (GQ == 4 ? 4 : 2)); };

template <typename T, int D>
struct RowGeom {
    static constexpr int E = D / 16;
    static constexpr int PART = E * ElemBytes<T>::v;
    static constexpr int ROW = 16 * PART;
    static constexpr int TILE = TOK_PER_IT * ROW;
};

// bf16 caches whose graphs serve several query heads use the tensor-core
// segment loop (ckv_decode_mma.cuh); the others the scalar one below.
template <typename T, int GQ>
struct UseMma {
    static constexpr bool v = std::is_same<T, __nv_bfloat16>::value && GQ >= 2;
};
template <typename T, int GQ>
struct DecMinBlocks {
    static constexpr int v = UseMma<T, GQ>::v ? 2 : MinBlocks<GQ>::v;
};
template <int D>
struct MmaGeom;

template <typename T, int D, int GQ>
struct DecSmem {
    static constexpr int PBUF = TOK_PER_IT * GQ * 4;
    static constexpr int SCALAR = Stages<GQ>::v * 2 * RowGeom<T, D>::TILE + ((PBUF + 127) / 128) * 128;
    static constexpr int MMA = 3 * 2 * 16 * D * 2;  // MMA_STAGES x (K, V) x MMA_TOK rows of bf16
    static constexpr int WARP = UseMma<T, GQ>::v ? MMA : SCALAR;
    static constexpr int CTA_FIXED = DEC_WARPS * WARP;
};

struct DecodeParams {
    const void* k;
    const void* v;
    int64_t sb, sh, st;
    const void* q;
    int Hq, Hkv;
    int U, G, per_head;
    int S;
    const int32_t* sel_tok;
    int tok_cap;
    int32_t* unit_prefix;   // written by block 0 of the attention kernel
    const int32_t* n_tok;
    int T;                  // dense only: tokens per unit
    int T_cap;              // rows per (sequence, KV head): debug checks of positions
    int32_t* dev_err;       // the graph's error word (debug checks; NULL for dense)
    float scale_log2;
    DecodeWs ws;
    int W;                  // warps in the grid
    int want_nbr;
    float* out;
    int32_t* nbr8;          // may be NULL when only the fused update needs them
    int append;             // fused community update (and K/V append) in the merge
    AssignParams ap;
};

__device__ __forceinline__ void unit_heads(const DecodeParams& p, int u, int gq, bool dense,
                                           int& b, int& kvh, int& h0) {
    b = u / p.G;
    const int g = u - b * p.G;
    if (!dense && p.per_head) {
        kvh = g / (p.Hq / p.Hkv);
        h0 = g;
    } else {
        kvh = g;
        h0 = g * gq;
    }
}

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32, relative error
// about 2^-22).  Arguments here are <= 8; results below 2^-126 flush to zero,
// which only drops weights below 1e-38 of the running maximum.
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

#include "ckv_decode_mma.cuh"

// One warp, one unit, list positions [lo, hi) of the unit's selection (or
// cache positions, dense).  Full iterations (all 8 tokens valid, past the
// sinks) take a path without per-token masks; only the last, partial
// iteration and the one holding the sinks test each token.
template <typename T, int D, int GQ, bool DENSE>
__device__ __forceinline__ void process_segment(const DecodeParams& p, int u, int lo, int hi, int slot,
                                                unsigned char* wsm, int lane) {
    using RG = RowGeom<T, D>;
    constexpr int E = RG::E, PART = RG::PART, ROW = RG::ROW, TILE = RG::TILE;
    constexpr int LG = Log2<GQ>::v;
    constexpr int NS = Stages<GQ>::v;
    const int half = lane >> 4, l16 = lane & 15;
    const int hl = head_of_lane<GQ>(lane);
    const bool owner = (lane & ((16 >> LG) - 1)) == 0;
    const int64_t st = p.st;
    const bool want_nbr = !DENSE && p.want_nbr;

    int b, kvh, h0;
    unit_heads(p, u, GQ, DENSE, b, kvh, h0);
    const T* Kb = static_cast<const T*>(p.k) + b * p.sb + kvh * p.sh + l16 * E;
    const T* Vb = static_cast<const T*>(p.v) + b * p.sb + kvh * p.sh + l16 * E;
    const int32_t* toks = DENSE ? nullptr : p.sel_tok + (size_t)u * p.tok_cap;

    float qr[GQ][E];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        load_row_part<T, E>(static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h0 + h) * D + l16 * E, qr[h]);
#pragma unroll
        for (int e = 0; e < E; ++e) qr[h][e] *= p.scale_log2;
    }

    const int n = hi - lo;
    const int nit = (n + TOK_PER_IT - 1) / TOK_PER_IT;
    const int nfull = n / TOK_PER_IT;
    float* pbuf = reinterpret_cast<float*>(wsm + NS * 2 * TILE);

    int win_cur = 0, win_nxt = 0;
    if constexpr (!DENSE) {
        win_cur = (lane < n) ? __ldg(toks + lo + lane) : 0;
        win_nxt = (32 + lane < n) ? __ldg(toks + lo + 32 + lane) : 0;
    }

    int stage_in = 0;  // ring slot the next issue fills
    auto issue = [&](int it, auto full_tag) {
        constexpr bool ALL_VALID = decltype(full_tag)::value;
        unsigned char* kt = wsm + stage_in * 2 * TILE;
        stage_in = (stage_in + 1 == NS) ? 0 : stage_in + 1;
        unsigned char* vt = kt + TILE;
        if constexpr (!DENSE) {
            if (it > 0 && (it & 3) == 0) {
                win_cur = win_nxt;
                const int nx = (it + 4) * TOK_PER_IT + lane;
                win_nxt = (nx < n) ? __ldg(toks + lo + nx) : 0;
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = it * TOK_PER_IT + 2 * j + half;
            const bool valid = ALL_VALID || i < n;
            int pos;
            if constexpr (DENSE) {
                pos = lo + i;
            } else {
                pos = __shfl_sync(ckv::FULL, win_cur, ((it & 3) << 3) + 2 * j + half);
                pos = checked_index(pos, 0, p.T_cap, p.dev_err, 0);
            }
            if (!ALL_VALID) pos = valid ? pos : 0;
            const int64_t off = (int64_t)pos * st;
            const int r = 2 * j + half;
            cp_async_part<PART>(kt + r * ROW + l16 * PART, Kb + off, valid);
            cp_async_part<PART>(vt + r * ROW + l16 * PART, Vb + off, valid);
        }
        cp_async_commit();
    };
    auto issue_any = [&](int it) {
        if (it < nfull) issue(it, std::true_type{});
        else if (it < nit) issue(it, std::false_type{});
        else cp_async_commit();
    };

#pragma unroll
    for (int s = 0; s < NS - 1; ++s) issue_any(s);

    float m_run = -INFINITY, l_run = 0.f;
    float acc[GQ][E];
#pragma unroll
    for (int h = 0; h < GQ; ++h)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
    float* lamu = DENSE ? nullptr : p.ws.lam + (size_t)u * p.ws.lam_cap;
    int stage_out = 0;  // ring slot computed next

    auto compute = [&](int it, auto full_tag) {
        constexpr bool ALL_VALID = decltype(full_tag)::value;
        const unsigned char* kt = wsm + stage_out * 2 * TILE;
        const unsigned char* vt = kt + TILE;
        stage_out = (stage_out + 1 == NS) ? 0 : stage_out + 1;

        float s[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float kf[E];
            load_row_part<T, E>(reinterpret_cast<const T*>(kt + (2 * j + half) * ROW + l16 * PART), kf);
            float part[GQ];
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) a = fmaf(qr[h][e], kf[e], a);
                part[h] = a;
            }
            s[j] = halfwarp_reduce_heads<GQ>(part, lane);
            if (!ALL_VALID && it * TOK_PER_IT + 2 * j + half >= n) s[j] = -INFINITY;
        }

        float mx = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
        mx = fmaxf(mx, __shfl_xor_sync(ckv::FULL, mx, 16));
        const bool need = mx > m_run + RESCALE_THRESH;
        if (__any_sync(ckv::FULL, need)) {
            const float m_new = need ? mx : m_run;
            const float f = (m_run == -INFINITY) ? 0.f : exp2_approx(m_run - m_new);
            l_run *= f;
            m_run = m_new;
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                const float fh = __shfl_sync(ckv::FULL, f, (lane & 16) | (h << (4 - LG)));
#pragma unroll
                for (int e = 0; e < E; ++e) acc[h][e] *= fh;
            }
        }

        float pj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) pj[j] = exp2_approx(s[j] - m_run);
        l_run += (pj[0] + pj[1]) + (pj[2] + pj[3]);

        if constexpr (GQ > 1) {
            if (owner) {
#pragma unroll
                for (int j = 0; j < 4; ++j) pbuf[(2 * j + half) * GQ + hl] = pj[j];
            }
            __syncwarp();
        }

#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float ph[GQ];
            if constexpr (GQ == 1) {
                ph[0] = pj[j];
            } else {
#pragma unroll
                for (int h = 0; h < GQ; h += 2) {
                    const float2 t2 = *reinterpret_cast<const float2*>(pbuf + (2 * j + half) * GQ + h);
                    ph[h] = t2.x;
                    ph[h + 1] = t2.y;
                }
            }
            float vf[E];
            load_row_part<T, E>(reinterpret_cast<const T*>(vt + (2 * j + half) * ROW + l16 * PART), vf);
#pragma unroll
            for (int h = 0; h < GQ; ++h)
#pragma unroll
                for (int e = 0; e < E; ++e) acc[h][e] = fmaf(ph[h], vf[e], acc[h][e]);
        }

        if (want_nbr) {
            // graph logit of each token (max over the group's heads) for the
            // neighbour search in the merge kernel
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float lam = halfwarp_max_over_heads<GQ>(s[j]);
                const int i = it * TOK_PER_IT + 2 * j + half;
                if (l16 == 0 && (ALL_VALID || i < n)) lamu[lo + i] = lam;
            }
        }
    };

    for (int it = 0; it < nit; ++it) {
        __syncwarp();
        issue_any(it + NS - 1);
        cp_async_wait<NS - 1>();
        if (it < nfull) compute(it, std::true_type{});
        else compute(it, std::false_type{});
    }
    cp_async_wait<0>();

#pragma unroll
    for (int h = 0; h < GQ; ++h)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] += __shfl_xor_sync(FULL, acc[h][e], 16);
    l_run += __shfl_xor_sync(FULL, l_run, 16);

    const DecodeWs& ws = p.ws;
    if (lane < 16) {
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float* dst = ws.acc + ((size_t)slot * GQ + h) * D + l16 * E;
#pragma unroll
            for (int e = 0; e < E; e += 4)
                *reinterpret_cast<float4*>(dst + e) = make_float4(acc[h][e], acc[h][e + 1], acc[h][e + 2], acc[h][e + 3]);
        }
        if (owner) {
            ws.m[(size_t)slot * GQ + hl] = m_run;
            ws.l[(size_t)slot * GQ + hl] = l_run;
        }
    }
}

template <typename T, int D, int GQ, bool DENSE>
__global__ void __launch_bounds__(DEC_WARPS * 32, DecMinBlocks<T, GQ>::v) decode_main(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    pdl_wait();  // the selection comes from the kernel before
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char* wsm = smem + warp * DecSmem<T, D, GQ>::WARP;
    int* s_pre = reinterpret_cast<int*>(smem + DecSmem<T, D, GQ>::CTA_FIXED);
    const int w = blockIdx.x * DEC_WARPS + warp;

    int total;
    if constexpr (!DENSE) {
        // exclusive prefix of the units' token counts, computed by every block
        // (each thread scans a contiguous chunk); block 0 also publishes it
        __shared__ int s_warp[33];
        const int seg = (p.U + blockDim.x - 1) / blockDim.x;
        const int b0 = min(p.U, (int)threadIdx.x * seg), b1 = min(p.U, b0 + seg);
        int own = 0;
        for (int i = b0; i < b1; ++i) {
            int x = p.n_tok[i];
            if constexpr (kDebugChecks) {
                if (x < 0 || x > p.tok_cap) {
                    atomicOr(p.dev_err, CKV_DEVERR_INDEX);
                    x = max(0, min(x, p.tok_cap));
                }
            }
            s_pre[i] = x;
            own += x;
        }
        int all;
        int run = block_exclusive_scan(own, s_warp, &all);
        for (int i = b0; i < b1; ++i) {
            const int x = s_pre[i];
            s_pre[i] = run;
            run += x;
        }
        if (threadIdx.x == 0) s_pre[p.U] = all;
        __syncthreads();
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i <= p.U; i += blockDim.x) p.unit_prefix[i] = s_pre[i];
        total = s_pre[p.U];
    } else {
        total = p.U * p.T;
    }
    if (total <= 0) return;
    const DynSplit sp = dyn_split(total, p.W, DENSE);

    // tokens [start, end) of the concatenated lists; partial of unit u in
    // slot sbase + u
    auto run_range = [&](int start, int end, int sbase) {
        int u;
        if constexpr (DENSE) {
            u = start / p.T;
        } else {
            int a = 0, c = p.U;  // s_pre[a] <= start < s_pre[c]
            while (c - a > 1) {
                const int mid = (a + c) >> 1;
                if (s_pre[mid] <= start) a = mid;
                else c = mid;
            }
            u = a;
        }
        while (true) {
            const int ubeg = DENSE ? u * p.T : s_pre[u];
            const int uend = DENSE ? ubeg + p.T : s_pre[u + 1];
            const int lo = max(start, ubeg), hi = min(end, uend);
            if (lo < hi) {
                if constexpr (UseMma<T, GQ>::v)
                    process_segment_mma<D, GQ, DENSE>(p, u, lo - ubeg, hi - ubeg, sbase + u, wsm, lane);
                else
                    process_segment<T, D, GQ, DENSE>(p, u, lo - ubeg, hi - ubeg, sbase + u, wsm, lane);
            }
            if (end <= uend || u + 1 >= p.U) break;
            ++u;
        }
    };

    // static slice: slots [0, W + U)
    const int start = w * sp.per_s;
    if (start < sp.R) run_range(start, min(start + sp.per_s, sp.R), w);
    // dynamic chunks: slots [W + U, W + 2U + nch)
    while (true) {
        int c = 0;
        if (lane == 0) c = atomicAdd(p.ws.ticket, 1);
        c = __shfl_sync(FULL, c, 0);
        if (c >= sp.nch) break;
        const int c0 = sp.R + c * sp.chk;
        run_range(c0, min(c0 + sp.chk, total), p.W + p.U + c);
    }
}

// Warps of the merge block that search the neighbours (sparse decode only).
constexpr int NBR_WARPS = 4;
// Spare partial slots after the last one: a merge chunk (<= 32 slots) may
// read past a unit's last slot without leaving the arrays.
constexpr int MERGE_PAD = 32;
constexpr int NBR_THREADS = NBR_WARPS * 32;
constexpr int NBR_KEEP = 16;  // list entries per thread held in registers
constexpr int NBR_CAP = 256;  // candidate slots in shared memory

// Neighbour ranking key: graph logit descending, then position ascending, as
// one unsigned 64-bit number (larger is better; 0 = no entry).  The logit is
// mapped to an order-preserving unsigned integer.
__device__ __forceinline__ unsigned long long nbr_key(float lam, int pos) {
    unsigned b = __float_as_uint(lam + 0.0f);  // -0 ranks as +0
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)b << 32) | (unsigned)(0x7fffffff - pos);
}
__device__ __forceinline__ int nbr_pos(unsigned long long k) {
    return 0x7fffffff - (int)(unsigned)(k & 0xffffffffu);
}

// The fused community update of unit u by the merge block's NBR_WARPS
// neighbour warps (thread xt of 32 NBR_WARPS), given its neighbour positions.
template <typename T, int D>
__device__ __forceinline__ void merge_assign(const DecodeParams& p, int u, const int* nbpos, int xt) {
    __shared__ __align__(16) AssignScratch<D> s_as;
    auto sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(NBR_THREADS) : "memory"); };
    assign_unit<T, D, NBR_WARPS, false>(p.ap, u, nbpos, xt, s_as, sync);
}

// One block per unit: threads 0..D-1 own one output dimension each (all the
// unit's heads); the NBR_WARPS extra warps search the top-8 neighbours.  Slots are
// combined in slot order, a chunk of slots at a time, by a per-thread online
// merge: no shared memory and no barriers, so the merge costs about two
// dependent rounds of loads.
template <typename T, int D, int GQ, bool DENSE>
__global__ void __launch_bounds__(D + (DENSE ? 0 : 32 * NBR_WARPS), 2) decode_merge(const __grid_constant__ DecodeParams p) {
    pdl_wait();  // the attention kernel's partials are complete and visible
    const int u = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    // no kernel of this call takes a ticket any more: return it to zero
    if (u == 0 && t == 0) *p.ws.ticket = 0;
    int b, kvh, h0;
    unit_heads(p, u, GQ, DENSE, b, kvh, h0);
    int ubeg, uend, total;
    if constexpr (DENSE) {
        ubeg = u * p.T;
        uend = ubeg + p.T;
        total = p.U * p.T;
    } else {
        ubeg = p.unit_prefix[u];
        uend = p.unit_prefix[u + 1];
        total = p.unit_prefix[p.U];
    }
    float* outu = p.out + ((size_t)b * p.Hq + h0) * D;
    // the new K/V rows go into the cache first, by the output threads (off
    // the neighbour search and update, which wait on more round trips)
    if (!DENSE && p.append && t < D) append_rows(p.ap, u, t, D);
    if (uend <= ubeg) {
        for (int i = t; i < GQ * D; i += blockDim.x) outu[i] = 0.f;
        if (!DENSE && p.want_nbr && p.nbr8 && t < 8) p.nbr8[(size_t)u * 8 + t] = -1;
        if (!DENSE && p.append && warp >= D / 32) {
            __shared__ int s_none[CKV_NEIGHBOURS];
            if (t - D < CKV_NEIGHBOURS) s_none[t - D] = -1;
            merge_assign<T, D>(p, u, s_none, t - D);  // no neighbour: the token joins nothing
        }
        return;
    }
    // the unit's partials: static slices [sA, sA + nA), then dynamic chunks
    // [sB, sB + nB) (the attention kernel's split, recomputed)
    const DynSplit sp = dyn_split(total, p.W, DENSE);
    int nA = 0, nB = 0;
    size_t sA = 0, sB = 0;
    if (ubeg < sp.R) {
        const int f = ubeg / sp.per_s, l = (min(uend, sp.R) - 1) / sp.per_s;
        sA = (size_t)f + u;
        nA = l - f + 1;
    }
    if (uend > sp.R) {
        const int f = (max(ubeg, sp.R) - sp.R) / sp.chk, l = (uend - 1 - sp.R) / sp.chk;
        sB = (size_t)p.W + p.U + f + u;
        nB = l - f + 1;
    }
    const DecodeWs& ws = p.ws;

    if (!DENSE && p.want_nbr && warp >= D / 32) {
        // neighbour search over the graph logits the attention kernel stored,
        // for the unit's non-sink list entries [S, n).  Threshold filter:
        // theta = the 8th largest of the NBR_THREADS per-thread maxima is a
        // distinct entry's key with 7 larger ones, so every top-8 entry has
        // key >= theta; those few candidates are collected in shared memory
        // and sorted by one warp.
        __shared__ unsigned long long s_top[NBR_THREADS / 4];
        __shared__ unsigned long long s_cand[NBR_CAP];
        __shared__ int s_cnt;
        const int xt = t - D, xw = xt >> 5;
        const int n = uend - ubeg;
        const float* lamu = ws.lam + (size_t)u * ws.lam_cap;
        const int32_t* toks = p.sel_tok + (size_t)u * p.tok_cap;
        auto key_at = [&](int i) { return nbr_key(lamu[i], __ldg(toks + i)); };
        // all loads first (clamped in-range indices, no branches), so the
        // 2 x NBR_KEEP loads are in flight together
        float lv[NBR_KEEP];
        int pv[NBR_KEEP];
#pragma unroll
        for (int k = 0; k < NBR_KEEP; ++k) {
            const int i = min(p.S + xt + k * NBR_THREADS, n - 1);
            lv[k] = lamu[i];
            pv[k] = __ldg(toks + i);
        }
        unsigned long long kk[NBR_KEEP];
#pragma unroll
        for (int k = 0; k < NBR_KEEP; ++k)
            kk[k] = p.S + xt + k * NBR_THREADS < n ? nbr_key(lv[k], pv[k]) : 0ull;
        unsigned long long mx = 0;
#pragma unroll
        for (int k = 0; k < NBR_KEEP; ++k) mx = kk[k] > mx ? kk[k] : mx;
        for (int i = p.S + xt + NBR_KEEP * NBR_THREADS; i < n; i += NBR_THREADS) {
            const unsigned long long k2 = key_at(i);
            mx = k2 > mx ? k2 : mx;
        }
        if (xt == 0) s_cnt = 0;
        const unsigned long long srt = warp_sort_desc(mx, lane);
        if (lane < 8) s_top[xw * 8 + lane] = srt;
        asm volatile("bar.sync 1, %0;" ::"n"(NBR_THREADS) : "memory");
        // every warp sorts the NBR_WARPS x 8 warp leaders itself (no extra barrier)
        const unsigned long long theta =
            __shfl_sync(FULL, warp_sort_desc(lane < NBR_WARPS * 8 ? s_top[lane] : 0ull, lane), 7);
        auto offer = [&](unsigned long long k2) {
            if (k2 != 0ull && k2 >= theta) {
                const int slot = atomicAdd(&s_cnt, 1);
                if (slot < NBR_CAP) s_cand[slot] = k2;
            }
        };
#pragma unroll
        for (int k = 0; k < NBR_KEEP; ++k) offer(kk[k]);
        for (int i = p.S + xt + NBR_KEEP * NBR_THREADS; i < n; i += NBR_THREADS) offer(key_at(i));
        asm volatile("bar.sync 1, %0;" ::"n"(NBR_THREADS) : "memory");
        __shared__ int s_nbpos[CKV_NEIGHBOURS];
        if (xw == 0) {
            const int cnt = s_cnt;
            int32_t* outn = p.nbr8 ? p.nbr8 + (size_t)u * 8 : nullptr;
            if (cnt <= 32) {
                const unsigned long long x = warp_sort_desc(lane < cnt ? s_cand[lane] : 0ull, lane);
                if (lane < 8) {
                    const int np = x ? nbr_pos(x) : -1;
                    s_nbpos[lane] = np;
                    if (outn) outn[lane] = np;
                }
            } else {
                // many candidates (ties in the logits): 8 rounds, each taking
                // the best key below the previous winner, from the shared
                // list or, past its capacity, from the whole list
                unsigned long long prev = ~0ull;
                for (int r = 0; r < 8; ++r) {
                    unsigned long long best = 0;
                    if (cnt <= NBR_CAP) {
                        for (int c = lane; c < cnt; c += 32) {
                            const unsigned long long k2 = s_cand[c];
                            if (k2 < prev && k2 > best) best = k2;
                        }
                    } else {
                        for (int i = p.S + lane; i < n; i += 32) {
                            const unsigned long long k2 = key_at(i);
                            if (k2 < prev && k2 > best) best = k2;
                        }
                    }
                    best = warp_max_u64(best);
                    if (lane == 0) {
                        const int np = best ? nbr_pos(best) : -1;
                        s_nbpos[r] = np;
                        if (outn) outn[r] = np;
                    }
                    prev = best;  // 0 once the entries run out: every later round finds none
                }
            }
        }
        if (p.append) {
            asm volatile("bar.sync 1, %0;" ::"n"(NBR_THREADS) : "memory");  // s_nbpos complete
            merge_assign<T, D>(p, u, s_nbpos, xt);
        }
        return;
    }

    if (t >= D) return;
    // online merge, in slot order, of this thread's output dimension for every
    // head: running max, rescaled sum and accumulator; all loads of a chunk of
    // slots are issued before any is used
    constexpr int CH = GQ >= 8 ? 4 : 32 / GQ;
    float M[GQ], Ls[GQ], A[GQ];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        M[h] = -INFINITY;
        Ls[h] = 0.f;
        A[h] = 0.f;
    }
    for (int part = 0; part < 2; ++part) {
      const size_t s0 = part ? sB : sA;
      const int nslots = part ? nB : nA;
      for (int c0 = 0; c0 < nslots; c0 += CH) {
        float xm[CH][GQ], xl[CH][GQ], xa[CH][GQ];
        // unconditional loads at constant offsets from one base (the slot
        // arrays carry MERGE_PAD spare slots, so a chunk never reads past
        // them), masked afterwards by selects: every load of the chunk is in
        // flight before the first is used
        const float* mb = ws.m + (s0 + c0) * GQ;
        const float* lb = ws.l + (s0 + c0) * GQ;
        const float* ab = ws.acc + (s0 + c0) * GQ * D + t;
#pragma unroll
        for (int r = 0; r < CH; ++r) {
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                xm[r][h] = mb[r * GQ + h];
                xl[r][h] = lb[r * GQ + h];
                xa[r][h] = ab[(r * GQ + h) * D];
            }
        }
#pragma unroll
        for (int r = 0; r < CH; ++r) {
            const bool ok = c0 + r < nslots;
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                xm[r][h] = ok ? xm[r][h] : -INFINITY;
                xl[r][h] = ok ? xl[r][h] : 0.f;
                xa[r][h] = ok ? xa[r][h] : 0.f;
            }
        }
        // the chunk's maximum first, then independent weights: the dependent
        // chain per chunk is one rescale instead of one per slot
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float mc = -INFINITY;
#pragma unroll
            for (int r = 0; r < CH; ++r) mc = fmaxf(mc, xm[r][h]);
            if (mc == -INFINITY) continue;
            const float mn = fmaxf(M[h], mc);
            const float fo = exp2_approx(M[h] - mn);
            float ls = 0.f, a = 0.f;
#pragma unroll
            for (int r = 0; r < CH; ++r) {
                const float f = exp2_approx(xm[r][h] - mn);
                ls = fmaf(xl[r][h], f, ls);
                a = fmaf(xa[r][h], f, a);
            }
            Ls[h] = fmaf(Ls[h], fo, ls);
            A[h] = fmaf(A[h], fo, a);
            M[h] = mn;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < GQ; ++h) outu[h * D + t] = A[h] / Ls[h];
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Partial slots: W + U for the static slices, then NCH_MAX + U for the
// dynamic chunks, then MERGE_PAD spares.
static size_t decode_slots(int U) { return (size_t)MAX_DECODE_WARPS + NCH_MAX + 2 * (size_t)U + MERGE_PAD; }

size_t decode_ws_bytes(int U, int gq, int d, int lam_cap) {
    const size_t slots = decode_slots(U);
    return align256(slots * gq * 4) * 2 + align256(slots * gq * d * 4) + align256((size_t)U * lam_cap * 4);
}

// ws: the workspace base (its head holds the ticket); the parts follow the head
DecodeWs carve_decode_ws(void* ws, size_t head, int U, int gq, int d, int lam_cap) {
    const size_t slots = decode_slots(U);
    char* p = static_cast<char*>(ws);
    DecodeWs w;
    w.ticket = reinterpret_cast<int*>(p);
    p += head;
    w.m = reinterpret_cast<float*>(p);
    p += align256(slots * gq * 4);
    w.l = reinterpret_cast<float*>(p);
    p += align256(slots * gq * 4);
    w.acc = reinterpret_cast<float*>(p);
    p += align256(slots * gq * d * 4);
    w.lam = reinterpret_cast<float*>(p);
    w.lam_cap = lam_cap;
    return w;
}

namespace {

template <typename T, int D, int GQ, bool DENSE>
cudaError_t launch_decode_t(DecodeParams p, cudaStream_t st) {
    static LaunchCache lc;
    auto kern = decode_main<T, D, GQ, DENSE>;
    const size_t smem = DecSmem<T, D, GQ>::CTA_FIXED + (DENSE ? 0 : (size_t)(p.U + 1) * 4);
    int per_sm = 0, sms = 0;
    cudaError_t e = prepare_launch(kern, lc, smem, DEC_WARPS * 32, &per_sm, &sms);
    if (e != cudaSuccess) return e;
    if (sms <= 0 || per_sm <= 0) return cudaErrorInvalidConfiguration;
    int blocks = sms * per_sm;
    if (blocks * DEC_WARPS > MAX_DECODE_WARPS) blocks = MAX_DECODE_WARPS / DEC_WARPS;
    p.W = blocks * DEC_WARPS;
    e = launch_pdl(KK_ATTENTION, kern, dim3(blocks), dim3(DEC_WARPS * 32), smem, st, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(KK_MERGE, decode_merge<T, D, GQ, DENSE>, dim3(p.U), dim3(D + (DENSE ? 0 : 32 * NBR_WARPS)),
                      0, st, p);
}

template <bool DENSE>
cudaError_t dispatch(const CacheView& c, int gq, DecodeParams p, cudaStream_t st) {
#define CKV_DEC_CASE(TT, DD, GG)                                                      \
    if (c.d == DD && gq == GG) return launch_decode_t<TT, DD, GG, DENSE>(p, st);
    if (c.dtype == CKV_DTYPE_BF16) {
        CKV_DEC_CASE(__nv_bfloat16, 128, 1) CKV_DEC_CASE(__nv_bfloat16, 128, 2)
        CKV_DEC_CASE(__nv_bfloat16, 128, 4) CKV_DEC_CASE(__nv_bfloat16, 128, 8)
        CKV_DEC_CASE(__nv_bfloat16, 64, 1) CKV_DEC_CASE(__nv_bfloat16, 64, 2)
        CKV_DEC_CASE(__nv_bfloat16, 64, 4) CKV_DEC_CASE(__nv_bfloat16, 64, 8)
    } else {
        CKV_DEC_CASE(float, 128, 1) CKV_DEC_CASE(float, 128, 2)
        CKV_DEC_CASE(float, 128, 4) CKV_DEC_CASE(float, 128, 8)
        CKV_DEC_CASE(float, 64, 1) CKV_DEC_CASE(float, 64, 2)
        CKV_DEC_CASE(float, 64, 4) CKV_DEC_CASE(float, 64, 8)
    }
#undef CKV_DEC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_sparse_decode(const CacheView& c, const GraphView& g, const SelView& s,
                                 const void* q, float* out, int32_t* nbr8, void* ws, const AssignParams* ap,
                                 cudaStream_t st) {
    DecodeParams p{};
    p.k = c.k;
    p.v = c.v;
    p.sb = c.sb;
    p.sh = c.sh;
    p.st = c.st;
    p.q = q;
    p.Hq = c.Hq;
    p.Hkv = c.Hkv;
    p.G = g.G;
    p.U = c.B * g.G;
    p.per_head = g.mode == CKV_GRAPH_PER_HEAD;
    p.S = g.S;
    p.sel_tok = s.sel_tok;
    p.tok_cap = s.tok_cap;
    p.T_cap = c.T_cap;
    p.dev_err = g.dev_err;
    p.unit_prefix = s.unit_prefix;
    p.n_tok = s.n_tok;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)c.d);
    p.ws = carve_decode_ws(ws, ws_head_bytes(c.B, c.Hq), p.U, g.gq, c.d, s.tok_cap);
    p.want_nbr = nbr8 != nullptr || ap != nullptr;
    p.out = out;
    p.nbr8 = nbr8;
    if (ap) {
        p.append = 1;
        p.ap = *ap;
    }
    return dispatch<false>(c, g.gq, p, st);
}

cudaError_t launch_dense_decode(const CacheView& c, const void* q, int T, float* out, void* ws,
                                cudaStream_t st) {
    DecodeParams p{};
    p.k = c.k;
    p.v = c.v;
    p.sb = c.sb;
    p.sh = c.sh;
    p.st = c.st;
    p.q = q;
    p.Hq = c.Hq;
    p.Hkv = c.Hkv;
    p.G = c.Hkv;
    p.U = c.B * c.Hkv;
    p.per_head = 0;
    p.T = T;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)c.d);
    const int gq = c.Hq / c.Hkv;
    p.ws = carve_decode_ws(ws, ws_head_bytes(c.B, c.Hq), p.U, gq, c.d, 0);
    p.out = out;
    return dispatch<true>(c, gq, p, st);
}

}  // namespace ckv
