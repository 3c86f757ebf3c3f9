// Community scoring and budgeted selection for sm_100a.
//
// During generation each query is first matched against the community
// centres alone, and only the chosen communities are then read from the KV
// cache (CommunityKV, rit.work summary, section "A graph of tokens replaces
// re-clustering", paragraph 4); the active token budget is small (section
// "The speed-up depends on how many graphs the model stores").
//
// The score is s_c = max over the graph's query heads of q_h . cent_c /
// sqrt(d) in fp32, and the selection is exactly the one those scores give;
// but the centres are streamed only once, in bf16 (cent_lp), which halves
// the bytes of the pass over every community:
//  * score_kernel, grid (centre blocks of 128, units): a streaming
//    matrix-vector product over the bf16 centres (one half-warp per row,
//    16-byte loads, the value-exchanging butterfly of the attention kernel
//    for the head sums) gives s~_c and a rigorous bound e_c >= |s_c - s~_c|
//    from sum |q| |cent_lp| (LP_REL_BOUND).  The upper bound s~ + e is
//    stored; the community's size is added, with a global atomic, to a
//    per-unit histogram over the top 12 bits of the key of the lower bound
//    s~ - e, key = (orderable score << 32) | ~id (unique; orders communities
//    by score desc, id asc);
//  * select_kernel, one block per unit, launched as a programmatic
//    dependent: the lower-bound histogram gives a bin edge t with more than
//    the budget's weight of communities certainly scoring >= t, so every
//    selected community scores >= t; the candidates are the communities
//    whose upper bound reaches t (typically a few dozen), and only they are
//    re-scored exactly in fp32 from cent.  A non-candidate scores below t
//    and so below every selected one, so ranking the candidates alone, each
//    against the others in shared memory (which also gives the size above
//    it and so the cut, at least the top community, with no sort), gives
//    the exact selection.  Then the unit's token list: sinks, build-time
//    members of each selected community (from the community-contiguous CSR),
//    then the selected tail members.
// The histograms live in the workspace head: zero on entry, and each
// selection block clears its unit's histogram after reading it.
#include <math.h>
#include <type_traits>

#include "ckv_internal.cuh"

namespace ckv {

constexpr int SEL_WARPS = 8;
constexpr int SEL_THREADS = SEL_WARPS * 32;
constexpr int SCORE_ROWS = SEL_WARPS * 16;      // centres per block (several heads per graph)
constexpr int SCORE_ROWS_GQ1 = SEL_WARPS * 16;  // centres per block (one head per graph)
template <int GQ> struct ScoreBlockRows { static constexpr int v = GQ == 1 ? SCORE_ROWS_GQ1 : SCORE_ROWS; };
constexpr int SEL_HBITS = HIST_BITS;
constexpr int SEL_HBINS = HIST_BINS;
constexpr int SEL_FAST = SEL_THREADS;       // candidates ranked in shared memory
// Bound on |fp32 score from cent - fp32 score from cent_lp| per unit of
// sum_i |q_i| |cent_lp_i| / sqrt(d): bf16 rounding contributes at most 2^-9
// (1 + 2^-9), the two fp32 dot products' rounding (depth <= 13 for d <= 128)
// about 2^-19 each; 2^-8 leaves a factor 1.9 of margin.  The absolute term
// covers bf16 subnormals.
constexpr float LP_REL_BOUND = 1.0f / 256.0f;
constexpr float LP_ABS_BOUND = 1e-30f;

struct SelectParams {
    const void* q;
    const float* cent;
    const __nv_bfloat16* cent_lp;
    float* scores;              // [U, Cmax] upper bound of each score (first pass)
    int32_t* hist;              // [U, SEL_HBINS]
    unsigned long long* gkey;   // [U, npow_max] scratch for large candidate sets
    int32_t* gw;                // [U, npow_max]
    const int32_t* cnt;
    const int32_t* offs;
    const int32_t* tok;
    const int32_t* num_comm;
    const int32_t* tail_tok;
    const int32_t* tail_comm;
    const int32_t* tail_len;
    int32_t* dev_err;
    int32_t* sel_comm;
    int32_t* n_sel;
    int32_t* sel_tok;
    int32_t* n_tok;
    int32_t* unit_prefix;
    int Hq, G, per_head;
    float inv_sqrt_d;
    int U, Cmax, npow_max, S, T_cap, max_tail, tok_cap, budget;
};

__device__ __forceinline__ unsigned long long score_key(float s, int c) {
    unsigned int b = __float_as_uint(s);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)b << 32) | (unsigned long long)(0xffffffffu - (unsigned)c);
}

__device__ __forceinline__ int key_id(unsigned long long k) {
    return (int)(0xffffffffu - (unsigned)(k & 0xffffffffull));
}

// In-place inclusive scan of n ints (shared or global memory, visible to the
// whole block); returns the total.
__device__ int block_scan_inplace(int* a, int n, int* s_warp) {
    const int nt = blockDim.x;
    const int seg = (n + nt - 1) / nt;
    const int b0 = min(n, threadIdx.x * seg), b1 = min(n, b0 + seg);
    int sum = 0;
    for (int i = b0; i < b1; ++i) sum += a[i];
    int total;
    int run = block_exclusive_scan(sum, s_warp, &total);
    for (int i = b0; i < b1; ++i) {
        run += a[i];
        a[i] = run;
    }
    __syncthreads();
    return total;
}

// Raw bf16 row part of a lane (E elements, 2E bytes), kept packed until used.
template <int E> struct RawPart;
template <> struct RawPart<8> {
    uint4 w;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { w = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void zero() { w = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[8]) const {
        x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
        x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
    }
};
template <> struct RawPart<16> {
    uint4 w0, w1;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) {
        w0 = reinterpret_cast<const uint4*>(p)[0];
        w1 = reinterpret_cast<const uint4*>(p)[1];
    }
    __device__ __forceinline__ void zero() { w0 = w1 = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[16]) const {
        const uint32_t v[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            x[2 * i] = bf16_lo(v[i]);
            x[2 * i + 1] = bf16_hi(v[i]);
        }
    }
};
template <> struct RawPart<32> {
    uint4 w[4];
    __device__ __forceinline__ void load(const __nv_bfloat16* p) {
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = reinterpret_cast<const uint4*>(p)[i];
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    __device__ __forceinline__ void unpack(float (&x)[32]) const {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t v[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                x[8 * i + 2 * k] = bf16_lo(v[k]);
                x[8 * i + 2 * k + 1] = bf16_hi(v[k]);
            }
        }
    }
};
template <> struct RawPart<4> {
    uint2 w;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { w = *reinterpret_cast<const uint2*>(p); }
    __device__ __forceinline__ void zero() { w = make_uint2(0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[4]) const {
        x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    }
};

// First-pass scores of this block's (up to) SCORE_ROWS centres of unit u:
// a warp owns SCORE_ROWS / SEL_WARPS consecutive rows, a half-warp every
// other one; all of a lane's row parts are loaded (packed) before any is
// used, so each warp keeps SCORE_ROWS / SEL_WARPS bf16 rows in flight.
// One query head per graph: SC_LPR lanes per row (D/SC_LPR elements each),
// so a warp instruction covers 32/SC_LPR rows and a row's sums take
// log2(SC_LPR) shuffle levels.
constexpr int SC_LPR = 8;
template <typename T, int D>
__device__ __forceinline__ void score_rows_gq1(const SelectParams& p, int u, int C) {
    constexpr int E = D / SC_LPR;
    constexpr int GR = 32 / SC_LPR;             // rows per warp instruction
    constexpr int RW = SCORE_ROWS_GQ1 / SEL_WARPS;  // rows per warp
    constexpr int RQ = RW / GR;                 // rows per lane group
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int oct = lane / SC_LPR, l8 = lane % SC_LPR;
    const int row0 = blockIdx.x * SCORE_ROWS_GQ1 + warp * RW;
    if (row0 >= C) return;
    RawPart<E> raw[RQ];
#pragma unroll
    for (int j = 0; j < RQ; ++j) {
        const int c = row0 + GR * j + oct;
        if (c < C) raw[j].load(p.cent_lp + ((size_t)u * p.Cmax + c) * D + l8 * E);
        else raw[j].zero();
    }
    const int wc = (lane < RW && row0 + lane < C) ? p.cnt[(size_t)u * p.Cmax + row0 + lane] : 0;
    const int b = u / p.G, g = u - b * p.G;
    float qr[E];
    {
        const T* qp = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + g) * D + l8 * E;  // head g
#pragma unroll
        for (int e = 0; e < E; ++e) qr[e] = to_f32(qp[e]);
    }
    int32_t* hist = p.hist + (size_t)u * SEL_HBINS;
#pragma unroll
    for (int j = 0; j < RQ; ++j) {
        float x[E];
        raw[j].unpack(x);
        float a = 0.f, m = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            a = fmaf(qr[e], x[e], a);
            m = fmaf(fabsf(qr[e]), fabsf(x[e]), m);
        }
#pragma unroll
        for (int o = SC_LPR / 2; o >= 1; o >>= 1) {
            a += __shfl_xor_sync(FULL, a, o);
            m += __shfl_xor_sync(FULL, m, o);
        }
        const float sc = a * p.inv_sqrt_d;
        // |exact score - sc| <= 2^-8 m / sqrt(d) (see LP_REL_BOUND)
        const float err = fmaf(LP_REL_BOUND, m * p.inv_sqrt_d, LP_ABS_BOUND);
        const int c = row0 + GR * j + oct;
        const int w = __shfl_sync(FULL, wc, GR * j + oct);
        if (l8 == 0 && c < C) {
            p.scores[(size_t)u * p.Cmax + c] = sc + err;
            if (w > 0) atomicAdd(hist + (int)(score_key(sc - err, c) >> (64 - SEL_HBITS)), w);
        }
    }
}

// Several query heads per graph with a bf16 q: both products on the tensor
// cores (mma.sync m16n8k16), heads as the A rows (padded with zeros), eight
// communities per n-tile as the B columns, loaded straight from global
// memory in fragment order: S = Q C~^T and the bound's M = |Q| |C~|^T, whose
// operands are the same registers with the sign bits cleared.  A warp takes
// two n-tiles (16 communities); the 4 lanes of quad 0 then hold, per
// community, the max over the group's heads of both.
__device__ __forceinline__ void mma_sc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a1), "r"(0u), "r"(b0), "r"(b1));
}

template <int D, int GQ>
__device__ __forceinline__ void score_rows_mma(const SelectParams& p, int u, int C) {
    constexpr int KS = D / 16;
    constexpr int RW = SCORE_ROWS / SEL_WARPS;  // 16 communities per warp
    static_assert(RW == 16, "two n-tiles of 8 per warp");
    constexpr uint32_t ABS = 0x7fff7fffu;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int row0 = blockIdx.x * SCORE_ROWS + warp * RW;
    if (row0 >= C) return;
    // B fragments of both n-tiles: community row0 + 8t + g, dims kk*16 + 2tq (+8)
    uint32_t bf[2][KS][2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int c = row0 + 8 * t + g;
        const __nv_bfloat16* row = p.cent_lp + ((size_t)u * p.Cmax + min(c, C - 1)) * D + 2 * tq;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const uint32_t x0 = *reinterpret_cast<const uint32_t*>(row + kk * 16);
            const uint32_t x1 = *reinterpret_cast<const uint32_t*>(row + kk * 16 + 8);
            bf[t][kk][0] = c < C ? x0 : 0u;
            bf[t][kk][1] = c < C ? x1 : 0u;
        }
    }
    const int wc = (lane < RW && row0 + lane < C) ? p.cnt[(size_t)u * p.Cmax + row0 + lane] : 0;
    const int b = u / p.G, gg = u - b * p.G;
    const int h0 = gg * GQ;  // per-group graphs (several heads)
    uint32_t qa[KS][2];
    {
        const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + h0 + min(g, GQ - 1)) * D + 2 * tq;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const uint32_t x0 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16);
            const uint32_t x1 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8);
            qa[kk][0] = g < GQ ? x0 : 0u;
            qa[kk][1] = g < GQ ? x1 : 0u;
        }
    }
    int32_t* hist = p.hist + (size_t)u * SEL_HBINS;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        float sacc[4] = {0.f, 0.f, 0.f, 0.f}, macc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            mma_sc(sacc, qa[kk][0], qa[kk][1], bf[t][kk][0], bf[t][kk][1]);
            mma_sc(macc, qa[kk][0] & ABS, qa[kk][1] & ABS, bf[t][kk][0] & ABS, bf[t][kk][1] & ABS);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            // max over the group's heads (rows g < GQ)
            float sv = g < GQ ? sacc[e] : -INFINITY, mv = g < GQ ? macc[e] : 0.f;
#pragma unroll
            for (int o = 4; o <= 16; o <<= 1) {
                sv = fmaxf(sv, __shfl_xor_sync(FULL, sv, o));
                mv = fmaxf(mv, __shfl_xor_sync(FULL, mv, o));
            }
            const int r = 8 * t + 2 * tq + e;  // community row within the warp's 16
            const int w = __shfl_sync(FULL, wc, r);
            const float sc = sv * p.inv_sqrt_d;
            const float err = fmaf(LP_REL_BOUND, mv * p.inv_sqrt_d, LP_ABS_BOUND);
            const int c = row0 + r;
            if (g == 0 && c < C) {
                p.scores[(size_t)u * p.Cmax + c] = sc + err;
                if (w > 0) atomicAdd(hist + (int)(score_key(sc - err, c) >> (64 - SEL_HBITS)), w);
            }
        }
    }
}

template <typename T, int D, int GQ>
__device__ __forceinline__ void score_rows(const SelectParams& p, int u, int C) {
    if constexpr (GQ == 1) {
        score_rows_gq1<T, D>(p, u, C);
        return;
    }
    if constexpr (GQ > 1 && std::is_same<T, __nv_bfloat16>::value) {
        score_rows_mma<D, GQ>(p, u, C);
        return;
    }
    constexpr int E = D / 16;
    constexpr int RW = SCORE_ROWS / SEL_WARPS;  // rows per warp
    constexpr int RH = RW / 2;                  // rows per half-warp
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4, l16 = lane & 15;
    const int row0 = blockIdx.x * SCORE_ROWS + warp * RW;
    if (row0 >= C) return;
    RawPart<E> raw[RH];
#pragma unroll
    for (int j = 0; j < RH; ++j) {
        const int c = row0 + 2 * j + half;
        if (c < C) raw[j].load(p.cent_lp + ((size_t)u * p.Cmax + c) * D + l16 * E);
        else raw[j].zero();
    }
    const int wc = (lane < RW && row0 + lane < C) ? p.cnt[(size_t)u * p.Cmax + row0 + lane] : 0;
    const int b = u / p.G, g = u - b * p.G;
    const int h0 = p.per_head ? g : g * GQ;
    float qr[GQ][E];
#pragma unroll
    for (int h = 0; h < GQ; ++h)
        load_row_part<T, E>(static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h0 + h) * D + l16 * E, qr[h]);

    int32_t* hist = p.hist + (size_t)u * SEL_HBINS;
#pragma unroll
    for (int j = 0; j < RH; ++j) {
        float x[E];
        raw[j].unpack(x);
        float part[GQ], mag[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float a = 0.f, m = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                a = fmaf(qr[h][e], x[e], a);
                m = fmaf(fabsf(qr[h][e]), fabsf(x[e]), m);
            }
            part[h] = a;
            mag[h] = m;
        }
        float s = halfwarp_reduce_heads<GQ>(part, lane);
        s = halfwarp_max_over_heads<GQ>(s) * p.inv_sqrt_d;
        float m = halfwarp_reduce_heads<GQ>(mag, lane);
        m = halfwarp_max_over_heads<GQ>(m) * p.inv_sqrt_d;
        // |exact score - s| <= 2^-8 m (see LP_REL_BOUND)
        const float err = fmaf(LP_REL_BOUND, m, LP_ABS_BOUND);
        const int c = row0 + 2 * j + half;
        const int w = __shfl_sync(FULL, wc, 2 * j + half);
        if (l16 == 0 && c < C) {
            p.scores[(size_t)u * p.Cmax + c] = s + err;
            if (w > 0) atomicAdd(hist + (int)(score_key(s - err, c) >> (64 - SEL_HBITS)), w);
        }
    }
}

// Selection for unit u after all its scores are in (see the file comment).
// Score bounds and the histogram were written by other blocks: read through L2.
template <typename T, int D, int GQ>
__device__ void select_unit(const SelectParams& p, int u, int C) {
    __shared__ unsigned long long s_key[SEL_FAST];
    __shared__ int s_w[SEL_FAST];
    __shared__ unsigned long long s_runs[SEL_FAST];
    __shared__ int s_bsz[SEL_FAST];
    __shared__ int s_ofs[SEL_FAST];
    __shared__ int s_len[SEL_FAST];  // candidate i's build-time run length
    __shared__ unsigned s_mask[MAX_CMAX / 32];
    __shared__ int s_warp[33];
    __shared__ int s_bstar, s_nc, s_nt, s_cnt;

    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const float* sc = p.scores + (size_t)u * p.Cmax;
    const int32_t* cn = p.cnt + (size_t)u * p.Cmax;
    const int32_t* hist = p.hist + (size_t)u * SEL_HBINS;
    for (int i = tid; i < (p.Cmax + 31) / 32; i += nt) s_mask[i] = 0u;
    if (tid == 0) {
        s_bstar = -1;
        s_nc = 0;
        s_cnt = 0;
    }

    // Every load that depends on nothing but u is issued first, together:
    // the histogram (16 bins per thread as four 16-byte loads) and the first
    // round of community sizes and scores (from clamped in-range ids, masked
    // by c < C later).
    constexpr int RND = 8;
    constexpr int per = SEL_HBINS / SEL_THREADS;
    static_assert(per == 16, "four int4 histogram loads per thread");
    int4 hv[4];
    {
        int4* h4 = reinterpret_cast<int4*>(const_cast<int32_t*>(hist) + per * tid);
#pragma unroll
        for (int i = 0; i < 4; ++i) hv[i] = __ldcg(h4 + i);
        // leave the histogram zero for the next call (each thread clears the
        // bins it alone read)
#pragma unroll
        for (int i = 0; i < 4; ++i) h4[i] = make_int4(0, 0, 0, 0);
    }
    int wv[RND];
    float sv[RND];
#pragma unroll
    for (int r = 0; r < RND; ++r) {
        const int c = min(tid + r * nt, p.Cmax - 1);
        wv[r] = cn[c];
        sv[r] = __ldcg(sc + c);
    }
    // this lane's part of the graph's queries, for the exact re-scoring
    constexpr int EW = D / 32;
    float qw[GQ][EW];
    {
        const int b = u / p.G, g = u - b * p.G;
        const int h0 = p.per_head ? g : g * GQ;
#pragma unroll
        for (int h = 0; h < GQ; ++h)
#pragma unroll
            for (int e = 0; e < EW; ++e)
                qw[h][e] = to_f32(static_cast<const T*>(p.q)[((size_t)b * p.Hq + h0 + h) * D + lane * EW + e]);
    }
    // exact fp32 scores, from cent, of the n candidates whose keys (built
    // from the upper bounds) are in keys[]: one warp per candidate, RSC
    // candidates' rows in flight per warp; the keys are replaced in place
    constexpr int RSC = 8;
    auto rescore = [&](unsigned long long* keys, int n) {
        for (int i0 = warp; i0 < n; i0 += RSC * nw) {
            float row[RSC][EW];
            int cid[RSC];
#pragma unroll
            for (int r = 0; r < RSC; ++r) {
                cid[r] = key_id(keys[min(i0 + r * nw, n - 1)]);
                const float* cr = p.cent + ((size_t)u * p.Cmax + cid[r]) * D + lane * EW;
#pragma unroll
                for (int e = 0; e < EW; ++e) row[r][e] = cr[e];
            }
            unsigned long long nk[RSC];
#pragma unroll
            for (int r = 0; r < RSC; ++r) {
                float best = -INFINITY;
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < EW; ++e) a = fmaf(qw[h][e], row[r][e], a);
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
                    best = fmaxf(best, a);
                }
                nk[r] = score_key(best * p.inv_sqrt_d, cid[r]);
            }
            __syncwarp();  // every lane has read its keys before lane 0 rewrites them
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < RSC; ++r)
                    if (i0 + r * nw < n) keys[i0 + r * nw] = nk[r];
            }
        }
    };

    // 1. crossing bin: thread t owns bins [per*t, per*t + per)
    {
        const int hw[per] = {hv[0].x, hv[0].y, hv[0].z, hv[0].w, hv[1].x, hv[1].y, hv[1].z, hv[1].w,
                             hv[2].x, hv[2].y, hv[2].z, hv[2].w, hv[3].x, hv[3].y, hv[3].z, hv[3].w};
        int own = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) own += hw[i];
        int total;
        const int pre = block_exclusive_scan(own, s_warp, &total);  // also orders the inits above
        int above = total - pre - own;  // weight of every bin above this thread's
#pragma unroll
        for (int i = per - 1; i >= 0; --i) {
            if (above + hw[i] > p.budget) {
                atomicMax(&s_bstar, per * tid + i);
                break;
            }
            above += hw[i];
        }
    }
    __syncthreads();
    const int bstar = max(s_bstar, 0);  // no crossing: every key is a candidate

    // 2. candidates: keys from the crossing bin up, with their sizes
    auto offer = [&](int c, int w, float sval) {
        if (c >= C || w <= 0) return;
        const unsigned long long k = score_key(sval, c);
        if ((int)(k >> (64 - SEL_HBITS)) >= bstar) {
            const int i = atomicAdd(&s_nc, 1);
            if (i < SEL_FAST) {
                s_key[i] = k;
                s_w[i] = w;
                // its fp32 centre is re-scored next: start fetching it into L2
                const char* row = reinterpret_cast<const char*>(p.cent + ((size_t)u * p.Cmax + c) * D);
#pragma unroll
                for (int l = 0; l < D * 4 / 128; ++l) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + 128 * l));
            }
        }
    };
#pragma unroll
    for (int r = 0; r < RND; ++r) offer(tid + r * nt, wv[r], sv[r]);
    for (int c0 = tid + RND * nt; c0 < C; c0 += RND * nt) {
#pragma unroll
        for (int r = 0; r < RND; ++r) {
            const int c = min(c0 + r * nt, p.Cmax - 1);
            wv[r] = cn[c];
            sv[r] = __ldcg(sc + c);
        }
#pragma unroll
        for (int r = 0; r < RND; ++r) offer(c0 + r * nt, wv[r], sv[r]);
    }
    __syncthreads();
    const int nc = s_nc;
    const int32_t* of = p.offs + (size_t)u * (p.Cmax + 1);
    // each candidate's CSR run, loaded now so the loads overlap the re-scoring
    // (the id bits of a key do not change when it is re-scored)
    int o0 = 0, o1 = 0;
    if (tid < min(nc, SEL_FAST)) {
        const int c = key_id(s_key[tid]);
        o0 = of[c];
        o1 = of[c + 1];
    }
    if (nc <= SEL_FAST) {
        rescore(s_key, nc);
        if (tid < nc) s_len[tid] = o1 - o0;
        __syncthreads();
    }

    // 3. the cut.  Few candidates (the usual case): no sort; candidate i's
    //    rank is the number of larger keys and the weight above it their size
    //    sum, so it is selected iff that sum plus its own size fits the budget
    //    (sizes are positive, so the selected set is a prefix of the ranking).
    //    Each candidate's CSR run is looked up meanwhile and stored at its rank.
    int kstar;
    const unsigned long long* sorted;
    const bool small = nc <= SEL_FAST;
    int* bsz = small ? s_bsz : p.gw + (size_t)u * p.npow_max;
    if (small) {
        bool in = false;
        if (tid < nc) {
            const unsigned long long k = s_key[tid];
            const int w = s_w[tid];
            // rank, the size ranked above (for the cut) and the run length
            // ranked above (the run's place in the token list)
            int rank = 0, above = 0, above_len = 0;
            for (int j = 0; j < nc; ++j) {
                const bool gt = s_key[j] > k;
                rank += gt;
                above += gt ? s_w[j] : 0;
                above_len += gt ? s_len[j] : 0;
            }
            in = above + w <= p.budget;
            s_runs[rank] = k;
            s_bsz[rank] = above_len + (o1 - o0);  // inclusive prefix in rank order
            s_ofs[rank] = o0;
            if (in || rank == 0) {
                // the token copy reads this run next: start fetching it into L2
                const int32_t* run = p.tok + (size_t)u * p.T_cap + o0;
                const int lines = min((o1 - o0 + 31) >> 5, 8);
                for (int l = 0; l < lines; ++l) asm volatile("prefetch.global.L2 [%0];" ::"l"(run + 32 * l));
            }
        }
        kstar = __syncthreads_count(in);
        if (kstar == 0 && nc > 0) kstar = 1;  // the top community alone exceeds the budget: take it
        sorted = s_runs;
    } else {
        // rare: more candidates than shared memory holds; sort them in
        // global scratch (block-wide bitonic, barriers between stages)
        unsigned long long* gk = p.gkey + (size_t)u * p.npow_max;
        int* gw = p.gw + (size_t)u * p.npow_max;
        if (tid == 0) s_nc = 0;
        __syncthreads();
        for (int c = tid; c < C; c += nt) {
            const int w = cn[c];
            if (w <= 0) continue;
            const unsigned long long k = score_key(__ldcg(sc + c), c);
            if ((int)(k >> (64 - SEL_HBITS)) >= bstar) gk[atomicAdd(&s_nc, 1)] = k;
        }
        __syncthreads();
        rescore(gk, nc);
        __syncthreads();
        int np2 = 1;
        while (np2 < nc) np2 <<= 1;
        for (int i = nc + tid; i < np2; i += nt) gk[i] = 0ull;
        __syncthreads();
        for (int k = 2; k <= np2; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int pi = tid; pi < (np2 >> 1); pi += nt) {
                    const int i = ((pi / j) * 2 * j) + (pi % j);
                    const int ixj = i + j;
                    const unsigned long long a = gk[i], bb = gk[ixj];
                    if (((i & k) == 0) ? (a < bb) : (a > bb)) {
                        gk[i] = bb;
                        gk[ixj] = a;
                    }
                }
                __syncthreads();
            }
        }
        for (int i = tid; i < nc; i += nt) gw[i] = cn[key_id(gk[i])];
        __syncthreads();
        block_scan_inplace(gw, nc, s_warp);
        int mine = 0;
        for (int i = tid; i < nc; i += nt) mine += gw[i] <= p.budget;
        atomicAdd(&s_cnt, mine);
        __syncthreads();
        kstar = s_cnt;
        if (kstar == 0 && nc > 0) kstar = 1;  // the top community alone exceeds the budget: take it
        sorted = gk;
        __syncthreads();
        for (int i = tid; i < kstar; i += nt) {  // gw's weights are no longer needed
            const int c = key_id(gk[i]);
            bsz[i] = of[c + 1] - of[c];
        }
    }

    // 4. ranked ids and membership mask
    int32_t* selc = p.sel_comm + (size_t)u * p.Cmax;
    for (int i = tid; i < kstar; i += nt) {
        const int c = key_id(sorted[i]);
        selc[i] = c;
        atomicOr(&s_mask[c >> 5], 1u << (c & 31));
    }
    __syncthreads();
    // tokens of the selected runs; their inclusive prefix (the small path
    // ranked it already)
    const int nb = small ? (kstar > 0 ? s_bsz[kstar - 1] : 0) : block_scan_inplace(bsz, kstar, s_warp);

    int32_t* out = p.sel_tok + (size_t)u * p.tok_cap;
    const int32_t* tk = p.tok + (size_t)u * p.T_cap;
    bool overflow = false;
    for (int i = tid; i < p.S; i += nt) {
        if (i < p.tok_cap) out[i] = i;
        else overflow = true;
    }
    if (small) {
        // one token per thread per round: its run is found by binary search in
        // the inclusive run prefix; a round's loads are issued before its stores
        for (int t0 = tid; t0 < nb; t0 += RND * nt) {
            // the run of each of the round's tokens: first k with s_bsz[k] > t
            // (the number of inclusive run ends <= t), by branch-free binary
            // lifting done for all of the round's tokens in lockstep, so the
            // RND searches' shared-memory loads overlap
            int tt[RND], lo[RND];
#pragma unroll
            for (int r = 0; r < RND; ++r) {
                tt[r] = min(t0 + r * nt, nb - 1);
                lo[r] = 0;
            }
#pragma unroll
            for (int step = SEL_FAST / 2; step > 0; step >>= 1) {
#pragma unroll
                for (int r = 0; r < RND; ++r) {
                    const int probe = min(lo[r] + step, kstar) - 1;  // in range: kstar >= 1
                    const bool fits = lo[r] + step <= kstar;
                    const bool le = s_bsz[probe] <= tt[r];
                    lo[r] += (fits & le) ? step : 0;
                }
            }
            int src[RND];
#pragma unroll
            for (int r = 0; r < RND; ++r) {
                const int start = lo[r] ? s_bsz[lo[r] - 1] : 0;
                src[r] = s_ofs[lo[r]] + (tt[r] - start);
            }
            // all of the round's loads in flight together (src 0 is in range)
            int val[RND];
#pragma unroll
            for (int r = 0; r < RND; ++r) val[r] = tk[src[r]];
#pragma unroll
            for (int r = 0; r < RND; ++r) {
                const int t = t0 + r * nt;
                if (t < nb) {
                    if (p.S + t < p.tok_cap) out[p.S + t] = val[r];
                    else overflow = true;
                }
            }
        }
    } else {
        for (int k = warp; k < kstar; k += nw) {
            const int c = key_id(sorted[k]);
            const int len = of[c + 1] - of[c];
            const int dst = p.S + bsz[k] - len;
            const int src = of[c];
            for (int i = lane; i < len; i += 32) {
                if (dst + i < p.tok_cap) out[dst + i] = tk[src + i];
                else overflow = true;
            }
        }
    }
    {
        // tail members of the selected communities, in tail order: the whole
        // block flags one entry per thread per round and compacts by a scan
        const int tl = min(p.tail_len[u], p.max_tail);
        const int32_t* tt = p.tail_tok + (size_t)u * p.max_tail;
        const int32_t* tc = p.tail_comm + (size_t)u * p.max_tail;
        int base = p.S + nb;
        for (int c0 = 0; c0 < tl; c0 += nt) {
            const int i = c0 + tid;
            int in = 0;
            if (i < tl) {
                const int c = tc[i];
                in = c >= 0 && c < p.Cmax && ((s_mask[c >> 5] >> (c & 31)) & 1u);
            }
            int total;
            const int off = block_exclusive_scan(in, s_warp, &total);
            if (in) {
                const int dst = base + off;
                if (dst < p.tok_cap) out[dst] = tt[i];
                else overflow = true;
            }
            base += total;
        }
        if (tid == 0) s_nt = base;
    }
    if (__syncthreads_or(overflow) && tid == 0) atomicOr(p.dev_err, CKV_DEVERR_TOKEN_CAP);
    if (tid == 0) {
        p.n_sel[u] = kstar;
        p.n_tok[u] = min(s_nt, p.tok_cap);
    }
}

template <typename T, int D, int GQ>
__global__ void __launch_bounds__(SEL_THREADS) score_kernel(SelectParams p) {
    pdl_wait();  // q may come from the kernel before
    const int u = blockIdx.y;
    const int C = min(p.num_comm[u], p.Cmax);
    score_rows<T, D, GQ>(p, u, C);
}

// Thread i < SEL_PREFETCH warms one page the selection of unit u reads or
// writes after its first loads (token list, members, CSR offsets, ranked
// ids, sizes, fp32 centres, tail), so the address translations are done
// before they are needed.  None is written by the scoring kernel: issued
// before waiting for it, they overlap its last blocks.
constexpr int SEL_PREFETCH = 11;
__device__ __forceinline__ void select_prefetch(const SelectParams& p, int u, int i, int D) {
    const size_t crow = (size_t)u * p.Cmax * D;
    const void* a = nullptr;
    switch (i) {
        case 0: a = p.sel_tok + (size_t)u * p.tok_cap; break;
        case 1: a = p.tok + (size_t)u * p.T_cap; break;
        case 2: a = p.tok + (size_t)u * p.T_cap + p.T_cap - 1; break;
        case 3: a = p.offs + (size_t)u * (p.Cmax + 1); break;
        case 4: a = p.sel_comm + (size_t)u * p.Cmax; break;
        case 5: a = p.cnt + (size_t)u * p.Cmax; break;
        case 6: a = p.cent + crow; break;
        case 7: a = p.cent + crow + (size_t)(p.Cmax - 1) * D; break;
        case 8: a = p.max_tail > 0 ? p.tail_tok + (size_t)u * p.max_tail : nullptr; break;
        case 9: a = p.max_tail > 0 ? p.tail_comm + (size_t)u * p.max_tail : nullptr; break;
        case 10: a = p.tail_len + u; break;
        default: break;
    }
    if (a) asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
}

template <typename T, int D, int GQ>
__global__ void __launch_bounds__(SEL_THREADS) select_kernel(SelectParams p) {
    const int u = blockIdx.x;
    if (threadIdx.x < SEL_PREFETCH) select_prefetch(p, u, threadIdx.x, D);
    pdl_wait();  // every score and histogram update of the scoring kernel is visible
    const int C = min(p.num_comm[u], p.Cmax);
    select_unit<T, D, GQ>(p, u, C);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static int next_pow2(int x) {
    int n = 1;
    while (n < x) n <<= 1;
    return n;
}

namespace {
struct SelWs {
    size_t scores, gkey, gw, total;
};
SelWs sel_ws_layout(int U, int Cmax) {
    SelWs l;
    const size_t np = (size_t)next_pow2(Cmax);
    l.scores = 0;
    l.gkey = l.scores + align256((size_t)U * Cmax * 4);
    l.gw = l.gkey + align256((size_t)U * np * 8);
    l.total = l.gw + align256((size_t)U * np * 4);
    return l;
}

template <typename T, int D, int GQ>
cudaError_t launch_t(const SelectParams& p, cudaStream_t st) {
    constexpr int rows = ScoreBlockRows<GQ>::v;
    dim3 grid((p.Cmax + rows - 1) / rows, p.U);
    cudaError_t e = launch_pdl(score_kernel<T, D, GQ>, grid, dim3(SEL_THREADS), 0, st, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(select_kernel<T, D, GQ>, dim3(p.U), dim3(SEL_THREADS), 0, st, p);
}
}  // namespace

size_t select_ws_bytes(int U, int Cmax) { return sel_ws_layout(U, Cmax).total; }

cudaError_t launch_score_select(const CacheView& c, const GraphView& g, const void* q, int budget,
                                const SelView& s, void* ws, cudaStream_t st) {
    const int U = c.B * g.G;
    const SelWs l = sel_ws_layout(U, g.Cmax);
    char* w = static_cast<char*>(ws) + ws_head_bytes(c.B, c.Hq);
    SelectParams p{};
    p.q = q;
    p.cent = g.cent;
    p.cent_lp = g.cent_lp;
    p.scores = reinterpret_cast<float*>(w + l.scores);
    p.hist = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + WS_RESERVED);  // zero on entry
    p.gkey = reinterpret_cast<unsigned long long*>(w + l.gkey);
    p.gw = reinterpret_cast<int32_t*>(w + l.gw);
    p.cnt = g.cnt;
    p.offs = g.offs;
    p.tok = g.tok;
    p.num_comm = g.num_comm;
    p.tail_tok = g.tail_tok;
    p.tail_comm = g.tail_comm;
    p.tail_len = g.tail_len;
    p.dev_err = g.dev_err;
    p.sel_comm = s.sel_comm;
    p.n_sel = s.n_sel;
    p.sel_tok = s.sel_tok;
    p.n_tok = s.n_tok;
    p.unit_prefix = s.unit_prefix;
    p.Hq = c.Hq;
    p.G = g.G;
    p.per_head = g.mode == CKV_GRAPH_PER_HEAD;
    p.inv_sqrt_d = 1.0f / sqrtf((float)c.d);
    p.U = U;
    p.Cmax = g.Cmax;
    p.npow_max = next_pow2(g.Cmax);
    p.S = g.S;
    p.T_cap = g.T_cap;
    p.max_tail = g.max_tail;
    p.tok_cap = s.tok_cap;
    p.budget = budget;

#define CKV_SC_CASE(TT, DD, GG) \
    if (c.d == DD && g.gq == GG) return launch_t<TT, DD, GG>(p, st);
    if (c.dtype == CKV_DTYPE_BF16) {
        CKV_SC_CASE(__nv_bfloat16, 128, 1) CKV_SC_CASE(__nv_bfloat16, 128, 2)
        CKV_SC_CASE(__nv_bfloat16, 128, 4) CKV_SC_CASE(__nv_bfloat16, 128, 8)
        CKV_SC_CASE(__nv_bfloat16, 64, 1) CKV_SC_CASE(__nv_bfloat16, 64, 2)
        CKV_SC_CASE(__nv_bfloat16, 64, 4) CKV_SC_CASE(__nv_bfloat16, 64, 8)
    } else {
        CKV_SC_CASE(float, 128, 1) CKV_SC_CASE(float, 128, 2)
        CKV_SC_CASE(float, 128, 4) CKV_SC_CASE(float, 128, 8)
        CKV_SC_CASE(float, 64, 1) CKV_SC_CASE(float, 64, 2)
        CKV_SC_CASE(float, 64, 4) CKV_SC_CASE(float, 64, 8)
    }
#undef CKV_SC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace ckv
