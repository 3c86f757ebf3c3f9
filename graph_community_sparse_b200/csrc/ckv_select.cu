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
// but the pass over every community streams the centres' int8 copy (codes
// cent_q with one fp32 scale s_c per row, cent_qs), a quarter of the fp32
// bytes:
//  * score_kernel, grid (centre blocks of 128, units): a streaming
//    matrix-vector product over the codes (16-byte loads; one query head:
//    8 lanes per row; several heads: tensor cores for a bf16 q, else a
//    half-warp per row with the value-exchanging butterfly of the attention
//    kernel for the head sums) gives s~_c = s_c q . code_c / sqrt(d) and a
//    rigorous bound e_c >= |s_c - s~_c| from s_c |q|_1 (Q8_BOUND).  The
//    upper bound s~ + e is stored; the community's size is added, with a global atomic, to a
//    per-unit histogram over the top 12 bits of the key of the lower bound
//    s~ - e, key = (orderable score << 32) | ~id (unique; orders communities
//    by score desc, id asc);
//  * select_kernel, one block per unit, launched as a programmatic
//    dependent: the lower-bound histogram gives a bin edge t with more than
//    the budget's weight of communities certainly scoring >= t, so every
//    selected community scores >= t; the candidates are the communities
//    whose upper bound reaches t (tens to a few hundred), and only they are
//    re-scored exactly in fp32 from cent.  A non-candidate scores below t
//    and so below every selected one, so ranking the candidates alone gives
//    the exact selection: up to 128 each against the others in shared
//    memory (which also gives the size ranked above it, so the cut needs no
//    sort), more by a sorting network in registers and one scan, more than
//    256 by a block-wide sort in global scratch; at least the top community
//    is taken.  Then the unit's token list: sinks, build-time members of
//    each selected community (from the community-contiguous CSR), then the
//    selected tail members; and the runs' offsets and the tail entries'
//    communities.
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
constexpr int RANK_LOOP_MAX = 128;          // up to this many: quadratic ranking; more: sorting network
// Bound on |fp32 score from cent - fp32 score from the int8 copy| per unit
// of s_c |q|_1 / sqrt(d) (s_c the row's scale): the codes contribute at most
// 1/2 + 2^-16 (see q8_scale); the fp32 dot products, of depth <= 19 over
// terms summing to at most 127 |q|_1 (codes) or 127 s_c |q|_1 (fp32 centre),
// about 2^-12.8 and 2^-13.8; the products by s_c and 1/sqrt(d) 2^-16.  So
// 1/2 + 2^-7 leaves a margin of 10 over the rounding terms.  The absolute
// term covers scales in the subnormal range.
constexpr float Q8_BOUND = 0.5f + 1.0f / 128.0f;
constexpr float Q8_ABS_BOUND = 1e-30f;

struct SelectParams {
    const void* q;
    const float* cent;
    const int8_t* cent_q;       // [U, Cmax, D] int8 scoring copy of cent
    const float* cent_qs;       // [U, Cmax] its row scales
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
    int32_t* tok_prefix;        // [U, Cmax + 1] run offsets of the list
    int32_t* tail_sel;          // [U, max(max_tail, 1)] communities of the list's tail part
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

// Exclusive scan of one 64-bit value per thread over the block (s_w64: 33
// entries of shared memory).
__device__ unsigned long long block_exclusive_scan_u64(unsigned long long x, unsigned long long* s_w64) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    unsigned long long inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_w64[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const unsigned long long w = lane < nw ? s_w64[lane] : 0ull;
        unsigned long long wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nw) s_w64[lane] = wi - w;
    }
    __syncthreads();
    return s_w64[warp] + inc - x;
}

// The token copy reads a selected run next: start fetching its first lines
// into L2.
__device__ __forceinline__ void prefetch_run(const int32_t* run, int len) {
    const int lines = min((len + 31) >> 5, 8);
    for (int l = 0; l < lines; ++l) asm volatile("prefetch.global.L2 [%0];" ::"l"(run + 32 * l));
}

// A lane's E int8 codes of a row (E bytes), kept packed until used.
__device__ __forceinline__ float q8_byte(uint32_t w, int k) {  // signed byte k of w
    return (float)((int)(w << (24 - 8 * k)) >> 24);
}
template <int E> struct Q8Part;
template <> struct Q8Part<4> {
    uint32_t w;
    __device__ __forceinline__ void load(const int8_t* p) { w = *reinterpret_cast<const uint32_t*>(p); }
    __device__ __forceinline__ void zero() { w = 0u; }
    __device__ __forceinline__ void unpack(float (&x)[4]) const {
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = q8_byte(w, k);
    }
};
template <> struct Q8Part<8> {
    uint2 w;
    __device__ __forceinline__ void load(const int8_t* p) { w = *reinterpret_cast<const uint2*>(p); }
    __device__ __forceinline__ void zero() { w = make_uint2(0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[8]) const {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            x[k] = q8_byte(w.x, k);
            x[4 + k] = q8_byte(w.y, k);
        }
    }
};
template <> struct Q8Part<16> {
    uint4 w;
    __device__ __forceinline__ void load(const int8_t* p) { w = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void zero() { w = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[16]) const {
        const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) x[4 * i + k] = q8_byte(v[i], k);
    }
};

// First-pass scores of this block's (up to) SCORE_ROWS centres of unit u,
// from the int8 copy: a warp owns SCORE_ROWS / SEL_WARPS consecutive rows;
// all of a lane's row parts (and the rows' scales) are loaded before any is
// used, so each warp keeps its rows in flight.  The score is
// s~ = s_c (q . code_c) / sqrt(d) and its bound e = Q8_BOUND s_c |q|_1 / sqrt(d).
// One query head per graph: SC_LPR lanes per row (D/SC_LPR codes each, one
// 16-byte load for d = 128), so a warp instruction covers 32/SC_LPR rows and
// a row's sum takes log2(SC_LPR) shuffle levels.
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
    Q8Part<E> raw[RQ];
    float rs[RQ];
    int wv[RQ];  // sizes, for the histogram
#pragma unroll
    for (int j = 0; j < RQ; ++j) {
        const int c = row0 + GR * j + oct;
        if (c < C) {
            raw[j].load(p.cent_q + ((size_t)u * p.Cmax + c) * D + l8 * E);
            rs[j] = p.cent_qs[(size_t)u * p.Cmax + c];
            wv[j] = p.cnt[(size_t)u * p.Cmax + c];
        } else {
            raw[j].zero();
            rs[j] = 0.f;
            wv[j] = 0;
        }
    }
    const int b = u / p.G, g = u - b * p.G;
    float qr[E], qn = 0.f;
    {
        const T* qp = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + g) * D + l8 * E;  // head g
#pragma unroll
        for (int e = 0; e < E; ++e) {
            qr[e] = to_f32(qp[e]);
            qn += fabsf(qr[e]);
        }
    }
#pragma unroll
    for (int o = SC_LPR / 2; o >= 1; o >>= 1) qn += __shfl_xor_sync(FULL, qn, o);  // |q|_1
    const float ebase = Q8_BOUND * qn * p.inv_sqrt_d;
    int32_t* hist = p.hist + (size_t)u * SEL_HBINS;
#pragma unroll
    for (int j = 0; j < RQ; ++j) {
        float x[E];
        raw[j].unpack(x);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) a = fmaf(qr[e], x[e], a);
#pragma unroll
        for (int o = SC_LPR / 2; o >= 1; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
        const float sc = a * rs[j] * p.inv_sqrt_d;
        const float err = fmaf(ebase, rs[j], Q8_ABS_BOUND);
        const int c = row0 + GR * j + oct;
        if (l8 == 0 && c < C) {
            p.scores[(size_t)u * p.Cmax + c] = sc + err;
            if (wv[j] > 0) atomicAdd(hist + (int)(score_key(sc - err, c) >> (64 - SEL_HBITS)), wv[j]);
        }
    }
}

// Several query heads per graph with a bf16 q: the products on the tensor
// cores (mma.sync m16n8k16, bf16 in, fp32 accumulate), heads as the A rows
// (padded with zeros), eight communities per n-tile as the B columns.  The
// int8 codes are exact in bf16, so S = Q code^T is the same sum as in the
// one-head path.  Lane (g, tq) owns dims [LB tq, LB tq + LB) of its rows
// (LB = D/4 bytes, one or two 16-byte loads) and of its head's q; k-step kk
// takes dims LB tq + 4kk .. +3 of every lane, which the fragment sees as
// k = 2tq, 2tq + 1 (register b0 / a0) and 2tq + 8, 2tq + 9 (b1 / a2): the
// same map on both operands, and over the k-steps every dim once.  A warp
// takes two n-tiles (16 communities); the 4 lanes of quad 0 then hold, per
// community, the max over the group's heads.
__device__ __forceinline__ void mma_sc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a1), "r"(0u), "r"(b0), "r"(b1));
}

// two signed bytes of w (k, k + 1) as a bf16 pair, low half first (exact)
__device__ __forceinline__ uint32_t q8_pair_bf16(uint32_t w, int k) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(q8_byte(w, k), q8_byte(w, k + 1));
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D, int GQ>
__device__ __forceinline__ void score_rows_mma(const SelectParams& p, int u, int C) {
    constexpr int KS = D / 16;   // k-steps
    constexpr int LB = D / 4;    // dims (bytes of codes) per lane and row
    constexpr int NV = LB / 16;  // 16-byte loads per lane and row
    constexpr int RW = SCORE_ROWS / SEL_WARPS;  // 16 communities per warp
    static_assert(RW == 16 && KS == LB / 4, "two n-tiles of 8 per warp; 4 dims per lane and k-step");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int row0 = blockIdx.x * SCORE_ROWS + warp * RW;
    if (row0 >= C) return;
    // codes of both n-tiles (community row0 + 8t + g) and the scales of the
    // four communities whose results this lane ends up holding (2tq + e)
    uint4 bw[2][NV];
    float rs[2][2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int c = row0 + 8 * t + g;
        const int8_t* row = p.cent_q + ((size_t)u * p.Cmax + min(c, C - 1)) * D + LB * tq;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const uint4 x = reinterpret_cast<const uint4*>(row)[v];
            bw[t][v] = c < C ? x : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int ce = row0 + 8 * t + 2 * tq + e;
            rs[t][e] = ce < C ? p.cent_qs[(size_t)u * p.Cmax + ce] : 0.f;
        }
    }
    const int wc = (lane < RW && row0 + lane < C) ? p.cnt[(size_t)u * p.Cmax + row0 + lane] : 0;
    const int b = u / p.G, gg = u - b * p.G;
    const int h0 = gg * GQ;  // per-group graphs (several heads)
    // this lane's dims of head g's q (bf16 pairs), and |q_g|_1 over the quad
    uint32_t qa[LB / 2];
    float qn = 0.f;
    {
        const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + h0 + min(g, GQ - 1)) * D + LB * tq;
#pragma unroll
        for (int v = 0; v < LB / 8; ++v) {
            const uint4 x = reinterpret_cast<const uint4*>(qrow)[v];
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                qa[4 * v + k] = g < GQ ? xs[k] : 0u;
                qn += fabsf(bf16_lo(qa[4 * v + k])) + fabsf(bf16_hi(qa[4 * v + k]));
            }
        }
    }
    qn += __shfl_xor_sync(FULL, qn, 1);
    qn += __shfl_xor_sync(FULL, qn, 2);
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) qn = fmaxf(qn, __shfl_xor_sync(FULL, qn, o));  // max over heads
    const float ebase = Q8_BOUND * qn * p.inv_sqrt_d;
    int32_t* hist = p.hist + (size_t)u * SEL_HBINS;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        uint32_t wd[4 * NV];  // code word kk: dims LB tq + 4kk .. +3
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            wd[4 * v] = bw[t][v].x;
            wd[4 * v + 1] = bw[t][v].y;
            wd[4 * v + 2] = bw[t][v].z;
            wd[4 * v + 3] = bw[t][v].w;
        }
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
            mma_sc(sacc, qa[2 * kk], qa[2 * kk + 1], q8_pair_bf16(wd[kk], 0), q8_pair_bf16(wd[kk], 2));
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            // max over the group's heads (rows g < GQ)
            float sv = g < GQ ? sacc[e] : -INFINITY;
#pragma unroll
            for (int o = 4; o <= 16; o <<= 1) sv = fmaxf(sv, __shfl_xor_sync(FULL, sv, o));
            const int r = 8 * t + 2 * tq + e;  // community row within the warp's 16
            const int w = __shfl_sync(FULL, wc, r);
            const float sc = sv * rs[t][e] * p.inv_sqrt_d;
            const float err = fmaf(ebase, rs[t][e], Q8_ABS_BOUND);
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
    Q8Part<E> raw[RH];
    float rs[RH];
#pragma unroll
    for (int j = 0; j < RH; ++j) {
        const int c = row0 + 2 * j + half;
        if (c < C) {
            raw[j].load(p.cent_q + ((size_t)u * p.Cmax + c) * D + l16 * E);
            rs[j] = p.cent_qs[(size_t)u * p.Cmax + c];
        } else {
            raw[j].zero();
            rs[j] = 0.f;
        }
    }
    const int wc = (lane < RW && row0 + lane < C) ? p.cnt[(size_t)u * p.Cmax + row0 + lane] : 0;
    const int b = u / p.G, g = u - b * p.G;
    const int h0 = p.per_head ? g : g * GQ;
    float qr[GQ][E], qn[GQ];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        load_row_part<T, E>(static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h0 + h) * D + l16 * E, qr[h]);
        qn[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) qn[h] += fabsf(qr[h][e]);
    }
    // max over the heads of |q_h|_1
    const float ebase = Q8_BOUND * halfwarp_max_over_heads<GQ>(halfwarp_reduce_heads<GQ>(qn, lane)) * p.inv_sqrt_d;

    int32_t* hist = p.hist + (size_t)u * SEL_HBINS;
#pragma unroll
    for (int j = 0; j < RH; ++j) {
        float x[E];
        raw[j].unpack(x);
        float part[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) a = fmaf(qr[h][e], x[e], a);
            part[h] = a;
        }
        float s = halfwarp_reduce_heads<GQ>(part, lane);
        s = halfwarp_max_over_heads<GQ>(s) * rs[j] * p.inv_sqrt_d;
        const float err = fmaf(ebase, rs[j], Q8_ABS_BOUND);
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
        if (nc <= RANK_LOOP_MAX) {  // uniform over the block
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
                if (in || rank == 0) prefetch_run(p.tok + (size_t)u * p.T_cap + o0, o1 - o0);
            }
        } else {
            // More candidates than the quadratic ranking pays for: the exact
            // keys are sorted best first in registers, a thread per entry, by
            // a bitonic network over next_pow2(nc) entries (partners in the
            // same warp exchange by shuffles, across warps through shared
            // memory); the low bits of a sort key carry the candidate's slot
            // next to its id, which keeps the tie order (lower id first).
            // One scan in rank order then gives the sizes and run lengths
            // ranked above each entry.
            __shared__ int s_o0[SEL_FAST];
            __shared__ unsigned long long s_w64[33];
            static_assert(SEL_FAST <= 256 && MAX_CMAX <= (1 << 24), "slot and id fit the key's low 32 bits");
            unsigned long long v = 0;  // below every real key
            if (tid < nc) {
                const unsigned long long k = s_key[tid];
                s_o0[tid] = o0;
                v = (k & 0xffffffff00000000ull) | ((unsigned long long)(MAX_CMAX - 1 - key_id(k)) << 8) |
                    (unsigned long long)tid;
            }
            int npow = 32;
            while (npow < nc) npow <<= 1;
            for (int k = 2; k <= npow; k <<= 1) {
                for (int j = k >> 1; j > 0; j >>= 1) {
                    unsigned long long o;
                    if (j >= 32) {  // uniform over the block
                        s_key[tid] = v;  // each thread read only its own entry above
                        __syncthreads();
                        o = s_key[tid ^ j];
                        __syncthreads();
                    } else {
                        o = __shfl_xor_sync(FULL, v, j);
                    }
                    const unsigned long long hi = v > o ? v : o, lo = v > o ? o : v;
                    v = (((tid & k) == 0) == ((tid & j) == 0)) ? hi : lo;
                }
            }
            int w = 0, len = 0, slot = 0;
            if (tid < nc) {
                slot = (int)(v & 0xffu);
                w = s_w[slot];
                len = s_len[slot];
            }
            // sizes and run lengths are each at most T_cap < 2^31: one 64-bit scan
            const unsigned long long pre =
                block_exclusive_scan_u64(((unsigned long long)w << 32) | (unsigned)len, s_w64);
            if (tid < nc) {
                const int above = (int)(pre >> 32), above_len = (int)(pre & 0xffffffffu);
                const int id = MAX_CMAX - 1 - (int)((v >> 8) & 0xffffffu);
                const int o0r = s_o0[slot];
                in = above + w <= p.budget;
                s_runs[tid] = (v & 0xffffffff00000000ull) | (unsigned long long)(0xffffffffu - (unsigned)id);
                s_bsz[tid] = above_len + len;  // inclusive prefix in rank order
                s_ofs[tid] = o0r;
                if (in || tid == 0) prefetch_run(p.tok + (size_t)u * p.T_cap + o0r, len);
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
    {
        // the runs' offsets in the list, for callers (and the attention's
        // update) that map a list entry back to its community
        int32_t* tp = p.tok_prefix + (size_t)u * (p.Cmax + 1);
        for (int k = tid; k <= kstar; k += nt) tp[k] = k ? bsz[k - 1] : 0;
    }

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
                p.tail_sel[(size_t)u * max(p.max_tail, 1) + (dst - p.S - nb)] = tc[i];
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
    cudaError_t e = launch_pdl(KK_SCORE, score_kernel<T, D, GQ>, grid, dim3(SEL_THREADS), 0, st, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(KK_SELECT, select_kernel<T, D, GQ>, dim3(p.U), dim3(SEL_THREADS), 0, st, p);
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
    p.cent_q = g.cent_q;
    p.cent_qs = g.cent_qs;
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
    p.tok_prefix = s.tok_prefix;
    p.tail_sel = s.tail_sel;
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
