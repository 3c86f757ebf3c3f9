// Community scoring and budgeted selection for sm_100a, in one kernel.
//
// During generation each query is first matched against the community
// centres alone, and only the chosen communities are then read from the KV
// cache (CommunityKV, rit.work summary, section "A graph of tokens replaces
// re-clustering", paragraph 4); the active token budget is small (section
// "The speed-up depends on how many graphs the model stores").
//
// The score is s_c = max over the graph's query heads of q_h . cent_c /
// sqrt(d) in fp32, and the selection is exactly the one those scores give.
// score_select_kernel: one block of SEL_THREADS per graph unit, all of its
// state in shared memory, no global atomics and no kernel boundary:
//  1. first pass over every community, streaming the centres' int8 copy
//     (codes cent_q with one fp32 scale s_c per row, cent_qs: a quarter of
//     the fp32 bytes).  The query of each head is split exactly into two
//     int8 vectors, q ~ sq (128 hi + lo) with |q_i - sq (128 hi_i + lo_i)|
//     <= 0.51 sq, so every product is an exact integer dot product (dp4a on
//     the CUDA cores, 8 lanes per centre row, one 16-byte load per lane).
//     That gives s~_c = s_c sq (q_int . code_c) / sqrt(d) and a rigorous
//     bound e_c >= |s_c - s~_c| (Q8_BOUND, QSPLIT_BOUND).  Each community's
//     upper bound s~ + e goes to shared memory, and its size is added to a
//     shared 4096-bin histogram over the top 12 bits of the key of its lower
//     bound s~ - e, key = (orderable score << 32) | ~id (unique; orders
//     communities by score desc, id asc);
//  2. the histogram gives a bin edge t with more than the budget's weight of
//     communities certainly scoring >= t, so every selected community scores
//     >= t; the candidates are the communities whose upper bound reaches t
//     (tens to a few hundred), and only they are re-scored exactly in fp32
//     from cent.  A non-candidate scores below t and so below every selected
//     one, so ranking the candidates alone gives the exact selection: each
//     warp sorts 32 of them and a candidate's rank (and the sizes ranked
//     above it) is its place in its own run plus binary searches in the
//     others; more than SEL_FAST candidates are sorted block-wide in global
//     scratch; at least the top community is taken;
//  3. the unit's token list: sinks, build-time members of each selected
//     community (from the community-contiguous CSR), then the selected tail
//     members; and the runs' offsets and the tail entries' communities.
#include <math.h>
#include <type_traits>

#include "ckv_internal.cuh"

namespace ckv {

constexpr int SEL_WARPS = 16;
constexpr int SEL_THREADS = SEL_WARPS * 32;
constexpr int SEL_HBITS = 12;
constexpr int SEL_HBINS = 1 << SEL_HBITS;
constexpr int SEL_FAST = SEL_THREADS;       // candidates ranked in shared memory
constexpr int SC_LPR = 8;                   // lanes per centre row in the first pass
constexpr int SC_RPI = 32 / SC_LPR;         // rows per warp instruction
template <int GQ> struct ScRq { static constexpr int v = GQ == 1 ? 4 : GQ == 2 ? 2 : 1; };  // row groups per lane in flight
// Range of the integer query: q_i ~ sq Q_i with |Q_i| <= 127 * 128, so
// Q_i = 128 hi_i + lo_i with hi_i in [-127, 127] and lo_i in [-64, 63].
constexpr int Q_SPLIT = 127 * 128;
// Bound on |fp32 score from cent - fp32 score from the int8 copy| per unit
// of s_c |q|_1 / sqrt(d) (s_c the row's scale): the codes contribute at most
// 1/2 + 2^-16 (see q8_scale); the fp32 dot products of the exact re-score,
// of depth <= 19 over terms summing to at most 127 s_c |q|_1, about 2^-13.8;
// the conversion of the integer dot product and the products by sq, s_c and
// 1/sqrt(d), relative 2^-22 of a value below 127 s_c (|q|_1 + d sq / 2),
// about 2^-15.  So 1/2 + 2^-7 leaves a margin of 10 over the rounding terms.
constexpr float Q8_BOUND = 0.5f + 1.0f / 128.0f;
// The integer query: Q_i = rn(q_i * fl(Q_SPLIT / amax)) is within 1/2 +
// 2^-10 of q_i / sq, sq = fl(amax / Q_SPLIT), so |q_i - sq Q_i| <= 0.503 sq,
// and |code . (q - sq Q)| <= 127 d 0.51 sq per unit of s_c.
constexpr float QSPLIT_BOUND = 0.51f;
// Covers scales in the subnormal range.
constexpr float Q8_ABS_BOUND = 1e-30f;

struct SelectParams {
    const void* q;
    const float* cent;
    const int8_t* cent_q;       // [U, Cmax, D] int8 scoring copy of cent
    const float* cent_qs;       // [U, Cmax] its row scales
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

// Community c's build-time run [o0, o1) in the member list; debug builds
// check 0 <= o0 <= o1 <= T_cap (an empty run otherwise, with the error bit).
__device__ __forceinline__ void member_run(const int32_t* of, int c, int T_cap, int32_t* err, int& o0, int& o1) {
    o0 = of[c];
    o1 = of[c + 1];
    if constexpr (kDebugChecks) {
        if (o0 < 0 || o1 < o0 || o1 > T_cap) {
            atomicOr(err, CKV_DEVERR_INDEX);
            o0 = o1 = 0;
        }
    }
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

// A lane's share of an int8 code row: D / SC_LPR bytes (16 for d = 128).
template <int D> struct CodePart;
template <> struct CodePart<128> {
    static constexpr int W = 4;  // 32-bit words
    uint4 v;
    __device__ __forceinline__ void load(const int8_t* p) { v = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ uint32_t word(int k) const { return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w; }
};
template <> struct CodePart<64> {
    static constexpr int W = 2;
    uint2 v;
    __device__ __forceinline__ void load(const int8_t* p) { v = *reinterpret_cast<const uint2*>(p); }
    __device__ __forceinline__ uint32_t word(int k) const { return k == 0 ? v.x : v.y; }
};

// Sum of GQ per-head integers over the SC_LPR lanes of a row group with value
// exchange: afterwards lane lr holds the full sum of head lr >> (3 - log2 GQ).
template <int GQ>
__device__ __forceinline__ int rowgroup_reduce_heads(int (&v)[GQ], int lr) {
    static_assert(GQ <= SC_LPR, "one head per lane at least");
    int cur[GQ];
#pragma unroll
    for (int i = 0; i < GQ; ++i) cur[i] = v[i];
    int n = GQ;
#pragma unroll
    for (int o = SC_LPR / 2; o >= 1; o >>= 1) {
        if (n > 1) {
            const bool upper = (lr & o) != 0;
            const int h = n >> 1;
#pragma unroll
            for (int i = 0; i < h; ++i) {
                const int send = upper ? cur[i] : cur[i + h];
                const int keep = upper ? cur[i + h] : cur[i];
                cur[i] = keep + __shfl_xor_sync(FULL, send, o);
            }
            n = h;
        } else {
            cur[0] += __shfl_xor_sync(FULL, cur[0], o);
        }
    }
    return cur[0];
}

// Thread i < SEL_PREFETCH warms one page that the unit's selection reads or
// writes after the first pass (token list, members, CSR offsets, ranked ids,
// fp32 centres, tail), so the address translations are done before they are
// needed; issued before waiting for the previous kernel.
constexpr int SEL_PREFETCH = 10;
__device__ __forceinline__ void select_prefetch(const SelectParams& p, int u, int i, int D) {
    const size_t crow = (size_t)u * p.Cmax * D;
    const void* a = nullptr;
    switch (i) {
        case 0: a = p.sel_tok + (size_t)u * p.tok_cap; break;
        case 1: a = p.tok + (size_t)u * p.T_cap; break;
        case 2: a = p.tok + (size_t)u * p.T_cap + p.T_cap - 1; break;
        case 3: a = p.offs + (size_t)u * (p.Cmax + 1); break;
        case 4: a = p.sel_comm + (size_t)u * p.Cmax; break;
        case 5: a = p.cent + crow; break;
        case 6: a = p.cent + crow + (size_t)(p.Cmax - 1) * D; break;
        case 7: a = p.max_tail > 0 ? p.tail_tok + (size_t)u * p.max_tail : nullptr; break;
        case 8: a = p.max_tail > 0 ? p.tail_comm + (size_t)u * p.max_tail : nullptr; break;
        case 9: a = p.tail_len + u; break;
        default: break;
    }
    if (a) asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
}

// Dynamic shared memory of the kernel: the histogram, then per community its
// upper score bound and its size.
__host__ __device__ inline size_t sel_dyn_smem(int Cmax) {
    return (size_t)SEL_HBINS * 4 + 2 * (((size_t)Cmax * 4 + 15) & ~size_t(15));
}

template <typename T, int D, int GQ>
__global__ void __launch_bounds__(SEL_THREADS, 2) score_select_kernel(SelectParams p) {
    extern __shared__ __align__(16) unsigned char sel_dyn[];
    int* s_hist = reinterpret_cast<int*>(sel_dyn);
    float* s_ub = reinterpret_cast<float*>(sel_dyn + SEL_HBINS * 4);
    int* s_sz = reinterpret_cast<int*>(sel_dyn + SEL_HBINS * 4 + (((size_t)p.Cmax * 4 + 15) & ~size_t(15)));
    __shared__ unsigned long long s_key[SEL_FAST];
    __shared__ int s_w[SEL_FAST];
    __shared__ unsigned long long s_runs[SEL_FAST];
    __shared__ int s_bsz[SEL_FAST];
    __shared__ int s_ofs[SEL_FAST];
    __shared__ int s_len[SEL_FAST];  // candidate i's build-time run length
    __shared__ unsigned s_mask[MAX_CMAX / 32];
    __shared__ int s_warp[33];
    __shared__ int s_bstar, s_nc, s_nt, s_cnt;
    // the graph's queries: fp32 (exact re-scoring) and the int8 split words
    // (hi, then lo) of the first pass, with each head's scale and bound term
    __shared__ __align__(16) float s_qf[GQ][D];
    __shared__ __align__(16) uint32_t s_qw[GQ][2][D / 4];
    __shared__ float s_sq[GQ], s_eb[GQ];
    __shared__ float s_f[SEL_WARPS][32];  // first-pass sums of a warp's round, before the bounds

    constexpr int EW = D / 32;  // q elements per lane
    const int u = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    if (tid < SEL_PREFETCH) select_prefetch(p, u, tid, D);
    {
        int4* h4 = reinterpret_cast<int4*>(s_hist);
        for (int i = tid; i < SEL_HBINS / 4; i += nt) h4[i] = make_int4(0, 0, 0, 0);
    }
    for (int i = tid; i < (p.Cmax + 31) / 32; i += nt) s_mask[i] = 0u;
    if (tid == 0) {
        s_bstar = -1;
        s_nc = 0;
        s_cnt = 0;
    }
    pdl_wait();  // q, the centres and the counts may come from the kernels before

    using CP = CodePart<D>;
    constexpr int W = CP::W;
    constexpr int RQ = ScRq<GQ>::v;
    constexpr int STEP = SEL_WARPS * RQ * SC_RPI;  // rows per round of the block
    const int sub = lane / SC_LPR, lr = lane % SC_LPR;
    const int8_t* codes = p.cent_q + (size_t)u * p.Cmax * D + lr * (D / SC_LPR);
    const int32_t* cn = p.cnt + (size_t)u * p.Cmax;
    // 1. first pass: lane lr of row group `sub` owns D/8 dims of one row; two
    //    rounds of RQ row groups per warp in flight (the next round's codes are
    //    requested before the current one is used).  The first round and the
    //    rows' scales and sizes (to shared memory: s_ub, s_sz; each row's upper
    //    bound later replaces its scale) are requested before anything else,
    //    up to Cmax rows (the number present is not known yet)
    CP cva[RQ], cvb[RQ];
    auto load_codes = [&](CP (&cv)[RQ], int b0, int lim) {
#pragma unroll
        for (int j = 0; j < RQ; ++j) cv[j].load(codes + (size_t)min(b0 + j * SC_RPI + sub, lim - 1) * D);
    };
    int base = warp * RQ * SC_RPI;
    if (base < p.Cmax) load_codes(cva, base, p.Cmax);
    {
        const float* scales = p.cent_qs + (size_t)u * p.Cmax;
        for (int c = tid; c < p.Cmax; c += nt) {
            cp_async_4(s_ub + c, scales + c);
            cp_async_4(s_sz + c, cn + c);
        }
        cp_async_commit();
    }
    const int C = min(p.num_comm[u], p.Cmax);

    const int b = u / p.G, g = u - b * p.G;
    const int h0 = p.per_head ? g : g * GQ;
    if (warp < GQ) {
        // head `warp`: fp32 copy, |q|_1, and the integer split
        const T* qp = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h0 + warp) * D + lane * EW;
        float x[EW];
        float amax = 0.f, qn = 0.f;
#pragma unroll
        for (int e = 0; e < EW; ++e) {
            x[e] = to_f32(qp[e]);
            s_qf[warp][lane * EW + e] = x[e];
            amax = fmaxf(amax, fabsf(x[e]));
            qn += fabsf(x[e]);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
            qn += __shfl_xor_sync(FULL, qn, o);
        }
        const float sq = amax > 0.f ? __fdiv_rn(amax, (float)Q_SPLIT) : 0.f;
        const float rq = amax > 0.f ? __fdiv_rn((float)Q_SPLIT, amax) : 0.f;
        uint32_t hw = 0u, lw = 0u;
#pragma unroll
        for (int e = 0; e < EW; ++e) {
            const int Q = max(-Q_SPLIT, min(Q_SPLIT, __float2int_rn(x[e] * rq)));
            const int hi = (Q + 64) >> 7;  // floor((Q + 64) / 128)
            const int lo = Q - 128 * hi;
            hw |= (uint32_t)(hi & 0xff) << (8 * e);
            lw |= (uint32_t)(lo & 0xff) << (8 * e);
        }
        if constexpr (EW == 4) {
            s_qw[warp][0][lane] = hw;
            s_qw[warp][1][lane] = lw;
        } else {
            reinterpret_cast<uint16_t*>(s_qw[warp][0])[lane] = (uint16_t)hw;
            reinterpret_cast<uint16_t*>(s_qw[warp][1])[lane] = (uint16_t)lw;
        }
        if (lane == 0) {
            s_sq[warp] = sq;
            s_eb[warp] = fmaf(Q8_BOUND, qn, (127.0f * D * QSPLIT_BOUND) * sq);
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    {
        constexpr int LG = GQ == 1 ? 0 : GQ == 2 ? 1 : GQ == 4 ? 2 : 3;
        const int hl = lr >> (3 - LG);  // head whose sum this lane ends up with
        const float sq_mine = s_sq[hl];
        float eb = 0.f;
#pragma unroll
        for (int h = 0; h < GQ; ++h) eb = fmaxf(eb, s_eb[h]);
        const float ebase = eb * p.inv_sqrt_d;
        // the lane's query words: registers for one or two heads, else read
        // from shared memory per row group
        uint32_t qreg[GQ <= 2 ? GQ : 1][2][W];
        if constexpr (GQ <= 2) {
#pragma unroll
            for (int h = 0; h < GQ; ++h)
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    qreg[h][0][k] = s_qw[h][0][lr * W + k];
                    qreg[h][1][k] = s_qw[h][1][lr * W + k];
                }
        }
        float* my_f = s_f[warp];
        // scores of the round's rows: each row group's sum goes to my_f, then
        // lane i < RQ * SC_RPI finishes row base + i (bounds, histogram)
        auto score_round = [&](const CP (&cv)[RQ], int b0) {
#pragma unroll
            for (int j = 0; j < RQ; ++j) {
                int acc[GQ];
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    int ah = 0, al = 0;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        uint32_t qh, ql;
                        if constexpr (GQ <= 2) {
                            qh = qreg[h][0][k];
                            ql = qreg[h][1][k];
                        } else {
                            qh = s_qw[h][0][lr * W + k];
                            ql = s_qw[h][1][lr * W + k];
                        }
                        ah = __dp4a((int)cv[j].word(k), (int)qh, ah);
                        al = __dp4a((int)cv[j].word(k), (int)ql, al);
                    }
                    acc[h] = ah * 128 + al;  // exact: |acc| < 2^29
                }
                float f = (float)rowgroup_reduce_heads<GQ>(acc, lr) * sq_mine;
#pragma unroll
                for (int o = SC_LPR >> LG; o < SC_LPR; o <<= 1) f = fmaxf(f, __shfl_xor_sync(FULL, f, o));
                if (lr == 0) my_f[j * SC_RPI + sub] = f;
            }
            __syncwarp();
            const int c = b0 + lane;
            if (lane < RQ * SC_RPI && c < C) {
                const float rs = s_ub[c];
                const int w = s_sz[c];
                const float sc = my_f[lane] * rs * p.inv_sqrt_d;
                const float err = fmaf(ebase, rs, Q8_ABS_BOUND);
                s_ub[c] = w > 0 ? sc + err : -INFINITY;
                if (w > 0) atomicAdd(&s_hist[(int)(score_key(sc - err, c) >> (64 - SEL_HBITS))], w);
            }
            __syncwarp();
        };
        while (base < C) {
            if (base + STEP < C) load_codes(cvb, base + STEP, C);
            score_round(cva, base);
            base += STEP;
            if (base >= C) break;
            if (base + STEP < C) load_codes(cva, base + STEP, C);
            score_round(cvb, base);
            base += STEP;
        }
    }
    __syncthreads();

    // exact fp32 scores, from cent, of the n candidates whose keys (built
    // from the upper bounds) are in keys[]: one warp per candidate, RSC
    // candidates' rows in flight per warp; the keys are replaced in place
    constexpr int RSC = GQ >= 4 ? 2 : GQ == 2 ? 4 : 8;
    auto rescore = [&](unsigned long long* keys, int n) {
        for (int i0 = warp; i0 < n; i0 += RSC * nw) {
            float row[RSC][EW];
            int cid[RSC];
#pragma unroll
            for (int r = 0; r < RSC; ++r) {
                cid[r] = key_id(keys[min(i0 + r * nw, n - 1)]);
                const float* cr = p.cent + ((size_t)u * p.Cmax + cid[r]) * D + lane * EW;
                if constexpr (EW == 4) {
                    const float4 v = *reinterpret_cast<const float4*>(cr);
                    row[r][0] = v.x; row[r][1] = v.y; row[r][2] = v.z; row[r][3] = v.w;
                } else {
#pragma unroll
                    for (int e = 0; e < EW; ++e) row[r][e] = cr[e];
                }
            }
            unsigned long long nk[RSC];
#pragma unroll
            for (int r = 0; r < RSC; ++r) {
                float best = -INFINITY;
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < EW; ++e) a = fmaf(s_qf[h][lane * EW + e], row[r][e], a);
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

    // 2a. crossing bin: thread t owns bins [per*t, per*t + per)
    constexpr int per = SEL_HBINS / SEL_THREADS;
    static_assert(per == 8, "two int4 histogram loads per thread");
    {
        int hw[per];
        {
            const int4* h4 = reinterpret_cast<const int4*>(s_hist) + 2 * tid;
            const int4 a = h4[0], c = h4[1];
            hw[0] = a.x; hw[1] = a.y; hw[2] = a.z; hw[3] = a.w;
            hw[4] = c.x; hw[5] = c.y; hw[6] = c.z; hw[7] = c.w;
        }
        int own = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) own += hw[i];
        int total;
        const int pre = block_exclusive_scan(own, s_warp, &total);
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

    // 2b. candidates: keys from the crossing bin up, with their sizes; one
    //     shared-memory atomic per warp and round
    for (int c0 = 0; c0 < C; c0 += nt) {
        const int c = c0 + tid;
        bool cand = false;
        int w = 0;
        unsigned long long k = 0ull;
        if (c < C) {
            w = s_sz[c];
            k = score_key(s_ub[c], c);
            cand = w > 0 && (int)(k >> (64 - SEL_HBITS)) >= bstar;
        }
        const unsigned m = __ballot_sync(FULL, cand);
        int first = 0;
        if (lane == 0 && m) first = atomicAdd(&s_nc, __popc(m));
        first = __shfl_sync(FULL, first, 0);
        if (cand) {
            const int i = first + __popc(m & ((1u << lane) - 1u));
            if (i < SEL_FAST) {
                s_key[i] = k;
                s_w[i] = w;
                // its fp32 centre is re-scored next: start fetching it into L2
                const char* row = reinterpret_cast<const char*>(p.cent + ((size_t)u * p.Cmax + c) * D);
#pragma unroll
                for (int l = 0; l < D * 4 / 128; ++l) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + 128 * l));
            }
        }
    }
    __syncthreads();
    const int nc = s_nc;
    const int32_t* of = p.offs + (size_t)u * (p.Cmax + 1);
    // each candidate's CSR run, loaded now so the loads overlap the re-scoring
    // (the id bits of a key do not change when it is re-scored)
    int o0 = 0, o1 = 0;
    if (tid < min(nc, SEL_FAST)) {
        const int c = key_id(s_key[tid]);
        member_run(of, c, p.T_cap, p.dev_err, o0, o1);
    }
    if (nc <= SEL_FAST) {
        rescore(s_key, nc);
        if (tid < nc) s_len[tid] = o1 - o0;
        __syncthreads();
    }

    // 2c. the cut, from each candidate's rank and the sizes ranked above it
    //     (sizes are positive, so the selected set is a prefix of the
    //     ranking): candidate i is in iff the size above it plus its own fits
    //     the budget.  Warp r sorts candidates [32r, 32r + 32) best first and
    //     scans their sizes and run lengths in that order; an entry's rank is
    //     its place in its own run plus, in every other run, the number of
    //     entries above it (binary search), and the sizes above it the
    //     matching prefixes.  Sort values carry the candidate's slot below the
    //     id, which keeps the tie order (lower id first) and finds the payload.
    int kstar;
    const unsigned long long* sorted;
    const bool small = nc <= SEL_FAST;
    int* bsz = small ? s_bsz : p.gw + (size_t)u * p.npow_max;
    if (small) {
        __shared__ unsigned long long s_sv[SEL_FAST];
        __shared__ int s_pw[SEL_FAST], s_pl[SEL_FAST], s_o0[SEL_FAST];
        static_assert(SEL_FAST <= 1024 && MAX_CMAX <= (1 << 22), "slot and id fit the value's low 32 bits");
        const int R = (nc + 31) >> 5;
        int w = 0, len = 0;
        unsigned long long v = 0ull;  // below every real value
        if (warp < R) {
            if (tid < nc) {
                const unsigned long long k = s_key[tid];
                s_o0[tid] = o0;
                v = (k & 0xffffffff00000000ull) | ((unsigned long long)(MAX_CMAX - 1 - key_id(k)) << 10) |
                    (unsigned long long)tid;
            }
            v = warp_sort_desc(v, lane);
            if (v) {
                const int slot = (int)(v & 0x3ffu);
                w = s_w[slot];
                len = s_len[slot];
            }
            int pw = w, pl = len;  // inclusive prefixes in the run's order
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int yw = __shfl_up_sync(FULL, pw, o), yl = __shfl_up_sync(FULL, pl, o);
                if (lane >= o) {
                    pw += yw;
                    pl += yl;
                }
            }
            s_sv[tid] = v;
            s_pw[tid] = pw;
            s_pl[tid] = pl;
        }
        __syncthreads();
        bool in = false;
        if (warp < R && v) {
            int rank = lane, above = s_pw[tid] - w, above_len = s_pl[tid] - len;
            for (int r = 0; r < R; ++r) {
                if (r == warp) continue;
                const unsigned long long* run = s_sv + (r << 5);
                int lo = 0;  // entries of run r above v: a prefix of the run
#pragma unroll
                for (int step = 16; step >= 1; step >>= 1) lo += run[lo + step - 1] > v ? step : 0;
                lo += (lo == 31 && run[31] > v) ? 1 : 0;
                rank += lo;
                if (lo) {
                    above += s_pw[(r << 5) + lo - 1];
                    above_len += s_pl[(r << 5) + lo - 1];
                }
            }
            const int slot = (int)(v & 0x3ffu);
            const int id = MAX_CMAX - 1 - (int)((v >> 10) & 0x3fffffu);
            const int o0r = s_o0[slot];
            in = above + w <= p.budget;
            s_runs[rank] = (v & 0xffffffff00000000ull) | (unsigned long long)(0xffffffffu - (unsigned)id);
            s_bsz[rank] = above_len + len;  // inclusive prefix in rank order
            s_ofs[rank] = o0r;
            if (in || rank == 0) prefetch_run(p.tok + (size_t)u * p.T_cap + o0r, len);
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
            const int w = s_sz[c];
            if (w <= 0) continue;
            const unsigned long long k = score_key(s_ub[c], c);
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
        for (int i = tid; i < nc; i += nt) gw[i] = s_sz[key_id(gk[i])];
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
            int r0, r1;
            member_run(of, key_id(gk[i]), p.T_cap, p.dev_err, r0, r1);
            bsz[i] = r1 - r0;
        }
    }

    // 3a. ranked ids and membership mask
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
    constexpr int RND = 4;
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
            int src, r1;
            member_run(of, key_id(sorted[k]), p.T_cap, p.dev_err, src, r1);
            const int len = r1 - src;
            const int dst = p.S + bsz[k] - len;
            for (int i = lane; i < len; i += 32) {
                if (dst + i < p.tok_cap) out[dst + i] = tk[src + i];
                else overflow = true;
            }
        }
    }
    {
        // tail members of the selected communities, in tail order: the whole
        // block flags one entry per thread per round and compacts by a scan
        int tl = min(p.tail_len[u], p.max_tail);
        if constexpr (kDebugChecks) {
            if (tl < 0) {
                if (tid == 0) atomicOr(p.dev_err, CKV_DEVERR_INDEX);
                tl = 0;
            }
        }
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
    size_t gkey, gw, total;
};
SelWs sel_ws_layout(int U, int Cmax) {
    SelWs l;
    const size_t np = (size_t)next_pow2(Cmax);
    l.gkey = 0;
    l.gw = l.gkey + align256((size_t)U * np * 8);
    l.total = l.gw + align256((size_t)U * np * 4);
    return l;
}

template <typename T, int D, int GQ>
cudaError_t launch_t(const SelectParams& p, cudaStream_t st) {
    static LaunchCache lc;
    auto kern = score_select_kernel<T, D, GQ>;
    const size_t smem = sel_dyn_smem(p.Cmax);
    cudaError_t e = prepare_launch(kern, lc, smem, SEL_THREADS, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    return launch_pdl(KK_SCORE, kern, dim3(p.U), dim3(SEL_THREADS), smem, st, p);
}
}  // namespace

size_t select_ws_bytes(int U, int Cmax) { return sel_ws_layout(U, Cmax).total; }

cudaError_t launch_score_select(const CacheView& c, const GraphView& g, const void* q, int budget,
                                const SelView& s, void* ws, cudaStream_t st) {
    const int U = c.B * g.G;
    if (U <= 0) return cudaSuccess;
    const SelWs l = sel_ws_layout(U, g.Cmax);
    char* w = static_cast<char*>(ws) + ws_head_bytes(c.B, c.Hq);
    SelectParams p{};
    p.q = q;
    p.cent = g.cent;
    p.cent_q = g.cent_q;
    p.cent_qs = g.cent_qs;
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
