// Community scoring and budgeted selection for sm_100a.
//
// During generation each query is first matched against the community
// centres alone, and only the chosen communities are then read from the KV
// cache (CommunityKV, rit.work summary, section "A graph of tokens replaces
// re-clustering", paragraph 4); the active token budget is small (section
// "The speed-up depends on how many graphs the model stores").
//
// score_kernel: s_c = max over the graph's query heads of q_h . cent_c /
//   sqrt(d).  A streaming matrix-vector product over the fp32 centres: one
//   half-warp per centre row, 16-byte loads, the same value-exchanging
//   butterfly as the attention kernel for the head sums.
// select_kernel: one block per graph unit.  Keys (orderable score << 32 |
//   ~id) are sorted descending in shared memory (bitonic), the sizes are
//   prefix-summed in rank order and the longest prefix within the budget is
//   kept (at least the top community).  The block then writes the unit's
//   token list: sinks, build-time members of each selected community (copied
//   from the community-contiguous CSR), then the selected tail members.  The
//   last block to finish (atomic ticket; no block ever waits) writes the
//   exclusive prefix of the token counts over units for the attention
//   kernel's work split.
#include <math.h>

#include "ckv_internal.cuh"

namespace ckv {

constexpr int SCORE_ROWS = 64;      // centres per block (8 warps x 8 rows)
constexpr int SEL_THREADS = 1024;

struct ScoreParams {
    const void* q;
    const float* cent;
    const int32_t* num_comm;
    float* scores;
    int32_t* counter;
    int Hq, Hkv, G, per_head, Cmax;
    float inv_sqrt_d;
};

template <typename T, int D, int GQ>
__global__ void __launch_bounds__(256) score_kernel(ScoreParams p) {
    constexpr int E = D / 16;
    const int u = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4, l16 = lane & 15;
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.counter = 0;
    const int C = p.num_comm[u];
    const int row0 = blockIdx.x * SCORE_ROWS + warp * 8;
    if (row0 >= C) return;

    const int b = u / p.G, g = u - b * p.G;
    const int h0 = p.per_head ? g : g * GQ;
    float qr[GQ][E];
#pragma unroll
    for (int h = 0; h < GQ; ++h)
        load_row_part<T, E>(static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h0 + h) * D + l16 * E, qr[h]);

    float x[4][E];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = row0 + 2 * j + half;
        if (c < C) {
            load_row_part<float, E>(p.cent + ((size_t)u * p.Cmax + c) * D + l16 * E, x[j]);
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) x[j][e] = 0.f;
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float part[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) a = fmaf(qr[h][e], x[j][e], a);
            part[h] = a;
        }
        float s = halfwarp_reduce_heads<GQ>(part, lane);
        s = halfwarp_max_over_heads<GQ>(s);
        const int c = row0 + 2 * j + half;
        if (l16 == 0 && c < C) p.scores[(size_t)u * p.Cmax + c] = s * p.inv_sqrt_d;
    }
}

struct SelectParams {
    const float* scores;
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
    int32_t* counter;
    int U, Cmax, npow_max, S, T_cap, max_tail, tok_cap, budget;
};

__device__ __forceinline__ unsigned long long score_key(float s, int c) {
    unsigned int b = __float_as_uint(s);
    b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)b << 32) | (unsigned long long)(0xffffffffu - (unsigned)c);
}

// In-place inclusive scan of n ints in shared memory; returns the total.
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

__global__ void __launch_bounds__(SEL_THREADS) select_kernel(SelectParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned long long* key = reinterpret_cast<unsigned long long*>(smem);
    int* sz = reinterpret_cast<int*>(key + p.npow_max);
    unsigned* mask = reinterpret_cast<unsigned*>(sz + p.npow_max);
    __shared__ int s_warp[33];
    __shared__ int s_kstar, s_last;

    const int u = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int C = min(p.num_comm[u], p.Cmax);
    int np = 1;
    while (np < C) np <<= 1;

    const float* sc = p.scores + (size_t)u * p.Cmax;
    const int32_t* cn = p.cnt + (size_t)u * p.Cmax;
    for (int i = tid; i < np; i += nt) key[i] = (i < C && cn[i] > 0) ? score_key(sc[i], i) : 0ull;
    for (int i = tid; i < (p.Cmax + 31) / 32; i += nt) mask[i] = 0u;
    if (tid == 0) s_kstar = 0;
    __syncthreads();

    // bitonic sort, descending
    for (int k = 2; k <= np; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int pi = tid; pi < (np >> 1); pi += nt) {
                const int i = ((pi / j) * 2 * j) + (pi % j);
                const int ixj = i + j;
                const unsigned long long a = key[i], bb = key[ixj];
                const bool desc = (i & k) == 0;
                if (desc ? (a < bb) : (a > bb)) {
                    key[i] = bb;
                    key[ixj] = a;
                }
            }
            __syncthreads();
        }
    }

    // sizes in rank order, inclusive prefix, cut
    for (int i = tid; i < np; i += nt) {
        const unsigned long long kk = key[i];
        sz[i] = kk ? cn[0xffffffffu - (unsigned)(kk & 0xffffffffull)] : 0;
    }
    __syncthreads();
    block_scan_inplace(sz, np, s_warp);
    for (int i = tid; i < np; i += nt) {
        const bool in_i = key[i] != 0ull && sz[i] <= p.budget;
        const bool in_n = (i + 1 < np) && key[i + 1] != 0ull && sz[i + 1] <= p.budget;
        if (in_i && !in_n) s_kstar = i + 1;
    }
    __syncthreads();
    int kstar = s_kstar;
    if (kstar == 0 && np > 0 && key[0] != 0ull) kstar = 1;

    int32_t* selc = p.sel_comm + (size_t)u * p.Cmax;
    for (int i = tid; i < kstar; i += nt) {
        const int c = (int)(0xffffffffu - (unsigned)(key[i] & 0xffffffffull));
        selc[i] = c;
        atomicOr(&mask[c >> 5], 1u << (c & 31));
    }
    __syncthreads();

    // build-time member counts in rank order -> exclusive offsets
    const int32_t* of = p.offs + (size_t)u * (p.Cmax + 1);
    for (int i = tid; i < np; i += nt) {
        int v = 0;
        if (i < kstar) {
            const int c = selc[i];
            v = of[c + 1] - of[c];
        }
        sz[i] = v;
    }
    __syncthreads();
    const int nb = block_scan_inplace(sz, np, s_warp);  // inclusive

    int32_t* out = p.sel_tok + (size_t)u * p.tok_cap;
    const int32_t* tk = p.tok + (size_t)u * p.T_cap;
    bool overflow = false;
    for (int i = tid; i < p.S; i += nt) {
        if (i < p.tok_cap) out[i] = i;
        else overflow = true;
    }
    for (int k = warp; k < kstar; k += nw) {
        const int c = selc[k];
        const int len = of[c + 1] - of[c];
        const int dst = p.S + sz[k] - len;
        const int src = of[c];
        for (int i = lane; i < len; i += 32) {
            if (dst + i < p.tok_cap) out[dst + i] = tk[src + i];
            else overflow = true;
        }
    }
    __shared__ int s_nt;
    if (warp == 0) {
        const int tl = min(p.tail_len[u], p.max_tail);
        const int32_t* tt = p.tail_tok + (size_t)u * p.max_tail;
        const int32_t* tc = p.tail_comm + (size_t)u * p.max_tail;
        int base = p.S + nb;
        for (int c0 = 0; c0 < tl; c0 += 32) {
            const int i = c0 + lane;
            bool in = false;
            if (i < tl) {
                const int c = tc[i];
                in = c >= 0 && c < p.Cmax && ((mask[c >> 5] >> (c & 31)) & 1u);
            }
            const unsigned bal = __ballot_sync(FULL, in);
            if (in) {
                const int dst = base + __popc(bal & ((1u << lane) - 1u));
                if (dst < p.tok_cap) out[dst] = tt[i];
                else overflow = true;
            }
            base += __popc(bal);
        }
        if (lane == 0) s_nt = base;
    }
    if (__syncthreads_or(overflow) && tid == 0) atomicOr(p.dev_err, CKV_DEVERR_TOKEN_CAP);

    if (tid == 0) {
        p.n_sel[u] = kstar;
        p.n_tok[u] = min(s_nt, p.tok_cap);
        __threadfence();
        const int t = atomicAdd(p.counter, 1);
        s_last = (t == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        int carry = 0;
        for (int base = 0; base < p.U; base += nt) {
            const int x = (base + tid < p.U) ? __ldcg(p.n_tok + base + tid) : 0;
            int tot;
            const int ex = block_exclusive_scan(x, s_warp, &tot);
            if (base + tid < p.U) p.unit_prefix[base + tid] = carry + ex;
            carry += tot;
        }
        if (tid == 0) {
            p.unit_prefix[p.U] = carry;
            *p.counter = 0;
        }
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

size_t select_ws_bytes(int U, int Cmax) { return align256((size_t)U * Cmax * 4) + 256; }

namespace {
template <typename T, int D, int GQ>
cudaError_t launch_score_t(const ScoreParams& p, int U, cudaStream_t st) {
    dim3 grid((p.Cmax + SCORE_ROWS - 1) / SCORE_ROWS, U);
    score_kernel<T, D, GQ><<<grid, 256, 0, st>>>(p);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_score_select(const CacheView& c, const GraphView& g, const void* q, int budget,
                                const SelView& s, void* ws, cudaStream_t st) {
    const int U = c.B * g.G;
    char* w = static_cast<char*>(ws);
    float* scores = reinterpret_cast<float*>(w);
    int32_t* counter = reinterpret_cast<int32_t*>(w + align256((size_t)U * g.Cmax * 4));

    ScoreParams sp{};
    sp.q = q;
    sp.cent = g.cent;
    sp.num_comm = g.num_comm;
    sp.scores = scores;
    sp.counter = counter;
    sp.Hq = c.Hq;
    sp.Hkv = c.Hkv;
    sp.G = g.G;
    sp.per_head = g.mode == CKV_GRAPH_PER_HEAD;
    sp.Cmax = g.Cmax;
    sp.inv_sqrt_d = 1.0f / sqrtf((float)c.d);

    cudaError_t e = cudaErrorInvalidValue;
#define CKV_SC_CASE(TT, DD, GG) \
    else if (c.d == DD && g.gq == GG) e = launch_score_t<TT, DD, GG>(sp, U, st);
    if (c.dtype == CKV_DTYPE_BF16) {
        if (false) {}
        CKV_SC_CASE(__nv_bfloat16, 128, 1) CKV_SC_CASE(__nv_bfloat16, 128, 2)
        CKV_SC_CASE(__nv_bfloat16, 128, 4) CKV_SC_CASE(__nv_bfloat16, 128, 8)
        CKV_SC_CASE(__nv_bfloat16, 64, 1) CKV_SC_CASE(__nv_bfloat16, 64, 2)
        CKV_SC_CASE(__nv_bfloat16, 64, 4) CKV_SC_CASE(__nv_bfloat16, 64, 8)
    } else {
        if (false) {}
        CKV_SC_CASE(float, 128, 1) CKV_SC_CASE(float, 128, 2)
        CKV_SC_CASE(float, 128, 4) CKV_SC_CASE(float, 128, 8)
        CKV_SC_CASE(float, 64, 1) CKV_SC_CASE(float, 64, 2)
        CKV_SC_CASE(float, 64, 4) CKV_SC_CASE(float, 64, 8)
    }
#undef CKV_SC_CASE
    if (e != cudaSuccess) return e;

    SelectParams pp{};
    pp.scores = scores;
    pp.cnt = g.cnt;
    pp.offs = g.offs;
    pp.tok = g.tok;
    pp.num_comm = g.num_comm;
    pp.tail_tok = g.tail_tok;
    pp.tail_comm = g.tail_comm;
    pp.tail_len = g.tail_len;
    pp.dev_err = g.dev_err;
    pp.sel_comm = s.sel_comm;
    pp.n_sel = s.n_sel;
    pp.sel_tok = s.sel_tok;
    pp.n_tok = s.n_tok;
    pp.unit_prefix = s.unit_prefix;
    pp.counter = counter;
    pp.U = U;
    pp.Cmax = g.Cmax;
    pp.npow_max = next_pow2(g.Cmax);
    pp.S = g.S;
    pp.T_cap = g.T_cap;
    pp.max_tail = g.max_tail;
    pp.tok_cap = s.tok_cap;
    pp.budget = budget;
    const size_t smem = (size_t)pp.npow_max * 12 + ((g.Cmax + 31) / 32) * 4;
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<<<U, SEL_THREADS, smem, st>>>(pp);
    return cudaGetLastError();
}

}  // namespace ckv
