// Community state build for sm_100a: CSR of the members and centroid means.
//
// Every community gets a centre (CommunityKV, rit.work summary, section "A
// graph of tokens replaces re-clustering", paragraph 4); the sink tokens are
// kept out of the graph (paragraph 3).  The partition itself is an
// input (labels).  Runs once per sequence and layer, not per decode step.
//
// Stable counting sort of positions by label, in three passes:
//   build_hist    per (unit, 4096-position chunk): validate labels, copy them
//                 to comm_of, per-chunk histogram in shared memory;
//   build_scan    per unit: CSR offsets, counts, and each chunk's starting
//                 cursor for every community;
//   build_scatter per (unit, chunk), one warp walking the chunk in position
//                 order (match_any gives the rank among equal labels), so
//                 members end up sorted by (community, position).
// build_mean: one block per (unit, community); 8 warps sum member rows in a
//   fixed interleaving in fp64 and combine in warp order: deterministic, and
//   the fp32 centre is the correctly rounded mean up to fp64 summation error;
//   the row's int8 scoring copy (scale and codes) is written with it.
#include "ckv_internal.cuh"

namespace ckv {

struct BuildParams {
    const void* k;
    int64_t sb, sh, st;
    const int32_t* labels;
    int64_t lstride;
    int T, T_cap, S, Cmax, G, Hq, Hkv, per_head, nchunks;
    int32_t* counts;  // [U, nchunks, Cmax]
    int32_t* comm_of;
    int32_t* offs;
    int32_t* tok;
    int32_t* cnt;
    float* cent;
    int8_t* cent_q;
    float* cent_qs;
    int32_t* num_comm;
    int32_t* tail_len;
    int32_t* dev_err;
};

__global__ void __launch_bounds__(256) build_hist(BuildParams p) {
    extern __shared__ int hist[];
    const int u = blockIdx.y, chunk = blockIdx.x;
    for (int c = threadIdx.x; c < p.Cmax; c += blockDim.x) hist[c] = 0;
    __syncthreads();
    const int t0 = chunk * BUILD_CHUNK, t1 = min(t0 + BUILD_CHUNK, p.T_cap);
    int err = 0;
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        int lab = -1;
        if (t < p.T) {
            lab = p.labels[(size_t)u * p.lstride + t];
            if (t < p.S) {
                if (lab != -1) err |= CKV_DEVERR_SINK_LABEL;
                lab = -1;
            } else if (lab < 0 || lab >= p.Cmax) {
                err |= CKV_DEVERR_LABEL_RANGE;
                lab = -1;
            } else {
                atomicAdd(&hist[lab], 1);
            }
        }
        p.comm_of[(size_t)u * p.T_cap + t] = lab;
    }
    if (err) atomicOr(p.dev_err, err);
    __syncthreads();
    int32_t* dst = p.counts + ((size_t)u * p.nchunks + chunk) * p.Cmax;
    for (int c = threadIdx.x; c < p.Cmax; c += blockDim.x) dst[c] = hist[c];
}

__global__ void __launch_bounds__(1024) build_scan(BuildParams p) {
    __shared__ int s_warp[33];
    __shared__ int s_maxc;
    const int u = blockIdx.x;
    if (threadIdx.x == 0) s_maxc = -1;
    __syncthreads();
    int32_t* base = p.counts + (size_t)u * p.nchunks * p.Cmax;
    int carry = 0;
    for (int c0 = 0; c0 < p.Cmax; c0 += blockDim.x) {
        const int c = c0 + threadIdx.x;
        int tot = 0;
        if (c < p.Cmax)
            for (int k = 0; k < p.nchunks; ++k) tot += base[(size_t)k * p.Cmax + c];
        int all;
        const int ex = block_exclusive_scan(tot, s_warp, &all);
        if (c < p.Cmax) {
            int run = carry + ex;
            p.offs[(size_t)u * (p.Cmax + 1) + c] = run;
            p.cnt[(size_t)u * p.Cmax + c] = tot;
            for (int k = 0; k < p.nchunks; ++k) {
                const int v = base[(size_t)k * p.Cmax + c];
                base[(size_t)k * p.Cmax + c] = run;
                run += v;
            }
            if (tot > 0) atomicMax(&s_maxc, c);
        }
        carry += all;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        p.offs[(size_t)u * (p.Cmax + 1) + p.Cmax] = carry;
        p.num_comm[u] = s_maxc + 1;
        p.tail_len[u] = 0;
    }
}

__global__ void __launch_bounds__(32) build_scatter(BuildParams p) {
    extern __shared__ int cur[];
    const int u = blockIdx.y, chunk = blockIdx.x, lane = threadIdx.x;
    const int32_t* src = p.counts + ((size_t)u * p.nchunks + chunk) * p.Cmax;
    for (int c = lane; c < p.Cmax; c += 32) cur[c] = src[c];
    __syncwarp();
    const int t0 = chunk * BUILD_CHUNK, t1 = min(t0 + BUILD_CHUNK, p.T);
    const unsigned lt = (1u << lane) - 1u;
    for (int tb = t0; tb < t1; tb += 32) {
        const int t = tb + lane;
        const int lab = (t < t1 && t >= p.S) ? p.comm_of[(size_t)u * p.T_cap + t] : -1;
        const bool valid = lab >= 0;
        const unsigned peers = __match_any_sync(FULL, valid ? lab : -1 - lane);
        const int rank = __popc(peers & lt);
        const int basepos = valid ? cur[lab] : 0;
        __syncwarp();
        if (valid && rank == 0) cur[lab] = basepos + __popc(peers);
        __syncwarp();
        if (valid) p.tok[(size_t)u * p.T_cap + basepos + rank] = t;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) build_mean(BuildParams p) {
    constexpr int E = D / 32;
    __shared__ double part[8][D];
    const int c = blockIdx.x, u = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = u / p.G, g = u - b * p.G;
    const int kvh = p.per_head ? g / (p.Hq / p.Hkv) : g;
    const int beg = p.offs[(size_t)u * (p.Cmax + 1) + c];
    const int n = p.offs[(size_t)u * (p.Cmax + 1) + c + 1] - beg;
    const T* Kb = static_cast<const T*>(p.k) + b * p.sb + kvh * p.sh + lane * E;
    const int32_t* tk = p.tok + (size_t)u * p.T_cap + beg;
    double acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.0;
    int i = warp;
    for (; i + 24 < n; i += 32) {
        int t[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) t[r] = tk[i + 8 * r];
        T x[4][E];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int e = 0; e < E; ++e) x[r][e] = Kb[(int64_t)t[r] * p.st + e];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] += (double)to_f32(x[r][e]);
    }
    for (; i < n; i += 8) {
        const int t = tk[i];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += (double)to_f32(Kb[(int64_t)t * p.st + e]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) part[warp][lane * E + e] = acc[e];
    __syncthreads();
    float m = 0.f;
    if (threadIdx.x < D) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += part[w][threadIdx.x];
        m = n > 0 ? (float)(s / (double)n) : 0.f;
        p.cent[((size_t)u * p.Cmax + c) * D + threadIdx.x] = m;
    }
    // the int8 scoring copy: the row's scale from its largest magnitude
    __shared__ float s_amax[8];
    float a = fabsf(m);  // 0 on the threads past D
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, o));
    if (lane == 0) s_amax[warp] = a;
    __syncthreads();
    float amax = s_amax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, s_amax[w]);
    const float sc = q8_scale(amax), rc = q8_recip(amax);
    if (threadIdx.x < D) p.cent_q[((size_t)u * p.Cmax + c) * D + threadIdx.x] = (int8_t)q8_code(m, rc);
    if (threadIdx.x == 0) p.cent_qs[(size_t)u * p.Cmax + c] = sc;
}

size_t build_ws_bytes(int U, int Cmax, int T_cap) {
    const int nchunks = (T_cap + BUILD_CHUNK - 1) / BUILD_CHUNK;
    return align256((size_t)U * nchunks * Cmax * 4);
}

cudaError_t launch_build(const CacheView& c, const GraphView& g, const int32_t* labels,
                         int64_t labels_stride, int T, void* ws, cudaStream_t st) {
    BuildParams p{};
    p.k = c.k;
    p.sb = c.sb;
    p.sh = c.sh;
    p.st = c.st;
    p.labels = labels;
    p.lstride = labels_stride;
    p.T = T;
    p.T_cap = g.T_cap;
    p.S = g.S;
    p.Cmax = g.Cmax;
    p.G = g.G;
    p.Hq = c.Hq;
    p.Hkv = c.Hkv;
    p.per_head = g.mode == CKV_GRAPH_PER_HEAD;
    p.nchunks = (g.T_cap + BUILD_CHUNK - 1) / BUILD_CHUNK;
    p.counts = static_cast<int32_t*>(ws);
    p.comm_of = g.comm_of;
    p.offs = g.offs;
    p.tok = g.tok;
    p.cnt = g.cnt;
    p.cent = g.cent;
    p.cent_q = g.cent_q;
    p.cent_qs = g.cent_qs;
    p.num_comm = g.num_comm;
    p.tail_len = g.tail_len;
    p.dev_err = g.dev_err;
    const int U = c.B * g.G;
    const size_t hsm = (size_t)g.Cmax * 4;
    static LaunchCache lc_hist, lc_scatter;
    cudaError_t e = prepare_launch(build_hist, lc_hist, hsm, 256, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    e = prepare_launch(build_scatter, lc_scatter, hsm, 32, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    const bool timed = timing_enabled();  // the four build kernels as one
    if (timed && (e = timing_mark(KK_BUILD, true, st)) != cudaSuccess) return e;
    build_hist<<<dim3(p.nchunks, U), 256, hsm, st>>>(p);
    build_scan<<<U, 1024, 0, st>>>(p);
    build_scatter<<<dim3(p.nchunks, U), 32, hsm, st>>>(p);
    const dim3 mg(g.Cmax, U);
    if (c.dtype == CKV_DTYPE_BF16) {
        if (c.d == 128) build_mean<__nv_bfloat16, 128><<<mg, 256, 0, st>>>(p);
        else build_mean<__nv_bfloat16, 64><<<mg, 256, 0, st>>>(p);
    } else {
        if (c.d == 128) build_mean<float, 128><<<mg, 256, 0, st>>>(p);
        else build_mean<float, 64><<<mg, 256, 0, st>>>(p);
    }
    e = cudaGetLastError();
    if (timed && e == cudaSuccess) e = timing_mark(KK_BUILD, false, st);
    return e;
}

}  // namespace ckv
