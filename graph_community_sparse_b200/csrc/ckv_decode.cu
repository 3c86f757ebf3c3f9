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
// unnormalised accumulator, top-8 logits) per unit segment into slot w + u,
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

#include "ckv_internal.cuh"

namespace ckv {

constexpr int DEC_WARPS = 4;
constexpr int TOK_PER_IT = 8;
constexpr float RESCALE_THRESH = 8.0f;
constexpr int MERGE_CHUNK = 128;  // slots whose weights are staged in shared memory at once

template <int GQ> struct Stages { static constexpr int v = GQ == 1 ? 2 : 3; };
template <int GQ> struct MinBlocks { static constexpr int v = GQ == 1 ? 6 : (GQ == 2 ? 5 : (GQ == 4 ? 4 : 2)); };

template <typename T, int D>
struct RowGeom {
    static constexpr int E = D / 16;
    static constexpr int PART = E * ElemBytes<T>::v;
    static constexpr int ROW = 16 * PART;
    static constexpr int TILE = TOK_PER_IT * ROW;
};

template <typename T, int D, int GQ>
struct DecSmem {
    static constexpr int PBUF = TOK_PER_IT * GQ * 4;
    static constexpr int WARP = Stages<GQ>::v * 2 * RowGeom<T, D>::TILE + ((PBUF + 127) / 128) * 128;
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
    float scale_log2;
    DecodeWs ws;
    int W;                  // warps in the grid
    int want_nbr;
    float* out;
    int32_t* nbr8;
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

// Insert (cv, cpos) into the warp's sorted top-8 list held by lanes 0..7
// (value descending, position ascending).
__device__ __forceinline__ void top8_insert(float cv, int cpos, float& tv, int& tp, float& thr, int lane) {
    const bool above = lane < 8 && (tv > cv || (tv == cv && tp < cpos));
    const int k = __popc(__ballot_sync(FULL, above));
    if (k < 8) {
        const float uv = __shfl_up_sync(FULL, tv, 1);
        const int up = __shfl_up_sync(FULL, tp, 1);
        if (lane < 8 && lane > k) {
            tv = uv;
            tp = up;
        }
        if (lane == k) {
            tv = cv;
            tp = cpos;
        }
        thr = __shfl_sync(FULL, tv, 7);
    }
}

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
    float* pbuf = reinterpret_cast<float*>(wsm + NS * 2 * TILE);

    int win_cur = 0, win_nxt = 0;
    if constexpr (!DENSE) {
        win_cur = (lane < n) ? __ldg(toks + lo + lane) : 0;
        win_nxt = (32 + lane < n) ? __ldg(toks + lo + 32 + lane) : 0;
    }

    int stage_in = 0;  // ring slot the next issue() fills
    auto issue = [&](int it) {
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
            const bool valid = i < n;
            int pos;
            if constexpr (DENSE) {
                pos = valid ? lo + i : 0;
            } else {
                const int pp = __shfl_sync(FULL, win_cur, ((it & 3) << 3) + 2 * j + half);
                pos = valid ? pp : 0;
            }
            const int r = 2 * j + half;
            cp_async_part<PART>(kt + r * ROW + l16 * PART, Kb + (int64_t)pos * p.st, valid);
            cp_async_part<PART>(vt + r * ROW + l16 * PART, Vb + (int64_t)pos * p.st, valid);
        }
        cp_async_commit();
    };

#pragma unroll
    for (int s = 0; s < NS - 1; ++s) {
        if (s < nit) issue(s);
        else cp_async_commit();
    }

    float m_run = -INFINITY, l_run = 0.f;
    float acc[GQ][E];
#pragma unroll
    for (int h = 0; h < GQ; ++h)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
    float tv = -INFINITY, thr = -INFINITY;
    int tp = 0x7fffffff;

    int stage_out = 0;  // ring slot computed in this iteration
    for (int it = 0; it < nit; ++it) {
        __syncwarp();
        if (it + NS - 1 < nit) issue(it + NS - 1);
        else cp_async_commit();
        cp_async_wait<NS - 1>();

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
            if (it * TOK_PER_IT + 2 * j + half >= n) s[j] = -INFINITY;
        }

        float mx = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
        const bool need = mx > m_run + RESCALE_THRESH;
        if (__any_sync(FULL, need)) {
            const float m_new = need ? mx : m_run;
            const float f = (m_run == -INFINITY) ? 0.f : exp2f(m_run - m_new);
            l_run *= f;
            m_run = m_new;
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                const float fh = __shfl_sync(FULL, f, (lane & 16) | (h << (4 - LG)));
#pragma unroll
                for (int e = 0; e < E; ++e) acc[h][e] *= fh;
            }
        }

        float pj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) pj[j] = exp2f(s[j] - m_run);
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

        if constexpr (!DENSE) {
            if (p.want_nbr) {
                bool f[4];
                bool anyf = false;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = it * TOK_PER_IT + 2 * j + half;
                    f[j] = (i < n) && (lo + i >= p.S) && (s[j] >= thr);
                    anyf |= f[j];
                }
                if (__any_sync(FULL, anyf)) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const unsigned bj = __ballot_sync(FULL, f[j]);
                        if (bj) {
                            const float lam = halfwarp_max_over_heads<GQ>(s[j]);
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                if (bj & (0xffffu << (16 * hh))) {
                                    const float cv = __shfl_sync(FULL, lam, 16 * hh);
                                    const int cpos = __ldg(toks + lo + it * TOK_PER_IT + 2 * j + hh);
                                    top8_insert(cv, cpos, tv, tp, thr, lane);
                                }
                            }
                        }
                    }
                }
            }
        }
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
    if constexpr (!DENSE) {
        if (p.want_nbr && lane < 8) {
            ws.tv[(size_t)slot * 8 + lane] = tv;
            ws.tp[(size_t)slot * 8 + lane] = (tv == -INFINITY) ? -1 : tp;
        }
    }
}

template <typename T, int D, int GQ, bool DENSE>
__global__ void __launch_bounds__(DEC_WARPS * 32, MinBlocks<GQ>::v) decode_main(DecodeParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
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
            const int x = p.n_tok[i];
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
    const int per = (total + p.W - 1) / p.W;
    const int start = w * per;
    if (start >= total) return;
    const int end = min(start + per, total);

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
        if (lo < hi) process_segment<T, D, GQ, DENSE>(p, u, lo - ubeg, hi - ubeg, w + u, wsm, lane);
        if (end <= uend || u + 1 >= p.U) break;
        ++u;
    }
}

// One block per unit: threads 0..D-1 own one output dimension each (all the
// unit's heads); the extra warp merges the top-8 neighbour lists.  Slots are
// combined in slot order, MERGE_CHUNK at a time, with every load of a chunk
// issued before any is used.
template <int D, int GQ, bool DENSE>
__global__ void __launch_bounds__(D + 32) decode_merge(DecodeParams p) {
    __shared__ float s_f[MERGE_CHUNK][GQ];
    __shared__ float s_red[(D + 32) / 32][GQ];
    __shared__ float s_M[GQ];
    // wait until the attention kernel's partials are complete and visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int u = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
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
    if (uend <= ubeg) {
        for (int i = t; i < GQ * D; i += blockDim.x) outu[i] = 0.f;
        if (!DENSE && p.want_nbr && t < 8) p.nbr8[(size_t)u * 8 + t] = -1;
        return;
    }
    const int per = (total + p.W - 1) / p.W;
    const int wf = ubeg / per, nslots = (uend - 1) / per - wf + 1;
    const size_t s0 = (size_t)wf + u;
    const DecodeWs& ws = p.ws;

    if (!DENSE && p.want_nbr && warp == D / 32) {
        // candidates: 8 per slot; each lane keeps its best 8 in registers
        // (value desc, position asc), then 8 warp-wide rounds pick the winners
        float cv[8];
        int cp[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            cv[r] = -INFINITY;
            cp[r] = 0x7fffffff;
        }
        for (int i = lane; i < nslots * 8; i += 32) {
            const size_t sl = (s0 + (i >> 3)) * 8 + (i & 7);
            float v = ws.tv[sl];
            int q = ws.tp[sl];
            if (q < 0) continue;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const bool better = (v > cv[r]) || (v == cv[r] && q < cp[r]);
                const float v2 = better ? cv[r] : v;
                const int q2 = better ? cp[r] : q;
                if (better) {
                    cv[r] = v;
                    cp[r] = q;
                }
                v = v2;
                q = q2;
            }
        }
        int head = 0;  // this lane's best remaining candidate
        for (int r = 0; r < 8; ++r) {
            float bv = -INFINITY;
            int bp = 0x7fffffff;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k == head) {
                    bv = cv[k];
                    bp = cp[k];
                }
            float wv = bv;
            int wp = bp;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(FULL, wv, o);
                const int op = __shfl_xor_sync(FULL, wp, o);
                if (ov > wv || (ov == wv && op < wp)) {
                    wv = ov;
                    wp = op;
                }
            }
            const bool valid = wp != 0x7fffffff;
            if (lane == 0) p.nbr8[(size_t)u * 8 + r] = valid ? wp : -1;
            if (valid && bp == wp) ++head;  // positions are unique: only the owner advances
        }
    }

    // running max per head over all slots
    float M[GQ];
#pragma unroll
    for (int h = 0; h < GQ; ++h) M[h] = -INFINITY;
    for (int sl = t; sl < nslots; sl += blockDim.x)
#pragma unroll
        for (int h = 0; h < GQ; ++h) M[h] = fmaxf(M[h], ws.m[(s0 + sl) * GQ + h]);
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M[h] = fmaxf(M[h], __shfl_xor_sync(FULL, M[h], o));
        if (lane == 0) s_red[warp][h] = M[h];
    }
    __syncthreads();
    if (t < GQ) {
        float m = -INFINITY;
        for (int w2 = 0; w2 < (int)(blockDim.x >> 5); ++w2) m = fmaxf(m, s_red[w2][t]);
        s_M[t] = m;
    }
    __syncthreads();

    float A[GQ], Lp[GQ];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        A[h] = 0.f;
        Lp[h] = 0.f;
    }
    for (int c0 = 0; c0 < nslots; c0 += MERGE_CHUNK) {
        const int cnt = min(MERGE_CHUNK, nslots - c0);
        for (int i = t; i < cnt; i += blockDim.x) {
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                const size_t sl = (s0 + c0 + i) * GQ + h;
                const float f = exp2f(ws.m[sl] - s_M[h]);
                s_f[i][h] = f;
                Lp[h] = fmaf(ws.l[sl], f, Lp[h]);
            }
        }
        __syncthreads();
        if (t < D) {
            int j = 0;
            for (; j + 8 <= cnt; j += 8) {
                float x[8][GQ];
#pragma unroll
                for (int r = 0; r < 8; ++r)
#pragma unroll
                    for (int h = 0; h < GQ; ++h) x[r][h] = ws.acc[((s0 + c0 + j + r) * GQ + h) * D + t];
#pragma unroll
                for (int r = 0; r < 8; ++r)
#pragma unroll
                    for (int h = 0; h < GQ; ++h) A[h] = fmaf(x[r][h], s_f[j + r][h], A[h]);
            }
            for (; j < cnt; ++j)
#pragma unroll
                for (int h = 0; h < GQ; ++h) A[h] = fmaf(ws.acc[((s0 + c0 + j) * GQ + h) * D + t], s_f[j][h], A[h]);
        }
        __syncthreads();
    }
    // sum of the weights per head
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) Lp[h] += __shfl_xor_sync(FULL, Lp[h], o);
        if (lane == 0) s_red[warp][h] = Lp[h];
    }
    __syncthreads();
    if (t < D) {
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float L = 0.f;
            for (int w2 = 0; w2 < (int)(blockDim.x >> 5); ++w2) L += s_red[w2][h];
            outu[h * D + t] = A[h] / L;
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

size_t decode_ws_bytes(int U, int gq, int d) {
    const size_t slots = (size_t)MAX_DECODE_WARPS + U;
    return align256(slots * gq * 4) * 2 + align256(slots * gq * d * 4) + align256(slots * 8 * 4) * 2;
}

DecodeWs carve_decode_ws(void* ws, int U, int gq, int d) {
    const size_t slots = (size_t)MAX_DECODE_WARPS + U;
    char* p = static_cast<char*>(ws);
    DecodeWs w;
    w.m = reinterpret_cast<float*>(p);
    p += align256(slots * gq * 4);
    w.l = reinterpret_cast<float*>(p);
    p += align256(slots * gq * 4);
    w.acc = reinterpret_cast<float*>(p);
    p += align256(slots * gq * d * 4);
    w.tv = reinterpret_cast<float*>(p);
    p += align256(slots * 8 * 4);
    w.tp = reinterpret_cast<int32_t*>(p);
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
    kern<<<blocks, DEC_WARPS * 32, smem, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.U);
    cfg.blockDim = dim3(D + 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_merge<D, GQ, DENSE>, p);
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
                                 const void* q, float* out, int32_t* nbr8, void* ws, cudaStream_t st) {
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
    p.unit_prefix = s.unit_prefix;
    p.n_tok = s.n_tok;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)c.d);
    p.ws = carve_decode_ws(ws, p.U, g.gq, c.d);
    p.want_nbr = nbr8 != nullptr;
    p.out = out;
    p.nbr8 = nbr8;
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
    p.ws = carve_decode_ws(ws, p.U, gq, c.d);
    p.out = out;
    return dispatch<true>(c, gq, p, st);
}

}  // namespace ckv
