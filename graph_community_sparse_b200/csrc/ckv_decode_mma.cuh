// Attention over one warp's segment with the tensor cores (mma.sync
// m16n8k16, bf16 operands, fp32 accumulators), for bf16 caches whose graphs
// serve several query heads (GQA groups).  Included by ckv_decode.cu inside
// namespace ckv, after DecodeParams, unit_heads and exp2_approx.
//
// Per iteration a warp takes 16 selected tokens: their K and V rows are
// staged by cp.async into a ring of MMA_STAGES tiles (16-byte chunks XOR-
// swizzled by row, so ldmatrix reads them without bank conflicts).  The
// graph's heads are the rows of the A operand (padded to 16 with zeros):
//   S = Q K^T   (16 x 16 tokens; K is read with ldmatrix as the B operand)
//   O += P V    (P from S's accumulators, V read with ldmatrix.trans)
// q is used unscaled (bf16, exact) and log2(e)/sqrt(d) multiplies the fp32
// scores.  P is split into two bf16 terms, P = P_hi + P_lo with
// P_lo = bf16(P - P_hi), so P V keeps about 16 bits of P instead of 8.
// The softmax bookkeeping (running max per head raised lazily, sum, the
// unnormalised accumulator) and the partial written per segment are those
// of the scalar path, so the merge kernel is shared.
#pragma once

constexpr int MMA_TOK = 16;     // tokens per iteration
constexpr int MMA_STAGES = 3;   // ring depth (iterations)

template <int D>
struct MmaGeom {
    static_assert(MMA_STAGES * 2 * MMA_TOK * D * 2 == DecSmem<__nv_bfloat16, D, 2>::MMA, "ring size");
    static constexpr int ROW = D * 2;            // bytes per bf16 row
    static constexpr int CH = D / 8;             // 16-byte chunks per row
    static constexpr int TILE = MMA_TOK * ROW;   // bytes of a K (or V) tile
    static constexpr int WARP = MMA_STAGES * 2 * TILE;
    static constexpr int KS = D / 16;            // k-steps of Q K^T
    static constexpr int NT = D / 8;             // n-tiles of P V
    static_assert(CH >= 8, "the swizzle permutes 8 chunks");
};

__device__ __forceinline__ unsigned smem_addr(const void* p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
// Byte offset of 16-byte chunk c of row r in a tile with ROW-byte rows.
__device__ __forceinline__ int swz(int r, int c, int row_bytes) { return r * row_bytes + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ void ldsm_x4(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// d += a b for one m16n8k16 tile; a2 = a3 = 0 (rows 8..15 of A are padding)
__device__ __forceinline__ void mma_rows8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a1), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// One warp, one unit, list positions [lo, hi) (cache positions when dense);
// thread lane = 4 g + tq holds head row g (g < GQ real) of the accumulators.
template <int D, int GQ, bool DENSE>
__device__ __forceinline__ void process_segment_mma(const DecodeParams& p, int u, int lo, int hi, int slot,
                                                    unsigned char* wsm, int lane) {
    using MG = MmaGeom<D>;
    constexpr int NS = MMA_STAGES;
    const int g = lane >> 2, tq = lane & 3;
    const int64_t st = p.st;
    const bool want_nbr = !DENSE && p.want_nbr;

    int b, kvh, h0;
    unit_heads(p, u, GQ, DENSE, b, kvh, h0);
    const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(p.k) + b * p.sb + kvh * p.sh;
    const __nv_bfloat16* Vb = static_cast<const __nv_bfloat16*>(p.v) + b * p.sb + kvh * p.sh;
    const int32_t* toks = DENSE ? nullptr : p.sel_tok + (size_t)u * p.tok_cap;

    // A fragments of Q (rows = heads): a0a1 = dims kk*16 + 2tq.., a2a3 (stored
    // as qa[kk][1]) = dims kk*16 + 8 + 2tq..; zero rows past the group
    uint32_t qa[MG::KS][2];
    {
        const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + h0 + min(g, GQ - 1)) * D;
#pragma unroll
        for (int kk = 0; kk < MG::KS; ++kk) {
            const uint32_t x0 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * tq);
            const uint32_t x1 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * tq);
            qa[kk][0] = g < GQ ? x0 : 0u;
            qa[kk][1] = g < GQ ? x1 : 0u;
        }
    }

    const int n = hi - lo;
    const int nit = (n + MMA_TOK - 1) / MMA_TOK;
    const int nfull = n / MMA_TOK;

    // index window: 32 list positions = 2 iterations, the next window loaded
    // one window ahead
    int win_cur = 0, win_nxt = 0;
    if constexpr (!DENSE) {
        win_cur = (lane < n) ? __ldg(toks + lo + lane) : 0;
        win_nxt = (32 + lane < n) ? __ldg(toks + lo + 32 + lane) : 0;
    }

    int stage_in = 0;
    auto issue = [&](int it) {
        if (it < nit) {
            unsigned char* kt = wsm + stage_in * 2 * MG::TILE;
            unsigned char* vt = kt + MG::TILE;
            if constexpr (!DENSE) {
                if (it > 0 && (it & 1) == 0) {
                    win_cur = win_nxt;
                    const int nx = (it + 2) * MMA_TOK + lane;
                    win_nxt = (nx < n) ? __ldg(toks + lo + nx) : 0;
                }
            }
            const int rem = n - it * MMA_TOK;  // valid rows of this tile
#pragma unroll
            for (int i = 0; i < MMA_TOK * MG::CH / 32; ++i) {
                const int idx = i * 32 + lane;
                const int r = idx / MG::CH, c = idx % MG::CH;
                int pos;
                if constexpr (DENSE) {
                    pos = lo + it * MMA_TOK + r;
                } else {
                    pos = __shfl_sync(FULL, win_cur, ((it & 1) << 4) + r);
                    pos = checked_index(pos, 0, p.T_cap, p.dev_err, 0);
                }
                const bool valid = r < rem;
                pos = valid ? pos : 0;
                const int64_t off = (int64_t)pos * st + c * 8;
                cp_async_16(kt + swz(r, c, MG::ROW), Kb + off, valid);
                cp_async_16(vt + swz(r, c, MG::ROW), Vb + off, valid);
            }
        }
        stage_in = (stage_in + 1 == NS) ? 0 : stage_in + 1;
        cp_async_commit();
    };
#pragma unroll
    for (int s = 0; s < NS - 1; ++s) issue(s);

    float m_run = -INFINITY, l_run = 0.f;
    float o[MG::NT][4];
#pragma unroll
    for (int j = 0; j < MG::NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[j][e] = 0.f;
    float* lamu = DENSE ? nullptr : p.ws.lam + (size_t)u * p.ws.lam_cap;
    int stage_out = 0;

    // ldmatrix lane addresses (before the tile base): for S, matrices
    // (tokens 0-7 | 8-15) x (chunk 2kk | 2kk+1); for P V, matrices
    // (tokens 0-7 | 8-15) x (chunk 2j | 2j+1), transposed
    const int mi = lane >> 3, mr = lane & 7;
    const int s_tok = (mi >> 1) * 8 + mr, s_chk = mi & 1;
    const int v_tok = (mi & 1) * 8 + mr, v_chk = mi >> 1;

    for (int it = 0; it < nit; ++it) {
        __syncwarp();  // every lane is done reading the slot refilled next
        issue(it + NS - 1);
        cp_async_wait<NS - 1>();
        __syncwarp();  // the tile's chunks copied by every lane are visible
        const unsigned char* kt = wsm + stage_out * 2 * MG::TILE;
        const unsigned char* vt = kt + MG::TILE;
        stage_out = (stage_out + 1 == NS) ? 0 : stage_out + 1;
        const unsigned kbase = smem_addr(kt), vbase = smem_addr(vt);

        // S = Q K^T: s[t] covers tokens 8t + 2tq + {0, 1} of head row g
        float s[2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[t][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < MG::KS; ++kk) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + swz(s_tok, 2 * kk + s_chk, MG::ROW), b0, b1, b2, b3);
            mma_rows8(s[0], qa[kk][0], qa[kk][1], b0, b1);
            mma_rows8(s[1], qa[kk][0], qa[kk][1], b2, b3);
        }
        const bool full = it < nfull;
        float x[4];  // this thread's 4 scores (log2 units), masked
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = it * MMA_TOK + 8 * t + 2 * tq + e;
                x[2 * t + e] = (full || i < n) ? s[t][e] * p.scale_log2 : -INFINITY;
            }

        if (want_nbr) {
            // graph logit of each token: max over the group's heads (rows)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float v = g < GQ ? x[k] : -INFINITY;
                v = fmaxf(v, __shfl_xor_sync(FULL, v, 4));
                v = fmaxf(v, __shfl_xor_sync(FULL, v, 8));
                v = fmaxf(v, __shfl_xor_sync(FULL, v, 16));
                const int i = it * MMA_TOK + 8 * (k >> 1) + 2 * tq + (k & 1);
                if (g == 0 && (full || i < n)) lamu[lo + i] = v;
            }
        }

        // online softmax for head row g (the 4 lanes of a quad hold its 16 tokens)
        float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
        const bool need = mx > m_run + RESCALE_THRESH;
        if (__any_sync(FULL, need)) {
            const float m_new = need ? mx : m_run;
            const float f = (m_run == -INFINITY) ? 0.f : exp2_approx(m_run - m_new);
            l_run *= f;
            m_run = m_new;
#pragma unroll
            for (int j = 0; j < MG::NT; ++j) {
                o[j][0] *= f;
                o[j][1] *= f;
            }
        }
        float pr[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) pr[k] = exp2_approx(x[k] - m_run);
        l_run += (pr[0] + pr[1]) + (pr[2] + pr[3]);

        // A fragments of P (rows = heads, k = tokens): a0a1 = tokens 2tq..,
        // a2a3 = tokens 8 + 2tq..; each as a bf16 high part and remainder
        const uint32_t ph0 = pack_bf16x2(pr[0], pr[1]), ph1 = pack_bf16x2(pr[2], pr[3]);
        const __nv_bfloat162 hb0 = *reinterpret_cast<const __nv_bfloat162*>(&ph0);
        const __nv_bfloat162 hb1 = *reinterpret_cast<const __nv_bfloat162*>(&ph1);
        const uint32_t pl0 = pack_bf16x2(pr[0] - __low2float(hb0), pr[1] - __high2float(hb0));
        const uint32_t pl1 = pack_bf16x2(pr[2] - __low2float(hb1), pr[3] - __high2float(hb1));

        // O += P V, two output n-tiles (16 dims) per ldmatrix
#pragma unroll
        for (int j = 0; j < MG::NT / 2; ++j) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vbase + swz(v_tok, 2 * j + v_chk, MG::ROW), b0, b1, b2, b3);
            mma_rows8(o[2 * j], ph0, ph1, b0, b1);
            mma_rows8(o[2 * j], pl0, pl1, b0, b1);
            mma_rows8(o[2 * j + 1], ph0, ph1, b2, b3);
            mma_rows8(o[2 * j + 1], pl0, pl1, b2, b3);
        }
    }
    cp_async_wait<0>();

    l_run += __shfl_xor_sync(FULL, l_run, 1);
    l_run += __shfl_xor_sync(FULL, l_run, 2);
    if (g < GQ) {
        const DecodeWs& ws = p.ws;
        float* dst = ws.acc + ((size_t)slot * GQ + g) * D + 2 * tq;
#pragma unroll
        for (int j = 0; j < MG::NT; ++j) *reinterpret_cast<float2*>(dst + 8 * j) = make_float2(o[j][0], o[j][1]);
        if (tq == 0) {
            ws.m[(size_t)slot * GQ + g] = m_run;
            ws.l[(size_t)slot * GQ + g] = l_run;
        }
    }
}
