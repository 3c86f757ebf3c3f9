// Internal declarations and device helpers shared by the libckv kernels.
#pragma once

#include <cuda_runtime.h>
#include <utility>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ckv.h"

namespace ckv {

constexpr unsigned FULL = 0xffffffffu;
constexpr int MAX_UNITS = 8192;      // B * G
constexpr int MAX_CMAX = 8192;       // communities per graph
constexpr int MAX_DECODE_WARPS = 8192;
constexpr int BUILD_CHUNK = 4096;    // positions per histogram / scatter block

// ---------------------------------------------------------------------------
// element access: a lane owns E = D/16 consecutive elements of a row
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T> struct ElemBytes;
template <> struct ElemBytes<float> { static constexpr int v = 4; };
template <> struct ElemBytes<__nv_bfloat16> { static constexpr int v = 2; };

// Convert E elements at a (shared or global) address to fp32.  Generic loads.
template <typename T, int E>
__device__ __forceinline__ void load_row_part(const T* p, float (&x)[E]);

template <>
__device__ __forceinline__ void load_row_part<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 w = *reinterpret_cast<const uint4*>(p);
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
template <>
__device__ __forceinline__ void load_row_part<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&x)[4]) {
    uint2 w = *reinterpret_cast<const uint2*>(p);
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
}
template <>
__device__ __forceinline__ void load_row_part<float, 8>(const float* p, float (&x)[8]) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <>
__device__ __forceinline__ void load_row_part<float, 4>(const float* p, float (&x)[4]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// ---------------------------------------------------------------------------
// Debug builds (CKV_DEBUG) check every index that a caller's array feeds to a
// kernel before using it; a bad one sets CKV_DEVERR_INDEX in the error word
// and is replaced by a harmless value.  Release builds compile the checks out.
// ---------------------------------------------------------------------------
#ifdef CKV_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
// i if lo <= i < hi; otherwise (debug builds) `fallback`, with the error bit set
__device__ __forceinline__ int checked_index(int i, int lo, int hi, int32_t* err, int fallback) {
    if constexpr (kDebugChecks) {
        if (i < lo || i >= hi) {
            if (err) atomicOr(err, CKV_DEVERR_INDEX);
            return fallback;
        }
    }
    return i;
}

// ---------------------------------------------------------------------------
// The int8 scoring copy of a centre row: scale s = max_i |c_i| / 127 and code
// round-half-even(c_i * r) with r = 127 / max_i |c_i| (both divisions IEEE,
// the product fp32; 0 for an all-zero row).  c_i r is within 127 * 2^-23 of
// c_i / s, so |c_i - s code_i| <= s (1/2 + 2^-16).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float q8_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f; }
__device__ __forceinline__ float q8_recip(float amax) { return amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f; }
__device__ __forceinline__ int q8_code(float c, float r) {
    return max(-127, min(127, __float2int_rn(c * r)));
}

// ---------------------------------------------------------------------------
// cp.async (global -> shared, L2 only); size 0 means zero-fill, nothing read
// ---------------------------------------------------------------------------

__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem, bool pred) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    int sz = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(sz)
                 : "memory");
}
__device__ __forceinline__ void cp_async_8(void* smem, const void* gmem, bool pred) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    int sz = pred ? 8 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(s), "l"(gmem), "r"(sz)
                 : "memory");
}
__device__ __forceinline__ void cp_async_4(void* smem, const void* gmem) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Copy `BYTES` bytes (8, 16 or 32) per lane.
template <int BYTES>
__device__ __forceinline__ void cp_async_part(void* smem, const void* gmem, bool pred) {
    if constexpr (BYTES == 8) {
        cp_async_8(smem, gmem, pred);
    } else if constexpr (BYTES == 16) {
        cp_async_16(smem, gmem, pred);
    } else {
        static_assert(BYTES == 32, "row part of 8, 16 or 32 bytes");
        cp_async_16(smem, gmem, pred);
        cp_async_16(static_cast<char*>(smem) + 16, static_cast<const char*>(gmem) + 16, pred);
    }
}

// ---------------------------------------------------------------------------
// half-warp reduction of GQ per-head partial sums with value exchange:
// after it, lane l holds the full sum of head (l & 15) >> (4 - log2 GQ).
// GQ values over 16 lanes cost GQ - 1 + 4 - log2 GQ shuffles instead of 4 GQ.
// ---------------------------------------------------------------------------

template <int GQ> struct Log2;
template <> struct Log2<1> { static constexpr int v = 0; };
template <> struct Log2<2> { static constexpr int v = 1; };
template <> struct Log2<4> { static constexpr int v = 2; };
template <> struct Log2<8> { static constexpr int v = 3; };

template <int GQ>
__device__ __forceinline__ float halfwarp_reduce_heads(float (&v)[GQ], int lane) {
    float cur[GQ];
#pragma unroll
    for (int i = 0; i < GQ; ++i) cur[i] = v[i];
    int n = GQ;
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
        if (n > 1) {
            const bool upper = (lane & o) != 0;
            const int h = n >> 1;
#pragma unroll
            for (int i = 0; i < h; ++i) {
                float send = upper ? cur[i] : cur[i + h];
                float keep = upper ? cur[i + h] : cur[i];
                cur[i] = keep + __shfl_xor_sync(FULL, send, o);
            }
            n = h;
        } else {
            cur[0] += __shfl_xor_sync(FULL, cur[0], o);
        }
    }
    return cur[0];
}

template <int GQ>
__device__ __forceinline__ int head_of_lane(int lane) {
    return (lane & 15) >> (4 - Log2<GQ>::v);
}

// Max over the lanes of one half-warp that hold different heads.
template <int GQ>
__device__ __forceinline__ float halfwarp_max_over_heads(float x) {
#pragma unroll
    for (int o = 16 >> Log2<GQ>::v; o <= 8; o <<= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
    return x;
}

// Bitonic sort of one key per lane, descending across the warp.
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long x, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const unsigned long long y = __shfl_xor_sync(FULL, x, j);
            const bool keep_max = ((lane & k) == 0) == ((lane & j) == 0);
            x = keep_max ? (x > y ? x : y) : (x < y ? x : y);
        }
    }
    return x;
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(FULL, x, o);
        x = x > y ? x : y;
    }
    return x;
}

// ---------------------------------------------------------------------------
// block-wide exclusive scan of one int per thread (blockDim multiple of 32)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exclusive_scan(int x, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? s_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nw) s_warp[lane] = wi - w;
        if (lane == 31) s_warp[32] = wi;
    }
    __syncthreads();
    int r = s_warp[warp] + inc - x;
    if (total) *total = s_warp[32];
    __syncthreads();
    return r;
}

// ---------------------------------------------------------------------------
// launch parameter packs (host builds them after validation)
// ---------------------------------------------------------------------------

struct CacheView {
    const void* k;
    const void* v;
    int64_t sb, sh, st;
    int B, Hkv, Hq, d, T_cap, dtype;
};

struct GraphView {
    int mode, S, Cmax, max_tail, T_cap, G, gq;
    int rule;  // ckv_assign_rule
    int32_t* comm_of;
    int32_t* offs;
    int32_t* tok;
    int32_t* cnt;
    float* cent;
    int8_t* cent_q;
    float* cent_qs;
    int32_t* num_comm;
    int32_t* tail_tok;
    int32_t* tail_comm;
    int32_t* tail_len;
    int32_t* dev_err;
};

struct SelView {
    int tok_cap;
    int32_t* sel_comm;
    int32_t* n_sel;
    int32_t* sel_tok;
    int32_t* n_tok;
    int32_t* unit_prefix;
    int32_t* tok_prefix;
    int32_t* tail_sel;
};

// workspace carving
// Workspace head, shared by every call on a workspace and zero before its
// first use: the attention kernels' work ticket.  Every call leaves it zero
// (the attention's merge returns the ticket).  The other parts of each call
// start after the head.
constexpr size_t WS_RESERVED = 256;

struct DecodeWs {
    int* ticket;   // dynamic chunk counter (the workspace's first bytes)
    float* m;      // [slots, GQ]
    float* l;      // [slots, GQ]
    float* acc;    // [slots, GQ, D]
    float* lam;    // [U * lam_cap] graph logit of every selected token (sparse only)
    int lam_cap;   // list entries per unit
};

size_t build_ws_bytes(int U, int Cmax, int T_cap);
size_t select_ws_bytes(int U, int Cmax);
// lam_cap: selection entries per unit whose graph logits are kept (the
// selection's tok_cap; 0 for the dense comparator)
size_t decode_ws_bytes(int U, int gq, int d, int lam_cap);
DecodeWs carve_decode_ws(void* ws, size_t head, int U, int gq, int d, int lam_cap);

cudaError_t launch_build(const CacheView& c, const GraphView& g, const int32_t* labels,
                         int64_t labels_stride, int T, void* ws, cudaStream_t st);
cudaError_t launch_score_select(const CacheView& c, const GraphView& g, const void* q, int budget,
                                const SelView& s, void* ws, cudaStream_t st);
struct AssignParams;
// ap non-NULL: the merge kernel also runs the community update (and the
// K/V append when ap carries the new rows) for every unit, after finding
// its neighbours.
cudaError_t launch_sparse_decode(const CacheView& c, const GraphView& g, const SelView& s,
                                 const void* q, float* out, int32_t* nbr8, void* ws, const AssignParams* ap,
                                 cudaStream_t st);
cudaError_t launch_dense_decode(const CacheView& c, const void* q, int T, float* out, void* ws,
                                cudaStream_t st);
// The prefill token graph (ckv_build_edges): its hash tables' size and the
// launch of its four kernels.
int edges_hcap_log2(int T, int S);
size_t edges_ws_bytes(int U, int T, int S);
cudaError_t launch_build_edges(const CacheView& c, int mode, int S, const void* q, int T, int32_t* nbr, float* lam,
                               int32_t* co_src, int32_t* co_dst, int32_t* co_w, int32_t* co_n, int pair_cap,
                               int32_t* dev_err, void* ws, cudaStream_t st);
// Device address and size of the library's own decode scratch (looked up once
// per device, with that device current).
cudaError_t static_decode_scratch(void** ptr, size_t* bytes);

// k_new/v_new NULL: the new key is read from the cache at pos; otherwise it
// comes from k_new and both rows are first written to the cache at pos.
cudaError_t launch_assign_update(const CacheView& c, const GraphView& g, int pos, const void* k_new,
                                 const void* v_new, const int32_t* nbr8, int32_t* assigned, cudaStream_t st);

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline size_t ws_head_bytes(int, int) { return WS_RESERVED; }

// Programmatic dependent launch.  Kernels launched by launch_pdl() start
// with pdl_wait(), so they read and write nothing before the previous kernel
// in the stream has completed and its memory is visible; what overlaps is
// the launch itself (block scheduling) with that kernel's tail.  No kernel
// signals its dependents early: measured on the step, letting the next
// kernel's blocks take SM slots before the previous kernel ends slowed the
// scoring and selection, and the attention followed by its merge (about
// 63 -> 71 us per call on a 128K-context batch of 8).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Diagnostic kernel timing (ckv_kernel_timing): while it is on, every
// launch is bracketed by two CUDA events on its stream, and the durations are
// summed per kind when they are read (ckv_kernel_times).  Off by default; the
// events also cost the programmatic overlap between a call's kernels.
enum KernelKind { KK_BUILD = 0, KK_SCORE, KK_SELECT, KK_ATTENTION, KK_MERGE, KK_UPDATE, KK_EDGES, KK_COUNT };
bool timing_enabled();
cudaError_t timing_mark(int kind, bool start, cudaStream_t st);
void timing_set(bool on);
cudaError_t timing_read(float* total_ms, int32_t* launches);

template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(int kind, void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    const bool timed = timing_enabled();
    if (timed) {
        const cudaError_t e = timing_mark(kind, true, st);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (timed && e == cudaSuccess) e = timing_mark(kind, false, st);
    return e;
}


// Launch-shape cache for one kernel: the dynamic shared memory limit it was
// raised to and its resident blocks per SM, per device, so that steady-state
// calls make no attribute or occupancy queries (only launches).
struct LaunchCache {
    int smem_set[64] = {};   // largest dynamic smem the attribute allows (bytes)
    int occ_smem[64] = {};   // smem the occupancy below was computed for (+1)
    int occ_blocks[64] = {};
    int sms[64] = {};
};

template <typename Kern>
inline cudaError_t prepare_launch(Kern kern, LaunchCache& lc, size_t smem, int threads, int* blocks_per_sm,
                                  int* sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (lc.sms[dev] == 0) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        lc.sms[dev] = n;
    }
    if ((int)smem > lc.smem_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        lc.smem_set[dev] = (int)smem;
    }
    if (blocks_per_sm) {
        if (lc.occ_smem[dev] != (int)smem + 1) {
            int nb = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, threads, smem);
            if (e != cudaSuccess) return e;
            lc.occ_blocks[dev] = nb;
            lc.occ_smem[dev] = (int)smem + 1;
        }
        *blocks_per_sm = lc.occ_blocks[dev];
    }
    if (sms) *sms = lc.sms[dev];
    return cudaSuccess;
}

}  // namespace ckv
