/*
 * ckv.h -- C ABI of libckv, the CommunityKV decode-time hot path for NVIDIA
 * B200 (sm_100a).
 *
 * CommunityKV ("CommunityKV: Efficient Long-Context Decoding via Graph
 * Partitioning", McKenna, Alexandridis, Susanj, Liu, 2026) keeps the whole KV
 * cache and groups its tokens into communities.  At each decode step a query
 * is compared with the community centres only; the best communities up to a
 * token budget, plus the always-kept sink tokens, are read from the full
 * cache and exact attention runs over them; each new token joins one
 * neighbouring community and one centre is updated at a cost independent of
 * the context length.  Sources used below:
 *   [R-A] rit.work summary of the preprint, section "A graph of tokens
 *         replaces re-clustering" (paragraphs 3-6);
 *   [R-B] same page, section "The speed-up depends on how many graphs the
 *         model stores" (graph per KV group vs per query head, small budget);
 *   [ABS] the preprint's abstract (omanscience.com listing): constant-time
 *         local update, one graph per query head or per query group.
 * The community partition itself (Leiden on the prefill QK^T graph) is not
 * computed here: callers pass labels.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All pointers in the descriptors and arguments are DEVICE pointers owned
 *    by the caller, except the descriptors themselves (host structs, read
 *    during the call only).  The library keeps no pointer after returning.
 *  - Calls are asynchronous on `stream` and never synchronise the device
 *    (ckv_get_device_error and the diagnostic ckv_kernel_times, which wait
 *    for what they read, excepted);
 *    they may be captured into a CUDA graph after one uncaptured call per
 *    device and kernel shape (the first call caches device attributes).
 *  - No call allocates device memory.  Scratch comes from the caller's
 *    workspace `ws` of `ws_bytes` bytes (256-byte aligned), sized by
 *    ckv_workspace_size(); a smaller workspace returns CKV_ERR_WORKSPACE.
 *    Its first 256 bytes (the head: the attention kernels' work counter)
 *    must be zero before the workspace's first use, e.g. zero-fill the whole
 *    workspace once after allocating it; every call leaves the head zero.  The rest needs no
 *    initialisation.  Calls sharing a workspace must not overlap on the GPU.
 *  - Host-side checks happen before any launch and return a status without
 *    touching the device; ckv_last_error() then names the failed check.
 *    Data-dependent faults detected on the device (a label out of range, a
 *    full tail, a token list longer than its capacity) set bits in the
 *    caller's `dev_err` word (ckv_graph_desc) and the offending item is
 *    skipped; kernels never trap and never wait on another block.
 *  - Graph unit u = b * G + g, with G = Hkv graphs per sequence in
 *    CKV_GRAPH_PER_GROUP mode (graph g serves query heads g*Hq/Hkv ...) and
 *    G = Hq in CKV_GRAPH_PER_HEAD mode (graph g serves query head g, whose
 *    KV head is g / (Hq/Hkv)).  [R-B], [ABS]
 *  - Supported: d in {64, 128}; Hq/Hkv in {1, 2, 4, 8}; K/V/q in bf16 or
 *    fp32; 1 <= Cmax <= 8192; B * G <= 8192.
 */
#ifndef CKV_H
#define CKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CKV_API __attribute__((visibility("default")))
#else
#define CKV_API
#endif

#define CKV_ABI_VERSION 7
#define CKV_NEIGHBOURS 8

typedef struct CUstream_st* ckv_stream_t; /* the same handle as cudaStream_t */

typedef enum {
    CKV_OK = 0,
    CKV_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, stride or value  */
    CKV_ERR_MISALIGNED = 2,   /* K/V rows or q rows not 16-byte aligned    */
    CKV_ERR_UNSUPPORTED = 3,  /* d, Hq/Hkv, dtype or size not supported     */
    CKV_ERR_CAPACITY = 4,     /* T or a position beyond T_cap              */
    CKV_ERR_WORKSPACE = 5,    /* ws too small or misaligned                 */
    CKV_ERR_CUDA = 6          /* a CUDA launch or attribute call failed     */
} ckv_status;

typedef enum { CKV_DTYPE_F32 = 0, CKV_DTYPE_BF16 = 1 } ckv_dtype;
typedef enum { CKV_GRAPH_PER_GROUP = 0, CKV_GRAPH_PER_HEAD = 1 } ckv_graph_mode;

/*
 * How a new token picks its community among those of its 8 neighbours
 * (ckv_assign_update and the calls fused with it).  [R-A] paragraph 6 only
 * says the token joins a fitting neighbouring community; two readings:
 *   CKV_ASSIGN_SCORE  the candidate maximising k_new . cent_c / sqrt(d),
 *                     ties to the lower id (the default)
 *   CKV_ASSIGN_VOTE   the community that holds the most of the neighbours
 *                     (a majority vote over graph edges); among equally
 *                     frequent ones the larger k_new . cent_c / sqrt(d), then
 *                     the lower id
 */
typedef enum { CKV_ASSIGN_SCORE = 0, CKV_ASSIGN_VOTE = 1 } ckv_assign_rule;

/* Bits of the device error word (ckv_graph_desc.dev_err). */
#define CKV_DEVERR_SINK_LABEL 1   /* a position < S did not carry label -1            */
#define CKV_DEVERR_LABEL_RANGE 2  /* a label outside [0, Cmax) at a position >= S      */
#define CKV_DEVERR_TAIL_FULL 4    /* ckv_assign_update found the tail full; not joined */
#define CKV_DEVERR_TOKEN_CAP 8    /* a selection longer than tok_cap was truncated     */
#define CKV_DEVERR_EDGE_CAP 32    /* ckv_build_edges: more co-attention pairs than pair_cap */
#define CKV_DEVERR_INDEX 16       /* debug builds: an index read from a caller's array
                                     (a position, a run offset, a token count, a tail
                                     length) was out of range; the access was skipped */

/*
 * The full KV cache of one layer: K and V are [B, Hkv, T_cap, d] with the d
 * elements of a row contiguous; strides are in elements and their byte
 * values must be multiples of 16 (as must the base pointers).  The library
 * only reads it, except ckv_append_assign and ckv_sparse_decode_append,
 * which write row `pos` of K and V and nothing else.  [R-A] paragraph 5: the cache stays whole so any
 * fragment can be selected again later.
 */
typedef struct {
    int32_t dtype;  /* ckv_dtype, also the dtype of q */
    int32_t B, Hkv, Hq, d;
    int32_t T_cap;  /* rows allocated per (b, kv head) */
    const void* k;
    const void* v;
    int64_t stride_b, stride_h, stride_t;
} ckv_cache_desc;

/*
 * Community graph state for all B * G graph units of one layer.
 *   comm_of  int32 [U, T_cap]   community of each position (-1: sink or none)
 *   offs     int32 [U, Cmax+1]  CSR offsets of the build-time members
 *   tok      int32 [U, T_cap]   members sorted by (community, position)
 *   cnt      int32 [U, Cmax]    member count, including tail members
 *   cent     fp32  [U, Cmax, d] running-mean centre of each community
 *   cent_q   int8  [U, Cmax, d] cent quantised per row: with
 *                  s = max_i |cent_i| / 127 and r = 127 / max_i |cent_i|
 *                  (fp32 divisions), cent_q_i = round-half-even(cent_i * r)
 *                  (fp32 product), 0 where s = 0
 *   cent_qs  fp32  [U, Cmax]    that row scale s
 *                  Both are kept in step with cent by the build and the
 *                  update.  The scoring streams them (a quarter of cent's
 *                  bytes) and re-scores from cent only the communities whose
 *                  score bounds reach the budget cut (see ckv_score_select)
 *   num_comm int32 [U]          1 + largest community id present
 *   tail_tok, tail_comm int32 [U, max_tail]  tokens joined after the build
 *   tail_len int32 [U]
 *   dev_err  int32 [1]          OR of CKV_DEVERR_* bits; the caller zeroes it
 * assign_rule is a ckv_assign_rule; any other value is CKV_ERR_INVALID_ARG.
 * S sink positions 0..S-1 belong to no community and are always attended
 * ([R-A] paragraph 3).  T_cap here must equal the cache's T_cap.
 */
typedef struct {
    int32_t mode;  /* ckv_graph_mode */
    int32_t S;
    int32_t Cmax;
    int32_t max_tail;
    int32_t T_cap;
    int32_t assign_rule; /* ckv_assign_rule */
    int32_t* comm_of;
    int32_t* offs;
    int32_t* tok;
    int32_t* cnt;
    float* cent;
    int8_t* cent_q;     /* [U, Cmax, d] cent quantised per row, for the first scoring pass */
    float* cent_qs;     /* [U, Cmax] the rows' quantisation scales */
    int32_t* num_comm;
    int32_t* tail_tok;
    int32_t* tail_comm;
    int32_t* tail_len;
    int32_t* dev_err;
} ckv_graph_desc;

/*
 * One step's selection, written by ckv_score_select, read by
 * ckv_sparse_decode.
 *   sel_comm    int32 [U, Cmax]     selected community ids, best first
 *   n_sel       int32 [U]
 *   sel_tok     int32 [U, tok_cap]  positions to attend: the S sinks, then the
 *                                   build-time members of each selected
 *                                   community in rank order, then its tail
 *                                   members
 *   n_tok       int32 [U]           length of each sel_tok row
 *   tok_prefix  int32 [U, Cmax+1]   the list's runs: the build-time members of
 *                                   sel_comm[k] are entries [S + tok_prefix[k],
 *                                   S + tok_prefix[k+1]) of sel_tok;
 *                                   tok_prefix[0] = 0 (values before any
 *                                   truncation to tok_cap)
 *   tail_sel    int32 [U, max(max_tail, 1)]  the community of each tail
 *                                   member in the list, in list order (list
 *                                   entries from S + tok_prefix[n_sel] on)
 *   unit_prefix int32 [U+1]         exclusive prefix sum of n_tok, written by
 *                                   ckv_sparse_decode (its work split)
 * tok_cap >= T_cap can never overflow; tok_cap >= S + max(budget, largest
 * community) + max_tail suffices too.
 */
typedef struct {
    int32_t tok_cap;
    int32_t* sel_comm;
    int32_t* n_sel;
    int32_t* sel_tok;
    int32_t* n_tok;
    int32_t* tok_prefix;
    int32_t* tail_sel;
    int32_t* unit_prefix;
} ckv_selection_desc;

/* Bytes of workspace that any call below needs for these descriptors
 * (`sel` may be NULL).  Host only; never touches the device. */
CKV_API ckv_status ckv_workspace_size(const ckv_cache_desc* cache, const ckv_graph_desc* graph,
                              const ckv_selection_desc* sel, size_t* bytes);

/*
 * Build the community state from labels, once per sequence and layer
 * ([R-A] paragraph 4: every community gets a centre).
 *   labels  int32, row u at labels + u * labels_stride, T entries:
 *           -1 at positions < S, in [0, Cmax) elsewhere.
 * Writes comm_of (positions >= T get -1), offs, tok, cnt, cent (fp32 mean of
 * the member keys, summed in fp64 in position order), num_comm; empties the
 * tails.  Requires S <= T <= T_cap.
 */
CKV_API ckv_status ckv_build_centroids(const ckv_cache_desc* cache, const int32_t* labels,
                               int64_t labels_stride, int32_t T, const ckv_graph_desc* graph,
                               void* ws, size_t ws_bytes, ckv_stream_t stream);

/*
 * Score every community against the step's queries and select the top ones
 * under the budget ([R-A] paragraph 4; [R-B] on the small active budget).
 *   q       [B, Hq, d] in the cache dtype, contiguous.
 *   score   s_c = max over the graph's query heads h of q_h . cent_c / sqrt(d)
 *   select  rank non-empty communities by (s_c desc, id asc); take the
 *           longest ranked prefix whose cnt sum is <= budget, and at least the
 *           top community; the sinks come on top of the budget.
 * Writes every field of `sel`.  budget >= 0.  The pass over all communities
 * reads the int8 copy (cent_q, cent_qs) against an exact integer split of q,
 * with a rigorous error bound per score (|q . (cent - s cent_q)| <=
 * s |q|_1 / 2, plus the split's and the rounding's share); only the
 * communities whose bound reaches the budget cut are re-scored from the fp32
 * cent, so the selection is the one the fp32 scores give.  One kernel
 * launch.
 */
CKV_API ckv_status ckv_score_select(const ckv_cache_desc* cache, const ckv_graph_desc* graph,
                            const void* q, int32_t budget, const ckv_selection_desc* sel,
                            void* ws, size_t ws_bytes, ckv_stream_t stream);

/*
 * Exact softmax attention over the selected positions only, read in place
 * from the full cache with no gather copy ([R-A] paragraphs 4-5).
 *   out   fp32 [B, Hq, d]: o_h = sum_t softmax_t(q_h . k_t / sqrt(d)) v_t over
 *         sel_tok of head h's graph unit (zero for an empty selection).
 *   nbr8  int32 [U, 8] or NULL: the 8 non-sink selected positions with the
 *         largest graph logit (max over the graph's heads), best first, ties
 *         to the lower position, -1 padded: the neighbours for
 *         ckv_assign_update.
 */
CKV_API ckv_status ckv_sparse_decode(const ckv_cache_desc* cache, const void* q,
                             const ckv_graph_desc* graph, const ckv_selection_desc* sel,
                             float* out, int32_t* nbr8, void* ws, size_t ws_bytes,
                             ckv_stream_t stream);

/*
 * ckv_sparse_decode without a workspace argument.  The paper has no
 * counterpart: this exists for callers that cannot allocate device memory
 * for scratch, for example a serving engine that has reserved almost all
 * of HBM for its own KV pools and gives plug-ins no allocator, or a
 * latency-critical decode loop that must not call cudaMalloc because it can
 * synchronise the device.  Same arguments and results as ckv_sparse_decode,
 * computed by the same kernels; the split-K scratch instead lives in a
 * 32 MiB array inside libckv that every GPU which loads the library keeps
 * until the process exits.
 *   - Calls needing more scratch than CKV_NOALLOC_SCRATCH_BYTES return
 *     CKV_ERR_UNSUPPORTED before touching the device.  The need is the size
 *     ckv_workspace_size reports for the attention alone: the 256-byte
 *     head, about
 *     4 * (12288 + 2U) * gq * (d + 2) bytes of split-K partials (gq query
 *     heads per graph, U = B * graphs per sequence) and 4 * U * sel->tok_cap
 *     bytes of neighbour logits.  Per-head graphs with d = 128 need about
 *     6.4 MiB + the head + the logits; Hq/Hkv = 8 with d = 128 in per-group
 *     mode needs over 32 MiB and is refused.
 *   - If a launch fails, the call zeroes the array's head before returning
 *     (an asynchronous memset on `stream`), so later calls start clean.
 *   - The first call on each device looks up the array's device address
 *     (with that device current); make that first call before any stream
 *     capture.  No call allocates or frees memory.
 *   - All calls share the one array and it keeps the previous call's
 *     contents (it starts at zero when the library loads; calls leave its
 *     work counter at zero).  Calls that overlap
 *     on the GPU, e.g. on two streams at once, race on it and give wrong
 *     results: serialise them.
 */
#define CKV_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
CKV_API ckv_status ckv_sparse_decode_noalloc(const ckv_cache_desc* cache, const void* q,
                                             const ckv_graph_desc* graph,
                                             const ckv_selection_desc* sel, float* out,
                                             int32_t* nbr8, ckv_stream_t stream);

/*
 * Local update for the token just written at position `pos` (its K/V rows are
 * already in the cache): in every graph unit it joins one of the candidate
 * communities (those of nbr8), chosen by graph->assign_rule (by default the
 * one maximising k_new . cent_c / sqrt(d), ties to the lower id); that centre moves by (k_new - cent)/(cnt + 1), cnt
 * grows by one, and (pos, c) is appended to the tail.  O(8 d) per graph,
 * independent of the context length ([R-A] paragraph 6; [ABS]: the
 * update takes constant time).  assigned int32 [U] or NULL receives the community (-1: no
 * candidate, or tail full).  0 <= pos < T_cap.
 */
CKV_API ckv_status ckv_assign_update(const ckv_cache_desc* cache, const ckv_graph_desc* graph,
                             int32_t pos, const int32_t* nbr8, int32_t* assigned,
                             ckv_stream_t stream);

/*
 * The decode step's cache append fused with ckv_assign_update: writes the new
 * token's rows k_new and v_new (each [B, Hkv, d] in the cache dtype,
 * contiguous, 16-byte aligned) at position `pos` of K and V, then updates
 * every graph unit exactly as ckv_assign_update does, taking the new key from
 * k_new.  One launch; with ckv_sparse_decode_append the only calls that
 * write the cache, and only row pos
 * (the selection of the step that produced nbr8 never holds pos, so no
 * read of this step races with the write).  0 <= pos < T_cap.
 */
CKV_API ckv_status ckv_append_assign(const ckv_cache_desc* cache, const ckv_graph_desc* graph,
                                     int32_t pos, const void* k_new, const void* v_new,
                                     const int32_t* nbr8, int32_t* assigned, ckv_stream_t stream);

/*
 * One call for the decode step after the selection: ckv_sparse_decode
 * followed by ckv_append_assign (pos, k_new, v_new, assigned as there),
 * with the update run by the attention's merge kernel as soon as each unit's
 * neighbours are known, so no separate update launch follows.  nbr8 may be
 * NULL (the neighbours are then not written out).  Same results, bit for
 * bit, as the two calls in sequence.
 */
CKV_API ckv_status ckv_sparse_decode_append(const ckv_cache_desc* cache, const void* q,
                                            const ckv_graph_desc* graph, const ckv_selection_desc* sel,
                                            float* out, int32_t* nbr8, int32_t pos, const void* k_new,
                                            const void* v_new, int32_t* assigned, void* ws,
                                            size_t ws_bytes, ckv_stream_t stream);

/*
 * Dense comparator: exact GQA decode attention over positions [0, T) of every
 * (b, kv head), out fp32 [B, Hq, d].  The pages measure their speed-ups against
 * dense attention ([R-B], [ABS]).  Workspace: ckv_workspace_size().
 */
CKV_API ckv_status ckv_dense_decode(const ckv_cache_desc* cache, const void* q, int32_t T, float* out,
                            void* ws, size_t ws_bytes, ckv_stream_t stream);

/*
 * The token graph of a prefill pass, the input of the community partition
 * ([R-A] paragraph 3: nodes are tokens; a query that pays a key much
 * attention links the two, keys attended together are linked too, and the
 * first tokens stay out of the graph).  The partition itself is not computed
 * here.  For every graph unit u = b * G + g (G by `mode` as in
 * ckv_graph_desc) and every query position i in [S, T):
 *   direct edges  the 8 key positions j in [S, i) with the largest graph
 *                 logit lambda_ij = max over the graph's query heads of
 *                 q_{h,i} . k_j / sqrt(d), ties to the lower position (the
 *                 rule of the decode-time neighbours): nbr int32 [U, T, 8],
 *                 best first, -1 padded (rows i < S all -1); lam fp32
 *                 [U, T, 8] their logits (-inf where -1), or NULL;
 *   co-attention  every pair of keys j < l found together in one query's
 *   edges         direct edges, weighted by the number of such queries:
 *                 co_src, co_dst, co_w int32 [U, pair_cap], co_n int32 [U]
 *                 the number of pairs; the order of a unit's pairs is
 *                 unspecified.  A unit with more than pair_cap pairs writes
 *                 pair_cap of them and sets CKV_DEVERR_EDGE_CAP in *dev_err
 *                 (co_n still counts them all); pair_cap >= 28 (T - S) can
 *                 never overflow.
 *   q_prefill     [B, Hq, T, d] bf16 (the prefill queries), contiguous.
 * The keys are K's rows [0, T) of the cache.  bf16 caches only
 * (CKV_ERR_UNSUPPORTED otherwise); S <= T <= T_cap; the workspace is sized by
 * ckv_edges_workspace_size (an open-addressing table per unit) and needs no
 * initialisation.  The Q K^T products run on the tensor cores.
 */
CKV_API ckv_status ckv_edges_workspace_size(const ckv_cache_desc* cache, int32_t mode, int32_t S, int32_t T,
                                            size_t* bytes);
CKV_API ckv_status ckv_build_edges(const ckv_cache_desc* cache, int32_t mode, int32_t S, const void* q_prefill,
                                   int32_t T, int32_t* nbr, float* lam, int32_t* co_src, int32_t* co_dst,
                                   int32_t* co_w, int32_t* co_n, int32_t pair_cap, int32_t* dev_err, void* ws,
                                   size_t ws_bytes, ckv_stream_t stream);

/*
 * Reads the graph's device error word (ckv_graph_desc.dev_err, an OR of
 * CKV_DEVERR_* bits) after everything queued on `stream` so far: the one
 * call that synchronises (it waits for the stream).  *code receives the
 * word; with reset != 0 the word is then set back to zero on the device.
 * NULL graph or code: CKV_ERR_INVALID_ARG; a failed copy or wait:
 * CKV_ERR_CUDA.
 */
CKV_API ckv_status ckv_get_device_error(const ckv_graph_desc* graph, ckv_stream_t stream, int32_t* code,
                                        int32_t reset);

/*
 * Diagnostic kernel timing; no result depends on it.  With enable != 0, every
 * kernel that later calls on this host thread launch is bracketed by two
 * CUDA events on its stream; ckv_kernel_times() waits for the recorded
 * events and fills the HOST arrays total_ms[kind] (summed duration, ms) and
 * launches[kind] for the launches since its previous call, then forgets
 * them.  The events cost the programmatic overlap between a call's kernels,
 * so time the step itself without them.  n < CKV_KERNEL_KINDS or NULL
 * arrays: CKV_ERR_INVALID_ARG; a failed event call: CKV_ERR_CUDA.
 */
typedef enum {
    CKV_KERNEL_BUILD = 0,      /* the four kernels of ckv_build_centroids, as one */
    CKV_KERNEL_SCORE = 1,      /* ckv_score_select: scoring, selection and token list, one kernel */
    CKV_KERNEL_SELECT = 2,     /* no kernel (kept so the kinds keep their numbers) */
    CKV_KERNEL_ATTENTION = 3,  /* split-K attention (sparse and dense decode) */
    CKV_KERNEL_MERGE = 4,      /* merge, neighbours and fused update */
    CKV_KERNEL_UPDATE = 5,     /* ckv_assign_update / ckv_append_assign */
    CKV_KERNEL_EDGES = 6       /* the four kernels of ckv_build_edges, as one */
} ckv_kernel_kind;
#define CKV_KERNEL_KINDS 7
CKV_API ckv_status ckv_kernel_timing(int32_t enable);
CKV_API ckv_status ckv_kernel_times(float* total_ms, int32_t* launches, int32_t n);

/*
 * 1 in the debug build of the library (libckv_debug.so, compiled with
 * CKV_DEBUG), 0 otherwise.  The debug build checks, on the device, every
 * index that a caller's array feeds to a kernel before using it: the
 * positions in sel_tok and n_tok against T_cap and tok_cap (attention), the
 * CSR run offsets against T_cap (selection), the tail length against
 * [0, max_tail] (selection, update).  A bad one sets CKV_DEVERR_INDEX in
 * dev_err and the access is skipped or clamped: results are then wrong but
 * nothing outside the arrays is touched, and no kernel traps.  Arithmetic
 * and results on valid inputs are those of the release build.  (A negative
 * tail length skips the join in every build.)
 */
CKV_API int32_t ckv_debug_build(void);

CKV_API const char* ckv_status_string(ckv_status status);
/* Message of the last failed call on this host thread ("" if none). */
CKV_API const char* ckv_last_error(void);
CKV_API int32_t ckv_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CKV_H */
