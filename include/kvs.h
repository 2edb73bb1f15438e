/*
 * kvs.h -- C ABI of the KVSlimmer asymmetric-KV-merging hot path on B200 (sm_100a).
 *
 * The method: "论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程" (blog deep dive of
 * arXiv 2603.00907) and the abstract pages of "KVSlimmer: Theoretical Insights and
 * Practical Optimizations for Asymmetric KV Merging". Adjacent Keys (k_m, k_m+1) of
 * a cache K = [k_1..k_n] are merged with forward-only closed-form weights (§数学主线二,
 * §数学主线四); Values are preserved (核心判断: merge homogeneous Keys, keep
 * heterogeneous Values); decode attention runs over the merged cache (Figure 5,
 * decoder stage).
 *
 * Data layout (all device memory, row-major, caller-owned):
 *   cache K, V      [B, H_kv, T_cap, d]   element type kvs_dtype (fp32 or bf16)
 *   log-count logn  [B, H_kv, T_cap]      fp32; log(number of original tokens a row
 *                                         stands for); 0 for unmerged rows. NULL on
 *                                         input means "all counts are 1".
 *   lengths len     [B, H_kv]             int32; valid prefix of each head's rows
 *   window queries  [B, H_q, W, d]        query head hq belongs to KV head hq / G,
 *                                         G = H_q / H_kv; query j sits at cache
 *                                         position len - W + j and sees positions
 *                                         <= its own.
 *   decode queries  [B, H_q, d]; decode output [B, H_q, d] (same dtype as the cache)
 *   pair arrays     [B, H_kv, T_cap / 2]  fp32, indexed by pair p; pair p of a head is
 *                                         the rows (c0 + 2p, c0 + 2p + 1), c0 = cand_begin.
 *
 * Candidate span of a head: [cand_begin, len - n_recent). Rows before it (sink
 * tokens; the pages keep 32, §实验设置) and after it (the recent window, §工程上怎么用)
 * are never merged. P = max(0, (len - n_recent - cand_begin) / 2) pairs; an odd
 * leftover row is never merged.
 *
 * Streams and memory: every call is asynchronous on `stream`, allocates nothing,
 * keeps no state between calls and never synchronises, unless its comment says
 * otherwise. Pointers must be 16-byte aligned (cache, query and output tensors)
 * or 4-byte aligned (int32 / fp32 arrays); the workspace 256-byte aligned.
 *
 * Errors: argument errors are found on the host and returned before anything is
 * launched. Launch failures return KVS_ERR_CUDA. Conditions only the device can
 * see (a length outside [0, T_cap], an output that would not fit) are skipped by
 * the kernels and recorded as bits in the workspace's device flag word, read with
 * kvs_device_flags().
 */
#ifndef KVS_H_
#define KVS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVS_OK = 0,
  KVS_ERR_INVALID_ARG = 1,   /* NULL pointer, non-positive size, misalignment, bad W / n_recent */
  KVS_ERR_UNSUPPORTED = 2,   /* head dim, dtype, group size or window size not built */
  KVS_ERR_BUDGET = 3,        /* a budget that the candidate pairs cannot reach (host-planned
                                calls; kvs_merge_compact reports it as KVS_FLAG_BUDGET) */
  KVS_ERR_WORKSPACE = 4,     /* workspace NULL, too small or not 256-byte aligned */
  KVS_ERR_ALIAS = 5,         /* an output overlaps an input in a way the call does not allow */
  KVS_ERR_CUDA = 6           /* a CUDA runtime call or kernel launch failed */
} kvs_status;

typedef enum { KVS_F32 = 0, KVS_BF16 = 1 } kvs_dtype;

/* Shape of a cache. d in {64, 128}; H_q a multiple of H_kv with G = H_q / H_kv <= 8;
   T_cap even. */
typedef struct {
  int32_t B, H_kv, H_q, d, T_cap;
  int32_t dtype; /* kvs_dtype */
} kvs_cache_desc;

typedef struct CUstream_st* kvs_stream_t; /* a cudaStream_t; NULL = legacy default stream */

enum { KVS_OP_SCORE = 0, KVS_OP_MERGE = 1, KVS_OP_DECODE = 2, KVS_OP_PREFILL = 3 };
enum { KVS_SCOPE_HEAD = 0, KVS_SCOPE_POOLED = 1 };
/* Scoring form: the coupled forward-only objective, or its diagonal-only ablation;
   either may be combined (bitwise or) with KVS_FORM_PER_QUERY, the per-query window
   reading (see kvs_score_pairs_form). */
enum { KVS_FORM_FULL = 0, KVS_FORM_DIAGONAL = 1, KVS_FORM_PER_QUERY = 2 };

/* Device flag bits (see kvs_device_flags). */
enum {
  KVS_FLAG_BAD_LENGTH = 1,      /* a len[] value was < 0 or > T_cap; that head was skipped */
  KVS_FLAG_OUT_CAPACITY = 2,    /* a merged head or an append did not fit the output capacity */
  KVS_FLAG_INPLACE_SPAN = 4,    /* in-place merge on a span longer than it supports; head skipped */
  KVS_FLAG_NONFINITE_STATS = 8, /* a window query had no finite softmax normaliser */
  KVS_FLAG_TIMEOUT = 16,        /* a pipeline wait gave up (bounded waits); results invalid */
  KVS_FLAG_BUDGET = 32          /* a unit's target is below the shortest length repeated rounds
                                   can reach (every candidate span shrinks to one row at best);
                                   the unit still merges what it can this round */
};

/*
 * Bytes of workspace `op` needs for caches of shape `desc` (and window W for
 * KVS_OP_SCORE). Returns 0 for an invalid shape. Every layout begins with the
 * same persistent region: the device flag word (first 256 bytes) and one decode
 * arrival counter per KV head (the next 256-byte-aligned block). Zero the whole
 * workspace once (cudaMemset) before its first use; every call leaves the
 * persistent region valid for the next call, so one zeroed workspace, sized for
 * the largest op, serves all three ops on one stream. Calls that share a
 * workspace must not overlap in time.
 */
size_t kvs_workspace_size(const kvs_cache_desc* desc, int32_t W, int32_t op);

/*
 * kvs_score_pairs -- one scoring pass: window statistics, then every candidate
 * pair's forward-only Hessian norms, merge weight and score.
 *
 *   alpha_bar_t = mean over the window queries of softmax_t(q k_t^T / sqrt(d) + logn_t)
 *   o_bar       = mean over the window queries of o_q = sum_t alpha_t v_t
 *       (attention forward: §数学主线三; averaging the window: the one-query formulas
 *        of the pages applied to the window mean)
 *   N11 = |a_a (1 - 2 a_a)| |v_a - o_bar|,  N22 = |a_b (1 - 2 a_b)| |v_b - o_bar|,
 *   N12 = a_a a_b |v_a + v_b - 2 o_bar|      (|c11|, |c22|, |c12| of §数学主线四)
 *   D = N11 - 2 N12 + N22;  w_b = (N22 - N12) / D;
 *   score = |k_b - k_a|^2 (N11 N22 - N12^2) / D  (minimum of the §数学主线二 objective
 *       with the forward-only scalars); when D <= 1e-6 (N11 + N22) or a term is not
 *       finite: w_b = 1/2, score = |k_b - k_a|^2 (N11 + 2 N12 + N22) / 4.
 *
 * In:  K, V [B,H_kv,T_cap,d]; logn (nullable); len [B*H_kv]; cand_begin [B*H_kv];
 *      n_recent >= 0; Q_win [B,H_q,W,d], 1 <= W, G*W <= 128 (else KVS_ERR_UNSUPPORTED).
 * Out: score, w_b [B,H_kv,T_cap/2] fp32 (entries p >= P of a head are not written).
 * Workspace: kvs_workspace_size(desc, W, KVS_OP_SCORE) bytes.
 */
kvs_status kvs_score_pairs(const kvs_cache_desc* desc, const void* K, const void* V,
                           const float* logn, const int32_t* len, const int32_t* cand_begin,
                           int32_t n_recent, const void* Q_win, int32_t W,
                           float* score, float* w_b,
                           void* ws, size_t ws_bytes, kvs_stream_t stream);

/*
 * kvs_score_pairs_form -- kvs_score_pairs with a choice of scoring form.
 *
 * form = KVS_FORM_FULL: exactly kvs_score_pairs.
 * form = KVS_FORM_DIAGONAL: the ablation that drops the coupling term of the
 *   §数学主线二 objective (g12 = 0; the per-key weighting of AsymKV that the pages
 *   contrast KVSlimmer with): N12 is taken as 0, so
 *     w_b = N22 / (N11 + N22),  score = |k_b - k_a|^2 N11 N22 / (N11 + N22),
 *   with the same degenerate rule (w_b = 1/2, score = |k_b - k_a|^2 (N11 + N22) / 4
 *   when N11 + N22 is not positive or a term is not finite).
 * form | KVS_FORM_PER_QUERY: the window of several queries read per query instead of
 *   through its mean. The pages derive the norms for one query; here every window query
 *   q gets its own single-query norms, and the pair's norms are their mean over the
 *   Qv window queries that see at least one row:
 *     N11 = mean_q |a_qa (1 - 2 a_qa)| |v_a - o_q|,  N22 likewise,
 *     N12 = mean_q a_qa a_qb |v_a + v_b - 2 o_q|,
 *   a_qt = softmax_t(q k_t^T / sqrt(d) + logn_t), o_q = sum_t a_qt v_t (the causal window
 *   as above); weight, score and degenerate rule as for the base form. For one window
 *   query it equals the base form. Built for bf16 caches with G*W <= 128 only (else
 *   KVS_ERR_UNSUPPORTED, nothing launched).
 * Any other form: KVS_ERR_INVALID_ARG, nothing launched. Arguments, outputs,
 * workspace and errors otherwise as kvs_score_pairs.
 */
kvs_status kvs_score_pairs_form(const kvs_cache_desc* desc, const void* K, const void* V,
                                const float* logn, const int32_t* len, const int32_t* cand_begin,
                                int32_t n_recent, const void* Q_win, int32_t W,
                                float* score, float* w_b, int32_t form,
                                void* ws, size_t ws_bytes, kvs_stream_t stream);

/*
 * kvs_merge_compact -- one merge round: select pairs to the budget, merge them,
 * and compact the cache (order preserved).
 *
 * Each unit merges R = min(P_unit, max(0, len_unit - target_unit)) pairs: the R
 * with the smallest (score, index); NaN scores rank as +inf, -0 as +0. With
 * scope KVS_SCOPE_HEAD a unit is one (b, h) and target has B*H_kv entries; with
 * KVS_SCOPE_POOLED a unit is one sequence b across its H_kv heads, target has B
 * entries (total rows over the heads), and the index order is (h, p).
 * A selected pair (a, b) becomes one row at the pair's slot:
 *   k* = k_a + w_b (k_b - k_a)                              (§数学主线四)
 *   v* = (n_a v_a + n_b v_b) / (n_a + n_b),  logn* = log(n_a + n_b),  n = exp(logn)
 *       (Values preserved: attention over the merged row equals attention over the
 *        n_a + n_b original rows sharing k*)
 * len_out = len - R. Repeating rounds reaches the budget exactly.
 *
 * Out-of-place (K_out != K): outputs must not overlap inputs (KVS_ERR_ALIAS).
 * In-place (K_out == K, V_out == V, logn_out == logn, len_out == len): allowed when
 * every head's span len - cand_begin is at most 8192 rows; rows before cand_begin
 * are left untouched. Longer spans set KVS_FLAG_INPLACE_SPAN and are skipped.
 *
 * In:  the cache (logn nullable), len, cand_begin, n_recent, score and w_b from
 *      kvs_score_pairs for the same cache, target, scope.
 * Out: K_out, V_out [B,H_kv,T_cap_out,d]; logn_out [B,H_kv,T_cap_out]; len_out [B*H_kv].
 *      Optional (nullable): dbg_selected [B,H_kv,T_cap/2] u8 (1 = merged);
 *      dbg_out_offset [B,H_kv,T_cap/2] i32 (output row of the pair's first row);
 *      dbg_kmerged_f32 [B,H_kv,T_cap/2,d] fp32 (merged key before rounding).
 * Workspace: kvs_workspace_size(desc, 0, KVS_OP_MERGE) bytes.
 * The selection and the out-of-place merge kernels are launched with programmatic
 * stream serialisation; each waits for the preceding kernel's completion and memory
 * before any access, so the call keeps plain stream order.
 */
kvs_status kvs_merge_compact(const kvs_cache_desc* desc, const void* K, const void* V,
                             const float* logn, const int32_t* len, const int32_t* cand_begin,
                             int32_t n_recent, const float* score, const float* w_b,
                             const int32_t* target, int32_t scope, int32_t T_cap_out,
                             void* K_out, void* V_out, float* logn_out, int32_t* len_out,
                             uint8_t* dbg_selected, int32_t* dbg_out_offset,
                             float* dbg_kmerged_f32, void* ws, size_t ws_bytes,
                             kvs_stream_t stream);

/*
 * kvs_prefill_chunk -- one step of chunked streaming prefill compression: append a
 * prompt chunk to every head, then merge in place back to the budget.
 *
 * The serving loop of §实验设置 (compression context budget 2048, chunk size 512, 32
 * preserved initial tokens): the prompt enters the cache one chunk at a time, and
 * after each chunk every head is merged back to `budget` rows. Reading of the pages
 * (they give only the three numbers): the rounds are kvs_score_pairs +
 * kvs_merge_compact rounds with candidate span [sink, len - W) (the first `sink` rows
 * and the newest W rows are never merged), per-head scope, target = budget, window
 * queries Q_win = the queries of the chunk's last W positions; rounds repeat while
 * len > budget, each merging R = min(P, len - budget) pairs.
 *
 * Every head must hold L rows on entry (all heads equal; the caller tracks L, e.g. 0
 * for an empty cache, then each call's *L_out). A head whose len differs is left
 * unchanged and sets KVS_FLAG_BAD_LENGTH.
 * In:  K, V [B,H_kv,T_cap,d] (updated in place); logn [B,H_kv,T_cap] (required: merged
 *      counts); len [B*H_kv]; k_chunk, v_chunk [B,H_kv,n,d] (cache dtype, nullable
 *      when n = 0); Q_win [B,H_q,W,d]; 1 <= W, G*W <= 128; sink >= 0; form as
 *      kvs_score_pairs_form.
 * Out: the cache advanced; *L_out (host) = the length of every head afterwards:
 *      min(L + n, budget) when budget is reachable.
 * Errors (nothing launched): KVS_ERR_INVALID_ARG (L + n > T_cap, bad pointers or
 * alignment), KVS_ERR_UNSUPPORTED (L + n - sink > 8192: the in-place rounds rewrite at
 * most 8192 rows of a head; or G*W > 128), KVS_ERR_BUDGET (budget below what the
 * protected rows allow), KVS_ERR_ALIAS, KVS_ERR_WORKSPACE.
 * Workspace: kvs_workspace_size(desc, W, KVS_OP_PREFILL) bytes, zeroed once.
 */
kvs_status kvs_prefill_chunk(const kvs_cache_desc* desc, void* K, void* V, float* logn,
                             int32_t* len, int32_t L, const void* k_chunk, const void* v_chunk,
                             int32_t n, const void* Q_win, int32_t W, int32_t budget,
                             int32_t sink, int32_t form, int32_t* L_out, void* ws,
                             size_t ws_bytes, kvs_stream_t stream);

/*
 * kvs_plan_rounds -- the round driver's plan, on the host: the lengths a head of `len`
 * rows passes through when merged round by round to `target` (reading R4: a round
 * merges R = min(P, len - target) pairs, P = floor((len - n_recent - cand_begin) / 2)
 * candidate pairs). A caller that knows its heads' lengths uses it to size the round
 * buffers and to capture the rounds into a graph without reading lengths back.
 * Out: lens_out[0] = len, lens_out[k] = the length after round k, lens_out[*n_rounds]
 *      = target (host arrays). Nothing touches a GPU.
 * Errors: KVS_ERR_INVALID_ARG (NULL pointers, negative arguments, or max_lens too small
 * for the plan), KVS_ERR_BUDGET (a round would merge nothing before reaching target).
 */
kvs_status kvs_plan_rounds(int32_t len, int32_t target, int32_t cand_begin, int32_t n_recent,
                           int32_t* lens_out, int32_t max_lens, int32_t* n_rounds);

/*
 * kvs_decode_attn -- one decode step of GQA attention over the merged cache
 * (attention of §数学主线三 with the log-count bias; the decoder stage of Figure 5).
 *
 *   out[b, hq] = sum_t softmax_t(q[b,hq] . k_t / sqrt(d) + logn_t) v_t over the
 *   rows t < len[b, hq / G], plus the appended row when k_new is given.
 *
 * If k_new and v_new are non-NULL ([B, H_kv, d]), the step first appends them
 * (count 1) at row len of every head: the row is attended, written into K, V
 * (and logn = 0 when logn is non-NULL) and len is incremented by 1. A head whose
 * len == T_cap cannot take the row: it sets KVS_FLAG_OUT_CAPACITY and is not
 * changed (its output is still written, without the new row).
 * In:  q [B,H_q,d]; K, V; logn (nullable); len [B*H_kv].
 * Out: out [B,H_q,d] (cache dtype); K, V, logn, len updated when appending.
 * Workspace: kvs_workspace_size(desc, 0, KVS_OP_DECODE) bytes; its counters must be
 * zero at the first call (each call leaves them zero).
 * The first call for a device and a B*H_kv sets kernel attributes and asks the CUDA
 * occupancy calculator which launch shape fits (host calls only, cached): make it
 * outside any stream capture. Launch shape: one thread-block cluster per KV head that
 * combines the head's splits in distributed shared memory, when every head's cluster
 * fits the GPU at once; else a grid of splits combined by the last one to finish.
 * The kernel is launched with programmatic stream serialisation: it may be scheduled
 * while the previous kernel of the stream runs, but it waits for that kernel's
 * completion and memory before any access, so the call keeps plain stream order.
 */
kvs_status kvs_decode_attn(const kvs_cache_desc* desc, const void* q, void* K, void* V,
                           float* logn, int32_t* len, const void* k_new, const void* v_new,
                           void* out, void* ws, size_t ws_bytes, kvs_stream_t stream);

/*
 * kvs_decode_attn_static -- kvs_decode_attn without a caller-provided workspace.
 * The pages have no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory at call time: a runtime whose memory plan is fixed
 * before it starts serving, a host framework that only hands a plugin a stream, or
 * code that must not let an allocation synchronise the device mid-step.
 *
 * It computes exactly what kvs_decode_attn computes (same kernels, same arguments
 * minus ws / ws_bytes) using a scratch buffer built into the library: a device
 * array of kvs_static_scratch_bytes() bytes (4 MiB) that every GPU which loads the
 * library holds until the process exits. Shapes whose decode workspace
 * (kvs_workspace_size(desc, 0, KVS_OP_DECODE)) exceeds it return KVS_ERR_WORKSPACE
 * and launch nothing. It allocates nothing: no cudaMalloc, no cudaFree.
 *
 * The first call on a device does the set-up for that device: under CUDA's default
 * lazy module loading it loads the library's device code there, which is when the
 * array is placed in device memory (and may synchronise the device), and it looks up
 * the array's device address. Make that first call (a warm-up call will do) while
 * setting up, outside any stream capture and before the serving loop; later calls
 * make no allocation and no synchronising call.
 *
 * All calls share the one buffer: calls that overlap on the GPU (other streams, other
 * host threads) race on it, and the buffer keeps the last call's contents. Every call
 * clears the arrival counters on `stream` before launching; the flag word is not
 * cleared, so device flags (KVS_FLAG_OUT_CAPACITY for a head that cannot take the
 * appended row, KVS_FLAG_BAD_LENGTH, KVS_FLAG_TIMEOUT) accumulate over calls until
 * kvs_static_device_flags reads and clears them.
 */
kvs_status kvs_decode_attn_static(const kvs_cache_desc* desc, const void* q, void* K, void* V,
                                  float* logn, int32_t* len, const void* k_new,
                                  const void* v_new, void* out, kvs_stream_t stream);

/* Size in bytes of the scratch buffer kvs_decode_attn_static uses. */
size_t kvs_static_scratch_bytes(void);

/*
 * kvs_static_device_flags -- read (and, if clear != 0, clear) the device flag word of
 * the built-in scratch buffer that kvs_decode_attn_static uses on the current device:
 * the bits every static call since the last clear has set. The read is ordered after
 * the work already queued on `stream`; the call synchronises `stream`. Host pointer
 * `flags` receives the bits. Errors: KVS_ERR_INVALID_ARG (flags NULL), KVS_ERR_CUDA.
 */
kvs_status kvs_static_device_flags(int32_t* flags, int32_t clear, kvs_stream_t stream);

/*
 * kvs_device_flags -- read (and optionally clear) the device flag word of a
 * workspace. Synchronises `stream`. Host pointer `flags` receives the bits.
 */
kvs_status kvs_device_flags(void* ws, int32_t* flags, int32_t clear, kvs_stream_t stream);

/*
 * kvs_stream_read -- a measurement helper, not part of the method: the device-memory
 * read ceiling of the decode step's access pattern. Streams the `rows` rows of a
 * [rows, d] bf16 device array (d in {64, 128}, 16-byte aligned, rows < 2^31) through
 * shared memory with the decode kernel's loads -- 2D TMA boxes of 128 rows, 128-byte
 * swizzle, a 3-stage ring, L2 evict-first -- split evenly over `ctas` CTAs (one per SM
 * at most), and computes nothing. Timing it over the bytes one decode launch reads, with
 * the launch's CTA count, gives the decode time with free arithmetic.
 * Workspace: at least 256 bytes, 256-byte aligned (its flag word records a wait that
 * gave up, KVS_FLAG_TIMEOUT). Errors: KVS_ERR_INVALID_ARG, KVS_ERR_UNSUPPORTED,
 * KVS_ERR_WORKSPACE, KVS_ERR_CUDA.
 */
kvs_status kvs_stream_read(const void* buf, int64_t rows, int32_t d, int32_t ctas, void* ws,
                           size_t ws_bytes, kvs_stream_t stream);

/* Static string for a status code. */
const char* kvs_status_str(kvs_status s);

/* Library version, for the binding's load check. */
int32_t kvs_version(void);

/* Number of kernels this process has launched through the library so far
   (host-side count at launch time; replays of a captured CUDA graph do not add). */
int64_t kvs_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* KVS_H_ */
