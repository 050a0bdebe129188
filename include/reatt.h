/*
 * reatt.h -- C ABI of the B200 (sm_100a) ReAttention top-k span attention path.
 *
 * The operation (pages about "ReAttention: Training-Free Infinite Context with
 * Finite Attention Scope", arXiv 2407.15176):
 *   - arXiv abstract: position-agnostic top-k attention is taken before the
 *     ordinary position-aware self-attention;
 *   - research-map summary, "Approach": middle KV-cache segments are scored by
 *     the dot product of the query with un-positioned keys, concatenated with
 *     the global and local caches, and only then given positional embeddings;
 *   - OpenReview discussion, "Decoding Phase" pseudocode: score = query .
 *     key[global:-local]^T, top-k recall, concatenation global ++ recalled ++
 *     local, then attention over that window;
 *   - OpenReview discussion, NIAH settings: global 32, local 4096, segment 32.
 * Fixed readings where the pages are silent: GQA scores sum q.k over the KV
 * head's query heads (fp32 accumulation); a span's score is the max over its
 * tokens (and over the C queries); ties prefer the lower span index; chosen
 * spans keep ascending order; the window is global ++ chosen ++ local ++
 * current; RoPE (rotate-half pairs (i, i+d/2), frequency base^(-2i/d)) at
 * window positions 0..W-1, query c at W-C+c; causal softmax, scale 1/sqrt(d).
 *
 * Partition of the T cached tokens of one (batch, KV head):
 *   global = [0, min(G,T)), local = [max(G, T-L), T), middle = [G, G+M),
 *   M = max(0, T-G-L), NS = ceil(M/S) spans tiled from the left (the last one
 *   may be short), k_eff = min(k, NS),
 *   W = min(G,T) + (rows of the chosen spans) + (T - max(G, T-L) if T > G) + C,
 *   Wmax = G + k*S + L + C  (an upper bound on W; at most 2^24, since window
 *   positions enter the RoPE angle as exact fp32 integers; larger windows are
 *   REATT_EUNSUPPORTED).
 *
 * Conventions for every entry point
 *   - Layouts are contiguous row-major:
 *       q            [B, Hq,  C,  d]     dtype
 *       k/v cache    [B, Hkv, T,  d]     dtype, un-rotated (pre-RoPE)
 *       k/v cur      [B, Hkv, C,  d]     dtype, un-rotated
 *       span_scores  [B, Hkv, NS]        float32
 *       sel          [B, Hkv, k]         int32, ascending span ids, -1 padded
 *       k/v window   [B, Hkv, Wmax, d]   float32 (K rotated, V as is)
 *       win_len      [B, Hkv]            int32
 *       out          [B, Hq,  C,  d]     float32
 *     Query head j reads KV head j / (Hq/Hkv).
 *   - Every data pointer is a DEVICE pointer on the current device, 16-byte
 *     aligned.  The caller owns all memory, including the workspace sized by
 *     reatt_workspace_bytes(); the library allocates nothing and keeps no
 *     state between calls (re-entrant on distinct workspaces).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: results are valid once the stream has
 *     reached that point.  Two calls that share a workspace must be ordered.
 *   - Return value: REATT_OK, or an error code.  Arguments are checked on the
 *     host before anything is enqueued; on an argument error nothing is
 *     launched.  REATT_ECUDA reports a launch error (cudaGetLastError).
 *     A kernel whose bounded wait gives up records REATT_ETIMEOUT in the
 *     workspace status word, readable with reatt_workspace_status().
 *     No C++ exception or abort crosses this interface.
 */
#ifndef REATT_H
#define REATT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define REATT_API __attribute__((visibility("default")))
#else
#define REATT_API
#endif

/* Same type as cudaStream_t, declared here so this header needs no CUDA headers. */
typedef struct CUstream_st *reatt_stream;

typedef enum {
    REATT_OK = 0,
    REATT_EINVAL = 1,       /* null/misaligned pointer, bad or inconsistent size  */
    REATT_EUNSUPPORTED = 2, /* valid request outside what the kernels implement    */
    REATT_ECUDA = 3,        /* a CUDA call or kernel launch failed                  */
    REATT_ETIMEOUT = 4      /* a kernel's bounded wait gave up (workspace status)   */
} reatt_status;

typedef enum { REATT_F32 = 0, REATT_BF16 = 1 } reatt_dtype;

typedef struct {
    int32_t B;          /* batch (independent sequences)                  >= 1 */
    int32_t Hq;         /* query heads                                    >= 1 */
    int32_t Hkv;        /* KV heads, Hq % Hkv == 0                        >= 1 */
    int32_t d;          /* head width: 64 or 128                               */
    int32_t C;          /* current (query) tokens: 1 = decode, >1 = prefill    */
    int32_t G;          /* global tokens kept at the start                >= 0 */
    int32_t L;          /* local tokens kept at the end                   >= 0 */
    int32_t S;          /* span length                                    >= 1 */
    int32_t k;          /* spans kept (top-k), 0 <= k <= 65536                 */
    int32_t dtype;      /* reatt_dtype of q, caches and current tokens         */
    int64_t T;          /* cached tokens, 0 <= T < 2^31                         */
    double rope_base;   /* RoPE base (> 0, finite)                              */
    int64_t T_cap;      /* rows allocated per (batch, KV head) in k_cache and
                           v_cache: row t of (b, h) is at ((b*Hkv + h)*T_cap + t)*d;
                           0 means T (dense caches); otherwise T <= T_cap < 2^31 */
} reatt_dims;

/* Text for a status code (static storage; never NULL). */
REATT_API const char *reatt_status_string(int status);

/* NS = ceil(max(0, T-G-L) / S).  EINVAL on bad dims or null output. */
REATT_API int reatt_num_spans(const reatt_dims *dims, int64_t *num_spans);

/* Wmax = G + k*S + L + C, the row capacity of the window buffers. */
REATT_API int reatt_window_max(const reatt_dims *dims, int64_t *wmax);

/* Bytes of device workspace any call with these dims may use (a multiple of
 * 256).  The workspace holds a status word, split-K partials, top-k
 * candidates, and, for reatt_step, the span scores and selection. */
REATT_API int reatt_workspace_bytes(const reatt_dims *dims, size_t *bytes);

/* Reads and clears the status word kept at the start of a workspace.  Waits
 * for `stream`.  *status is REATT_OK or REATT_ETIMEOUT. */
REATT_API int reatt_workspace_status(void *ws, int *status, reatt_stream stream);

/*
 * Span scoring (decoding pseudocode: score = query . key[global:-local]^T;
 * research-map summary "Approach": un-positioned keys).
 *   span_scores[b,h,s] = max over tokens t of span s and over queries c of
 *                        sum_{j in group(h)} q[b,j,c,:] . k_cache[b,h,t,:]
 * on un-rotated vectors, fp32 accumulation.  Writes B*Hkv*NS floats; no
 * per-token score is ever stored.  ws: workspace of reatt_workspace_bytes().
 */
REATT_API int reatt_score_spans(const reatt_dims *dims, const void *q, const void *k_cache,
                      float *span_scores, void *ws, reatt_stream stream);

/*
 * Top-k spans (decoding pseudocode: idx_recall = score.topk), per (b, h):
 * the k_eff = min(k, NS) highest span_scores, ties to the lower span id,
 * written in ascending span order (the cache order the window keeps);
 * entries k_eff..k-1 are -1.  NaN scores are not supported.
 */
REATT_API int reatt_topk(const reatt_dims *dims, const float *span_scores, int32_t *sel, void *ws,
               reatt_stream stream);

/*
 * Window construction (decoding pseudocode: concatenation global ++ recalled
 * ++ local; "Approach": positional embedding applied after concatenation).
 * For each (b, h): window rows = global ++ rows of the spans in sel (in the
 * order given, which reatt_topk makes ascending) ++ local ++ the C current
 * tokens.  K row p is rotated by RoPE at position p (fp32 arithmetic, angles
 * reduced in fp64); V rows are copied.  Rows W..Wmax-1 are left untouched.
 * win_len[b,h] = W.  sel must be laid out as reatt_topk writes it: the
 * min(k, NS) chosen span ids in ascending order, then -1.  Other contents give
 * unspecified rows, but every read stays inside the cache.
 */
REATT_API int reatt_gather_rope(const reatt_dims *dims, const void *k_cache, const void *v_cache,
                      const void *k_cur, const void *v_cur, const int32_t *sel,
                      float *k_win, float *v_win, int32_t *win_len, reatt_stream stream);

/*
 * Windowed attention (decoding pseudocode: flash_attention(query, key_recall,
 * value_recall)).  Query c of head j is rotated at position W-C+c and attends
 * window rows p <= W-C+c of KV head j/(Hq/Hkv) with softmax(q.k/sqrt(d)).
 * k_win/v_win/win_len as written by reatt_gather_rope.  fp32 softmax and
 * accumulation; split over the window with an in-kernel combine.
 */
REATT_API int reatt_attend(const reatt_dims *dims, const void *q, const float *k_win, const float *v_win,
                 const int32_t *win_len, float *out, void *ws, reatt_stream stream);

/*
 * One whole step: score_spans -> topk -> attention over the virtual window.
 * The window is never materialised: the attention reads global, chosen and
 * local rows straight from the un-rotated cache (and the current tokens from
 * k_cur/v_cur) and rotates them in registers.  Equal, up to fp32 rounding
 * order, to reatt_score_spans + reatt_topk + reatt_gather_rope + reatt_attend.
 * sel_out (nullable): receives the selection [B,Hkv,k].
 * Appending the current tokens to the cache afterwards is the caller's job.
 */
REATT_API int reatt_step(const reatt_dims *dims, const void *q, const void *k_cache, const void *v_cache,
               const void *k_cur, const void *v_cur, int32_t *sel_out, float *out, void *ws,
               reatt_stream stream);

/*
 * Appends the C current tokens' K and V rows to the caches (the caller's step
 * after each reatt_step of a decoding loop or a chunked prefill; the pages'
 * prefilling and decoding pseudocode add the new keys and values to the cache
 * after the attention, ReAttention OpenReview discussion):
 *   k_cache[b,h,T+c,:] = k_cur[b,h,c,:], same for v, for c < C,
 * with cache rows at stride T_cap (dims->T_cap >= T + C, else EINVAL).
 * k_cur, v_cur [B,Hkv,C,d] in dims->dtype; all pointers 16-byte aligned.
 * The next call then uses dims with T + C.
 */
REATT_API int reatt_append_kv(const reatt_dims *dims, void *k_cache, void *v_cache,
                              const void *k_cur, const void *v_cur, reatt_stream stream);

/*
 * Diagnostic for the failure-detection path: launches one thread that waits
 * on an mbarrier nothing completes, bounded by limit_ns (0 < limit_ns <= 10 s),
 * after which it records REATT_ETIMEOUT in the workspace status word and
 * returns.  No fault, trap or hang; the context stays usable.  Read the
 * result with reatt_workspace_status().  EINVAL for a null/misaligned ws or
 * a limit out of range.
 */
REATT_API int reatt_selftest_bounded_wait(void *ws, int64_t limit_ns, reatt_stream stream);

/* ---------------------------------------------------------------------------
 * One sequence's cache split by token ranges over several GPUs ("shards").
 *
 * The research-map summary ("Limitations") and the OpenReview reply on W4
 * ("memory overhead tradeoff", 400K tokens on one GPU) name memory as the
 * method's only bound: the cache of one sequence can outgrow one GPU.  The
 * step then runs in three local phases with two small exchanges between
 * them, which the caller performs (e.g. an all-gather over NCCL):
 *
 *   1. reatt_shard_candidates  each shard scores the middle spans it holds
 *                              and keeps its own top-k (score, span id);
 *   -- exchange: every shard receives every shard's candidates --
 *   2. reatt_shard_select      every shard computes the same global top-k
 *                              from the candidates (the global top-k under
 *                              the order "score desc, id asc" lies inside
 *                              the union of the shards' top-k);
 *   3. reatt_shard_attend      each shard attends over the window rows it
 *                              holds, at their global window positions, and
 *                              writes an unnormalised partial (m, l, acc);
 *   -- exchange: every shard (or one) receives every shard's partial --
 *   4. reatt_merge_partials    out = sum_r 2^(m_r - M) acc_r /
 *                                    sum_r 2^(m_r - M) l_r,  M = max_r m_r.
 *
 * The result equals reatt_step on the whole cache, up to fp32 rounding order.
 * dims describe the WHOLE sequence (T = all cached tokens); `shard` says
 * which rows this GPU holds.  Shard r holds cache rows [t_begin, t_end) of
 * every (batch, KV head), stored at k_cache[((b*Hkv + h)*rows_cap + t -
 * t_begin)*d] (rows_cap = 0 means t_end - t_begin).  The shards, in rank
 * order, cover [0, T) without gaps; a boundary inside the middle must fall on
 * a span boundary (G + multiple of S); exactly one shard owns the current
 * tokens (owns_current = 1).  reatt_shard_plan makes such a split.  dims->T_cap
 * is ignored by these calls.  Span scoring of a shard with C > 1 runs on CUDA
 * cores (the tensor-core prefill scan is not used for shards).
 * --------------------------------------------------------------------------- */
typedef struct {
    int64_t t_begin;        /* first cached token (whole-sequence index) held here  */
    int64_t t_end;          /* one past the last                                     */
    int64_t rows_cap;       /* rows allocated per (b, KV head); 0 = t_end - t_begin   */
    int32_t owns_current;   /* 1 on exactly one shard: it attends the current tokens  */
    int32_t reserved;       /* 0                                                     */
} reatt_shard;

/* Splits [0, T) into n (1 <= n <= 1024) contiguous shards that hold nearly
 * equal numbers of middle spans (boundaries on span boundaries; the global
 * tokens go with shard 0, the local ones with the last shard, which also owns
 * the current tokens).  shards: n entries, written on success. */
REATT_API int reatt_shard_plan(const reatt_dims *dims, int32_t n, reatt_shard *shards);

/* Bytes of device workspace the shard calls of this shard need with
 * n_shards shards (a multiple of 256).  The status word sits at offset 0, as
 * in every workspace (reatt_workspace_status reads it). */
REATT_API int reatt_shard_workspace_bytes(const reatt_dims *dims, const reatt_shard *shard,
                                          int32_t n_shards, size_t *bytes);

/*
 * Phase 1 (decoding pseudocode: score = query . key[global:-local]^T,
 * idx_recall = score.topk, restricted to the spans this shard holds).  For
 * each (b, h): the min(k, NS_shard) best of this shard's middle spans (ties
 * to the lower id), as whole-sequence span ids in ascending order with their
 * fp32 scores; the remaining entries are (-inf, -1).
 *   q [B,Hq,C,d]; k_cache: this shard's rows; cand_score float [B,Hkv,k];
 *   cand_id int32 [B,Hkv,k].
 */
REATT_API int reatt_shard_candidates(const reatt_dims *dims, const reatt_shard *shard,
                                     const void *q, const void *k_cache, float *cand_score,
                                     int32_t *cand_id, void *ws, reatt_stream stream);

/*
 * Phase 2: the global top-k from every shard's candidates.
 *   cand_score_all float [n_shards, B, Hkv, k], cand_id_all int32 [n_shards,
 *   B, Hkv, k] (shard r's phase-1 output at index r, shards in token order)
 *   -> sel int32 [B, Hkv, k]: ascending span ids, -1 padded, exactly what
 *   reatt_topk gives on the whole sequence's span scores.
 */
REATT_API int reatt_shard_select(const reatt_dims *dims, int32_t n_shards,
                                 const float *cand_score_all, const int32_t *cand_id_all,
                                 int32_t *sel, void *ws, reatt_stream stream);

/*
 * Phase 3 (decoding pseudocode: attention over global ++ recalled ++ local;
 * "Approach": RoPE after the concatenation): the window rows this shard
 * holds (its global rows, its chosen spans, its local rows, the current
 * tokens if it owns them), each rotated at its position in the whole
 * window, against the queries rotated at W-C+c, causal, scale 1/sqrt(d).
 * Writes this shard's partial per query row (b, j, c):
 *   part_ml [B,Hq,C] float2 (m, l): m = max over visible keys of the logit
 *   times log2(e) (-inf when the shard holds no visible key), l = sum of
 *   2^(logit*log2(e) - m);
 *   part_acc [B,Hq,C,d] float: sum of 2^(logit*log2(e) - m) * v.
 * sel: the phase-2 selection.  k_cur/v_cur are read only by the shard that
 * owns the current tokens (others may pass them too; NULL is allowed there).
 */
REATT_API int reatt_shard_attend(const reatt_dims *dims, const reatt_shard *shard,
                                 const void *q, const void *k_cache, const void *v_cache,
                                 const void *k_cur, const void *v_cur, const int32_t *sel,
                                 void *part_ml, float *part_acc, void *ws, reatt_stream stream);

/*
 * Phase 4: the log-sum-exp merge of n_parts partials (n_parts >= 1):
 *   part_ml_all [n_parts,B,Hq,C] float2, part_acc_all [n_parts,B,Hq,C,d]
 *   -> out [B,Hq,C,d] float32.  A row that no part sees is written as 0.
 */
REATT_API int reatt_merge_partials(const reatt_dims *dims, int32_t n_parts,
                                   const void *part_ml_all, const float *part_acc_all,
                                   float *out, reatt_stream stream);

/*
 * reatt_step without a caller-supplied workspace.  The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory: a plugin interface that gives its kernels no allocator, or a
 * latency-critical loop where cudaMalloc would synchronize the device.
 *
 * Same arguments, results and errors as reatt_step, minus `ws`.  The
 * workspace is a 16 MiB (16 * 2^20 bytes) array in the library's device
 * globals, which every GPU that loads the library holds until the process
 * exits.  Calls whose reatt_workspace_bytes() exceeds 16 MiB return
 * REATT_EUNSUPPORTED before anything is launched.  For scale: the 128K
 * LLaMA3-8B-shaped decode needs 3.4 MiB, the 4M-token Qwen2-1.5B-shaped decode
 * 4.4 MiB, four 1M-token LLaMA3-8B-shaped sequences 7.4 MiB; a 2048-query
 * bf16 prefill chunk over 256K tokens needs 92.7 MiB (its tensor-core
 * attention operands) and is rejected.
 *   - Allocates nothing: no cudaMalloc/cudaFree or allocating library call.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress; nothing is cached, so the call stays valid after
 *     a cudaDeviceReset).  The first call on a device also loads the
 *     library's device globals there; make that first call before any stream
 *     capture.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents; what must start at zero is cleared inside each call.  Calls
 *     that overlap on the GPU race: order them on one stream.
 *   - A bounded-wait timeout is recorded in the shared array's status word
 *     (offset 0), like any workspace's: pass reatt_fixed_scratch_address()'s
 *     result to reatt_workspace_status() to read and clear it.
 */
REATT_API int reatt_step_fixed_scratch(const reatt_dims *dims, const void *q, const void *k_cache,
                                       const void *v_cache, const void *k_cur, const void *v_cur,
                                       int32_t *sel_out, float *out, reatt_stream stream);

/*
 * Device address of the fixed scratch that reatt_step_fixed_scratch uses, on
 * the current device (looked up on every call, like the step does; the first
 * call on a device loads the library's device globals there).  It is meant
 * for reatt_workspace_status() and reatt_selftest_bounded_wait(); the array's
 * other contents belong to the library and change with every fixed-scratch
 * step.  *ws_out is set only on REATT_OK.  EINVAL for a null ws_out, ECUDA if
 * the lookup fails.
 */
REATT_API int reatt_fixed_scratch_address(void **ws_out);

#ifdef __cplusplus
}
#endif

#endif /* REATT_H */
