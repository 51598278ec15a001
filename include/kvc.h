/*
 * kvc.h -- C ABI of libkvc, the B200 (sm_100a) hot path of observation-window
 * KV-cache compression: window saliency scoring, budgeted per-KV-head top-k,
 * compact KV gather, GQA decode attention over the compact cache, and
 * FastKV-style token-selective propagation (TSP); with FreeKV's decode-time
 * correction, per-layer budgets, an int8 compact cache, and xKV's cross-layer
 * factorisation with selective reconstruction.
 *
 * Sources of the method (web pages; the library implements their outline and
 * states its readings of the points they leave open):
 *   - "Variantes de l'attention et compression du cache KV" (nickwang.xyz):
 *     section "MHA et GQA" (head sharing, cache-size formula), section
 *     "Quand la reutilisation est-elle exacte ?" (causal offset of appended
 *     rows; original positions kept after eviction), section "Compresser un
 *     cache existant" (SnapKV observation-window scoring; sliding windows keep
 *     a recent region; PyramidKV's per-layer budgets; a cache stored at lower
 *     precision).
 *   - "FastKV: Decoupling of Context Reduction and KV Cache Compression for
 *     Prefill-Decoding Acceleration" (gist.science 2502.01068): section 2.A
 *     (token-selective propagation from window-attention saliency), section
 *     2.B (TSP rate independent of the KV retention rate).
 *   - "FreeKV: Boosting KV Cache Retrieval for Efficient LLM Inference"
 *     (gist.science 2505.13109), technical summary section 2.A (speculative
 *     retrieval with fine-grained correction) and section 2.B (NHD layout on
 *     the GPU, which every cache tensor here uses).
 *   - "xKV - Compression de Cache KV Inter-couche par Extraction de Vecteurs
 *     Singuliers Alignes" (gist.science 2503.18893), technical summary
 *     sections 2.2 (cross-layer factorisation) and 2.3 (selective
 *     reconstruction).
 *
 * Conventions shared by every entry point
 *   - All calls are asynchronous on the caller's stream (a cudaStream_t passed
 *     as kvc_stream_t; NULL is the legacy default stream).  No call allocates,
 *     frees or synchronises; no call reads device memory on the host.
 *   - The caller owns every buffer.  Device pointers must be 16-byte aligned
 *     and dense in the layouts stated below.  Host pointers are read during the
 *     call only.
 *   - Scratch memory is a caller-provided device workspace whose size comes
 *     from the matching *_workspace_size() query; it may be reused between
 *     calls on the same stream.  The score and decode workspaces hold
 *     counters that must be zero before their first use (cudaMemset to 0
 *     once); every call leaves them zero again.  The first int32 of every
 *     workspace is a device error word: a kernel whose bounded wait gave up
 *     (a pipeline or another CTA did not answer in time) sets it nonzero and
 *     stops waiting instead of hanging; that call's results are invalid.
 *     After such a call, zero the workspace again before reusing it.
 *   - Ragged batches: n_seqs sequences packed along the token axis; seqlens_host
 *     (host int32[n_seqs]) gives the lengths, cu_seqlens (device int32[n_seqs+1])
 *     their prefix sums starting at 0.  Both must describe the same batch.
 *   - Layouts: K, V, compact K_c/V_c: [rows, n_kv, d_h] (NHD).  Window queries
 *     q_win: [n_seqs * w, n_h, d_h], the last w query rows of each sequence in
 *     order.  Scores: float32 [n_kv, T], T = sum of lengths.  Index lists:
 *     int32 [n_kv, sum_b min(budget, len_b)], sequence b's segment starting at
 *     cu_budget[b].
 *   - GQA: query head qh attends with KV head qh / (n_h / n_kv).
 *   - scale <= 0 selects 1/sqrt(d_h).
 *   - Errors: validation failures return before anything is launched and set a
 *     thread-local message readable with kvc_last_error().  A failed launch
 *     returns KVC_ERR_CUDA; work already enqueued by that call is not undone.
 */
#ifndef KVC_H_
#define KVC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvc_stream_t; /* identical to cudaStream_t */

typedef enum kvc_status {
  KVC_OK = 0,
  KVC_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or count */
  KVC_ERR_UNSUPPORTED = 2,  /* valid request outside the kernels' shapes/dtypes */
  KVC_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
  KVC_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  KVC_ERR_DEVICE_CHECK = 5  /* a workspace's device error word is set (kvc_check_workspace) */
} kvc_status;

typedef enum kvc_dtype {
  KVC_F32 = 0,   /* IEEE binary32 */
  KVC_BF16 = 1   /* bfloat16 */
} kvc_dtype;

/* Library version: major * 10000 + minor * 100 + patch. */
int kvc_version(void);

/* Number of kernels this library has enqueued in this process (kernels
 * recorded into a CUDA graph under stream capture count once, at capture).
 * For launch accounting by callers; the pages have no counterpart. */
int64_t kvc_launch_count(void);

/* Read a workspace's device error word (its first int32).  The one
 * synchronous call of the library: it waits for `stream`, then copies the
 * word to the host; it allocates nothing.  Returns KVC_OK when the word is
 * zero, KVC_ERR_DEVICE_CHECK when a kernel that used this workspace gave up
 * a bounded wait (the results of the calls since the workspace was last
 * zeroed are invalid; zero it again before reuse), KVC_ERR_INVALID_ARG for a
 * NULL or misaligned ws, KVC_ERR_CUDA when the copy or the wait failed. */
kvc_status kvc_check_workspace(const void *ws, kvc_stream_t stream);

/* Static text for a status code. */
const char *kvc_status_string(int status);

/* Message of the last failing call on this thread ("" if none). */
const char *kvc_last_error(void);

/*
 * Bytes of a K+V cache for one sequence: 2 * L * S * n_kv * d_h * b.
 * The factor 2 counts keys and values ("MHA et GQA" on the attention-variants
 * page; its worked example L=32, S=4096, n_kv=8, d_h=128, b=2 gives
 * 536,870,912).  Returns 0 if an argument is negative.  Host only.
 */
uint64_t kvc_cache_bytes(int L, int64_t S, int n_kv, int d_h, int b);

/*
 * Host helper: cu_budget_host[0] = 0, cu_budget_host[b+1] = cu_budget_host[b]
 * + min(budget, seqlens_host[b]).  cu_budget_host has n_seqs + 1 entries.
 * Returns the total (the compact-cache row count) or -1 on invalid input.
 */
int64_t kvc_budget_offsets(int n_seqs, const int32_t *seqlens_host, int budget,
                           int32_t *cu_budget_host);

/*
 * PyramidKV per-layer budgets (host only).  Source: "Variantes de l'attention
 * et compression du cache KV", section "Compresser un cache existant":
 * PyramidKV gives different layers different cache budgets.  The page gives no
 * shape; this library's reading is the arithmetic sequence falling from
 * B_max = 2 * avg_budget - min_budget at layer 0 to min_budget at layer L - 1:
 *   budgets_host[l] = B_max - floor((B_max - min_budget) * l / (L - 1))
 * (L == 1: avg_budget), so the mean is avg_budget, rounded up by less than one
 * token per layer.  Each layer then calls kvc_compress_window with its own
 * budget.  Returns the sum of the budgets, or -1 on invalid input (L < 1,
 * min_budget < 0, min_budget > avg_budget, NULL output).
 */
int64_t kvc_pyramid_budgets(int L, int avg_budget, int min_budget, int32_t *budgets_host);

/* ------------------------------------------------------------------------
 * Window saliency scores (SnapKV observation window; FastKV 2.A saliency).
 *
 * For sequence b (length len_b >= w, prefix P_b = len_b - w), KV head h,
 * query head g of h's group and window row i (position P_b + i), with logits
 * z_j = scale * q . k_j over the visible keys j <= P_b + i (causal rule of the
 * attention-variants page, "Quand la reutilisation est-elle exacte ?"):
 *   raw[h][t0 + j]    = sum_{g, i} softmax_j(z)      for every j < len_b
 *   scores[h][t0 + j] = max_{|t| <= r, 0 <= j+t < P_b} raw[h][t0 + j + t]
 *                       for j < P_b (r = (pool_k - 1) / 2), and +inf on the
 *                       window positions j >= P_b (always retained).
 * The softmax is exact (two passes over K: row max/sum, then probabilities).
 *
 * dt: KVC_F32 or KVC_BF16 for q_win and k.  d_h in {64, 128}.  n_h % n_kv == 0,
 * G = n_h / n_kv; the window block has G * w <= 256 rows (and a multiple of 16
 * rows for KVC_BF16).  pool_k odd in [1, 31].  scores_raw may be NULL.
 * q_win: [n_seqs * w, n_h, d_h];  k: [T, n_kv, d_h];  scores, scores_raw:
 * float32 [n_kv, T].  ws: kvc_score_window_workspace_size() bytes, zeroed
 * before its first use (it holds per-(sequence, head) arrival counters).
 * When every (sequence, head, key chunk) work item fits on the GPU at once,
 * KVC_BF16 scoring runs as one cooperative launch (both passes and the pool);
 * otherwise as three launches.  Results are the same either way.
 * ------------------------------------------------------------------------ */
size_t kvc_score_window_workspace_size(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host,
                                       int n_h, int n_kv, int d_h, int w);
kvc_status kvc_score_window(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host,
                            const int32_t *cu_seqlens, int n_h, int n_kv, int d_h, int w,
                            int pool_k, float scale, const void *q_win, const void *k,
                            float *scores, float *scores_raw, void *ws, size_t ws_bytes,
                            kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * kvc_compress_window: kvc_score_window, kvc_select_topk and kvc_gather_kv in
 * one call, with the same arguments, layouts and results as the three calls
 * in sequence (plus v, idx, k_out, v_out, budget and cu_budget of the latter
 * two).  KVC_BF16 batches whose every (sequence, head, key chunk) work item
 * fits on the GPU at once, with key chunks of at most 32768 keys, run it as
 * ONE cooperative launch: after the pool, the CTAs of each (sequence, head)
 * find the budgeted top-k together (a three-level radix select through small
 * per-head histograms in the workspace) and each gathers the rows it kept.
 * Other batches run the three calls.  ws: kvc_score_window_workspace_size()
 * bytes, zeroed before its first use.  The pages define the three steps
 * (SnapKV observation window, "Variantes de l'attention et compression du
 * cache KV", section "Compresser un cache existant"); fusing them is this
 * library's.
 * ------------------------------------------------------------------------ */
kvc_status kvc_compress_window(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host,
                               const int32_t *cu_seqlens, const int32_t *cu_budget, int n_h, int n_kv,
                               int d_h, int w, int pool_k, int budget, float scale, const void *q_win,
                               const void *k, const void *v, float *scores, float *scores_raw,
                               int32_t *idx, void *k_out, void *v_out, void *ws, size_t ws_bytes,
                               kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * Budgeted per-KV-head top-k.  Source: "Variantes de l'attention et
 * compression du cache KV", section "Compresser un cache existant" (SnapKV
 * keeps a chosen subset of past keys and values; windowed attention keeps a
 * bounded recent region, here the w window tokens), and section "Quand la
 * reutilisation est-elle exacte ?" (positions keep their original indices
 * after eviction, never renumbered).
 *
 * For sequence b and KV head h: if budget >= len_b the segment is 0..len_b-1.
 * Otherwise it holds the budget - w prefix positions with the largest
 * scores[h][t0 + j], j < P_b (ties: lower position first), in ascending order,
 * followed by P_b .. len_b - 1.  Positions are sequence-local originals
 * (never renumbered).  Scores are compared as float32 with NaN above +inf.
 *
 * budget >= w >= 1.  cu_budget: device int32[n_seqs + 1] from
 * kvc_budget_offsets().  scores: float32 [n_kv, T] (as written by
 * kvc_score_window).  idx: int32 [n_kv, cu_budget[n_seqs]].
 * ------------------------------------------------------------------------ */
kvc_status kvc_select_topk(int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                           const int32_t *cu_budget, int n_kv, int w, int budget,
                           const float *scores, int32_t *idx, kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * Compact cache gather.  Source: "Variantes de l'attention et compression du
 * cache KV", section "Compresser un cache existant" (the retained keys and
 * values form the compressed cache); NHD layout of GPU caches from the FreeKV
 * page, technical summary section 2.B.  For each sequence b, KV head h and
 * slot t < min(budget, len_b):
 *   K_c[cb_b + t][h][:] = K[t0_b + idx[h][cb_b + t]][h][:]
 * and likewise for V (bytes copied unchanged, so the copy is exact).
 *
 * k, v: [T, n_kv, d_h];  k_out, v_out: [cu_budget[n_seqs], n_kv, d_h];  idx
 * as written by kvc_select_topk (every entry must lie in [0, len_b)).
 * ------------------------------------------------------------------------ */
kvc_status kvc_gather_kv(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host,
                         const int32_t *cu_seqlens, const int32_t *cu_budget, int n_kv, int d_h,
                         int budget, const int32_t *idx, const void *k, const void *v,
                         void *k_out, void *v_out, kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * FastKV token-selective propagation for one sequence of S tokens (FastKV
 * 2.A; its rate is independent of the KV budget, 2.B):
 *   agg[j]    = sum_{r < n_rows} scores_raw[r][j]          for j < P = S - w
 *   pooled[j] = max_{|t| <= (pool_k-1)/2, 0 <= j+t < P} agg[j + t]
 *   idx_out   = the k_tsp prefix positions with the largest pooled value
 *               (ties: lower position), ascending, then P .. S-1
 *   hidden_out[t][:] = hidden[idx_out[t]][:]   (k_tsp + w rows of D elements)
 * scores_raw: float32 [n_rows, S] (the raw output of kvc_score_window for one
 * sequence; summing its KV-head rows sums all query heads).  hidden: [S, D] of
 * dt, D % 8 == 0.  idx_out: int32 [k_tsp + w].  0 <= k_tsp <= S - w.
 * ws: kvc_tsp_workspace_size() bytes.
 * ------------------------------------------------------------------------ */
size_t kvc_tsp_workspace_size(int S, int w);
kvc_status kvc_tsp_select_gather(kvc_dtype dt, int S, int n_rows, int w, int pool_k, int k_tsp,
                                 const float *scores_raw, const void *hidden, int D,
                                 int32_t *idx_out, void *hidden_out, void *ws, size_t ws_bytes,
                                 kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * kvc_tsp_select_gather_static: the same computation as
 * kvc_tsp_select_gather, for callers that cannot allocate device memory for a
 * workspace (code that must not touch the process' device allocator, e.g.
 * running inside another component's memory pool or out-of-memory handler,
 * or a serving loop that forbids allocations).  The pages have no
 * counterpart: this is an interface convenience of the library.
 *
 * Scratch: a fixed array inside the library (1 MiB, every GPU that loads the
 * library keeps it until the process exits).  S - w must not exceed 262,144;
 * larger requests return KVC_ERR_UNSUPPORTED (use the workspace variant).
 * The first call on a device resolves the array's device address for that
 * device; make that first call before any stream capture.  All calls on one
 * device share that device's array, which keeps the last call's contents:
 * calls whose kernels can overlap on the GPU (for instance on different
 * streams) race, so keep them on one stream or synchronise them.  Nothing in
 * the array has to start at zero.  The call allocates and frees nothing.
 * Other arguments, layouts and errors are those of kvc_tsp_select_gather.
 * ------------------------------------------------------------------------ */
kvc_status kvc_tsp_select_gather_static(kvc_dtype dt, int S, int n_rows, int w, int pool_k, int k_tsp,
                                        const float *scores_raw, const void *hidden, int D,
                                        int32_t *idx_out, void *hidden_out, kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * GQA decode attention over compact caches (decode reads the whole cache per
 * step: FastKV section 1; attention-variants page introduction):
 *   out[b][qh][:] = sum_{t < kv_len[b]} softmax_t(scale * q[b][qh] . Kc[o_b + t][h])
 *                   * Vc[o_b + t][h],   h = qh / G,  o_b = kv_row_offset[b]
 * and 0 when kv_len[b] == 0.  Offsets may alias (several queries on one cache).
 *
 * q: [batch, n_h, d_h] of dt;  k_c, v_c: [cache_rows, n_kv, d_h] of dt, with
 * kv_row_offset[b] + kv_len[b] <= cache_rows (cache_rows < 2^31);
 * kv_row_offset: device int64[batch];  kv_len: device int32[batch], each
 * <= max_kv_len;  out: float32 [batch, n_h, d_h].  G in {1, 2, 4, 8};
 * d_h in {64, 128}.  ws: kvc_gqa_decode_workspace_size() bytes, counters
 * zeroed before first use (see conventions).
 * ------------------------------------------------------------------------ */
size_t kvc_gqa_decode_workspace_size(int batch, int n_h, int n_kv, int d_h, int max_kv_len);
kvc_status kvc_gqa_decode_attn(kvc_dtype dt, int batch, int n_h, int n_kv, int d_h, float scale,
                               const void *q, const void *k_c, const void *v_c, int64_t cache_rows,
                               const int64_t *kv_row_offset, const int32_t *kv_len,
                               int max_kv_len, float *out, void *ws, size_t ws_bytes,
                               kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * Quantised compact cache.  Source: "Variantes de l'attention et compression
 * du cache KV", section "Compresser un cache existant" (KV-cache quantisation
 * stores the cache elements at a lower precision; custom layouts need their
 * own kernels).  Format: int8 codes in the compact cache's NHD layout
 * [rows, n_kv, d_h] plus one float32 scale per (row, head) in
 * [n_kv, scale_pitch]; the value a code stands for is code * scale.
 *
 * kvc_gather_kv_q8: the gather of kvc_gather_kv from bf16 caches k, v, and
 * for every retained (slot, head) vector x: scale = max|x| / 127 and code =
 * round-half-even(x / scale) clipped to [-127, 127], both quotients IEEE
 * float32 divisions (a zero vector: scale 0, codes 0).  k_q, v_q: int8
 * [cu_budget[n_seqs], n_kv, d_h]; k_scale, v_scale: float32 [n_kv,
 * scale_pitch], scale_pitch >= cu_budget[n_seqs].  d_h in {64, 128}.
 * ------------------------------------------------------------------------ */
kvc_status kvc_gather_kv_q8(int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                            const int32_t *cu_budget, int n_kv, int d_h, int budget, const int32_t *idx,
                            const void *k, const void *v, int8_t *k_q, int8_t *v_q, float *k_scale,
                            float *v_scale, int64_t scale_pitch, kvc_stream_t stream);

/* kvc_gqa_decode_attn_q8: kvc_gqa_decode_attn over int8 caches, with the
 * logits and weights of the dequantised values code * scale (the K scale of
 * a row multiplies its logit, the V scale its weight).  q: bf16 [batch, n_h,
 * d_h]; k_q, v_q: int8 [cache_rows, n_kv, d_h]; k_scale, v_scale: float32
 * [n_kv, scale_pitch], scale_pitch >= cache_rows.  Other arguments, the
 * workspace (kvc_gqa_decode_workspace_size) and errors as kvc_gqa_decode_attn. */
kvc_status kvc_gqa_decode_attn_q8(int batch, int n_h, int n_kv, int d_h, float scale, const void *q,
                                  const int8_t *k_q, const int8_t *v_q, const float *k_scale,
                                  const float *v_scale, int64_t scale_pitch, int64_t cache_rows,
                                  const int64_t *kv_row_offset, const int32_t *kv_len, int max_kv_len,
                                  float *out, void *ws, size_t ws_bytes, kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * FreeKV decode step with fine-grained correction.  Source: "FreeKV: Boosting
 * KV Cache Retrieval for Efficient LLM Inference", technical summary section
 * 2.A ("Recuperation Speculative": a step reuses the tokens retrieved for the
 * previous step; "Correction Fine": the heads whose query similarity to the
 * previous step falls below tau are selected and retrieved again before
 * attention).  All caches stay in device memory (the page's CPU offload is
 * not part of this library).
 *
 * For sequence b and KV head h (query heads h*G .. h*G+G-1):
 *   reselected[b][h] = 1 if min_g cos(q_cur[b][hG+g], q_prev[b][hG+g]) < tau
 *                      (cos = 0 when a vector is zero), else 0;
 *   if reselected: its index list is replaced by the budgeted selection (the
 *     rule of kvc_select_topk: w most recent tokens kept, max-pooled prefix
 *     scores, lowest position first on ties) over the scores
 *     raw[j] = sum_g softmax_j(scale * q_cur[b][hG+g] . k_j), j < len_b (the
 *     decode query sees every cached key), max-pooled over [0, len_b - w);
 *     its rows of k_c / v_c are gathered again;
 *   otherwise idx, k_c and v_c keep their contents for that head;
 *   out[b] = kvc_gqa_decode_attn of q_cur[b] over the compact cache rows
 *     [cu_budget[b], cu_budget[b+1]) of every head.
 * Heads whose flag is 0 read no full-cache key.
 *
 * bf16 only; d_h in {64, 128}; G in {1, 2, 4, 8}.  q_cur, q_prev: [batch,
 * n_h, d_h]; k, v: full caches [T, n_kv, d_h] (cu_seqlens, len_b >= w);
 * cu_budget from kvc_budget_offsets(budget); idx: int32 [n_kv,
 * cu_budget[batch]] and k_c, v_c: [cu_budget[batch], n_kv, d_h], in/out
 * (hold the previous step's selection; on the first step pass tau > 1 so
 * that every head is selected); reselected: int32 [batch, n_kv], out;
 * out: float32 [batch, n_h, d_h].  ws: kvc_freekv_workspace_size() bytes,
 * zeroed before its first use (decode counters, left zero by every call).
 * ------------------------------------------------------------------------ */
size_t kvc_freekv_workspace_size(int batch, const int32_t *seqlens_host, int n_h, int n_kv, int d_h, int w,
                                 int budget);
kvc_status kvc_freekv_step(int batch, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                           const int32_t *cu_budget, int n_h, int n_kv, int d_h, int w, int pool_k, int budget,
                           float tau, float scale, const void *q_cur, const void *q_prev, const void *k,
                           const void *v, int32_t *idx, void *k_c, void *v_c, int32_t *reselected, float *out,
                           void *ws, size_t ws_bytes, kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * xKV cross-layer factorisation and selective reconstruction.  Source: "xKV -
 * Compression de Cache KV Inter-couche par Extraction de Vecteurs Singuliers
 * Alignes" (gist.science 2503.18893), technical summary section 2.2
 * ("Factorisation Inter-couche": the caches of a window of W consecutive
 * layers are concatenated along the features, a rank-r SVD of the result
 * gives a token basis shared by the window and one reconstruction matrix per
 * layer) and section 2.3 ("Reconstruction Selective": only the rows of the
 * chosen tokens are rebuilt, from the shared basis and the layer's matrix).
 *
 * One sequence of S tokens; the factorisation is per KV head h:
 *   X_h = [K_0[:, h] | K_1[:, h] | ... | K_{W-1}[:, h]]   (S x F, F = W d_h)
 *   Vt_h (r x F) spans the top-r right singular subspace of X_h (orthonormal
 *     rows), A_h = X_h Vt_h^T (S x r), so A_h Vt_h is the rank-r truncated SVD
 *     of X_h; layer l's reconstruction matrix is Vt_h[:, l d_h : (l+1) d_h].
 * The subspace is computed by `iters` steps of subspace iteration on the
 * Gram matrix X_h^T X_h (float32, bf16 products) from the start basis v0,
 * each step re-orthonormalised by Cholesky-QR in float64.  Its distance to
 * the exact singular subspace shrinks like (s_{r+1} / s_r)^(2 iters) (s: the
 * singular values of X_h) down to float32 resolution; where s_r = s_{r+1} the
 * subspace is not unique and any converged one is valid.  A_h and Vt_h are
 * unique only up to a rotation of the r basis vectors; A_h Vt_h is unique.
 *
 * kvc_xkv_factorize: bf16 only.  d_h in {64, 128}; 1 <= W <= 8; W d_h <= 512;
 * r in {16, 32, 64}, r <= min(S, W d_h); 1 <= iters <= 1000.
 *   k_layers: host array of W device pointers, each bf16 [S, n_kv, d_h] (the
 *     keys of the window's layers; values are factorised the same way by a
 *     second call).
 *   v0: float32 [n_kv, W d_h, r] start basis (e.g. Gaussian; its columns must
 *     not be orthogonal to the top-r subspace).
 *   basis_dt: KVC_F32 or KVC_BF16 (round to nearest even) for A.
 *   basis: [n_kv, S, r] of basis_dt (A_h);  blocks: float32 [n_kv, r, W d_h]
 *     (Vt_h).  ws: kvc_xkv_workspace_size() bytes; no zeroing needed.
 *
 * kvc_xkv_reconstruct: rows idx[h][t] (t < n_sel) of layer `layer`:
 *   out[t][h][:] = bf16_rn( A_h[idx[h][t]] Vt_h[:, layer d_h : (layer+1) d_h] )
 *   idx: int32 [n_kv, n_sel] (e.g. a kvc_select_topk segment); an index
 *   outside [0, S) yields a zero row.  out: bf16 [n_sel, n_kv, d_h], the
 *   layout of a compact cache, ready for kvc_gqa_decode_attn.  Shapes and
 *   basis_dt as given to kvc_xkv_factorize.
 * Both calls are asynchronous on `stream`; errors as for every entry point.
 * ------------------------------------------------------------------------ */
size_t kvc_xkv_workspace_size(int S, int n_kv, int d_h, int W, int r);
kvc_status kvc_xkv_factorize(int S, int n_kv, int d_h, int W, int r, int iters, const void *const *k_layers,
                             const float *v0, kvc_dtype basis_dt, void *basis, float *blocks, void *ws,
                             size_t ws_bytes, kvc_stream_t stream);
kvc_status kvc_xkv_reconstruct(int S, int n_kv, int d_h, int W, int r, int layer, int n_sel, kvc_dtype basis_dt,
                               const void *basis, const float *blocks, const int32_t *idx, void *out,
                               kvc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H_ */
