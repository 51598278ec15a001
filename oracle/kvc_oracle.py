"""Plain fp64 CPU oracle for observation-window KV-cache compression.

TEST INFRASTRUCTURE.  Only the test-suite, the package smoke check and the
bench's CPU-baseline and reference legs may import this module.  The CUDA
library never calls it and shares no code with it.

What it computes, step by step, in float64 from the stored inputs (fp32 values
or bf16 bit patterns, both widened exactly):

1. ``window_probs`` -- for each sequence b, KV head h, query head g of the GQA
   group of h and window row i (absolute position p = len_b - w + i): the
   logits z_j = scale * q . k_j for the keys j <= p, and the softmax
   pi_j = exp(z_j - max z) / sum exp(z - max z).  Observation-window scoring of
   SnapKV ("Variantes de l'attention et compression du cache KV", section
   "Compresser un cache existant"); FastKV's saliency from the attention of the
   recent window (FastKV, section 2.A).  The causal rule -- row i of a q-row
   segment appended after S cached tokens sees keys up to S + i -- is from the
   same attention-variants page, section "Quand la reutilisation est-elle
   exacte ?".
2. ``raw_scores`` -- raw[h][j] = sum over the G heads and w rows of pi_j.
3. ``pool_prefix`` -- 1-D max-pool of raw over the prefix [0, P), P = len - w.
4. ``select_topk`` -- per KV head the B - w prefix positions with the largest
   pooled score (ties: lower index first), ascending, then the w window
   positions.  Original positions are kept, never renumbered (attention-variants
   page, section "Quand la reutilisation est-elle exacte ?").
5. ``gather_kv`` -- byte copy of the retained rows into a compact cache.
6. ``gqa_decode`` -- textbook softmax attention of one query per head over the
   retained rows of its KV head (GQA head sharing: attention-variants page,
   section "MHA et GQA").
7. ``tsp_select`` / ``tsp_gather`` -- FastKV token-selective propagation
   (FastKV, section 2.A): scores summed over all heads, pooled, one token set
   of k_tsp prefix positions plus the window, hidden rows copied.
8. ``cache_bytes`` -- 2 * L * S * n_kv * d_h * b (attention-variants page,
   section "MHA et GQA").
9. ``quantize_rows_int8`` / ``gather_kv_q8`` / ``gqa_decode_q8`` -- the KV cache
   stored at lower precision (attention-variants page, section "Compresser un
   cache existant": cache quantisation): every retained (row, head) vector is
   stored as int8 codes with one float32 scale, and decode attention runs over
   the dequantised values.
11. ``freekv_flags`` / ``decode_query_scores`` / ``freekv_step`` -- FreeKV's
   decode-time retrieval with fine-grained correction (FreeKV, technical
   summary 2.A): a step reuses the token set retrieved for the previous step;
   a KV head whose query has drifted -- cosine similarity between the current
   and the previous query below tau -- is scored again with the current
   query, its tokens are selected again and retrieved before attention.
12. ``xkv_factorize`` / ``xkv_reconstruct`` -- xKV cross-layer factorisation
   and selective reconstruction (xKV, sections 2.2 and 2.3): the keys of a
   window of W consecutive layers, concatenated along the feature axis, get a
   rank-r truncated SVD X ~ U_r S_r V_r^T; the window keeps the shared token
   basis A = U_r S_r = X V_r and one reconstruction block B_l (rows l*d ..
   (l+1)*d of V_r, transposed) per layer; selective reconstruction rebuilds
   only the chosen rows, K_l[idx] ~ A[idx] B_l.
10. ``pyramid_budgets`` -- PyramidKV's per-layer cache budgets (attention-variants
   page, section "Compresser un cache existant": different layers get different
   budgets): a budget that falls linearly from the first layer to the last
   around a given mean.

Every function above is pinned by tests/test_oracle_pins.py (closed forms,
invariants, the pages' worked cache-size example, brute force on tiny inputs,
library cross-checks).  The readings below are choices, not facts from the
pages: parity is unpinned for them.

Readings of points the pages leave open:
* logit scale: passed explicitly, 1/sqrt(d_h) by default;
* GQA mapping: query head qh uses KV head qh // G (contiguous groups);
* softmax domain: the whole visible row, window keys included; only prefix
  positions are pooled and selected;
* order: sum over heads and rows first, then pool;
* pool: stride 1, same length, neighbours outside [0, P) ignored;
* the per-head budget B counts the window (B - w prefix positions);
  the TSP count k_tsp does not (k_tsp + w rows);
* B >= len keeps every position; B < w is rejected; even pool sizes rejected;
* PyramidKV schedule (the page gives no shape): for L layers, a mean budget
  B_avg and a last-layer budget B_min <= B_avg, layer l keeps
  B_max - floor((B_max - B_min) * l / (L - 1)) tokens per KV head, with
  B_max = 2 * B_avg - B_min -- the arithmetic sequence from B_max down to B_min
  whose mean is B_avg, rounded so that the total is never below L * B_avg;
  a single layer keeps B_avg;
* FreeKV: the similarity of a KV head is the smallest cosine over the query
  heads of its group (cosine 0 when a vector is zero); the head is corrected
  when it is below tau.  A corrected head is scored as in the observation
  window, with the current decode query as the only window row, seeing every
  cached key: raw[j] = sum over the group of softmax_j(scale * q . k_j); the
  same pool over the prefix [0, len - w) and the same budgeted selection (the
  w most recent tokens always kept) then pick its tokens.  Heads above tau
  keep their index list (and compact rows); decode attention then runs over
  every head's compact cache;
* xKV: the factorisation is per (sequence, KV head) -- X_h = [K_1[:, h] | ...
  | K_W[:, h]] of shape [S, W * d_h] -- and applies to the keys (values
  alike); the chosen rows are an input (an index list per KV head, e.g. the
  library's budgeted selection); reconstructed rows are stored as bf16
  (round to nearest even) for decode;
* quantised cache: symmetric int8 per (row, head) vector, scale = max|x| / 127
  and code = round-half-even(x / scale), both quotients in float32 (the
  precision the stored values have), codes clipped to [-127, 127]; an all-zero
  vector has scale 0 and codes 0.  Dequantised value = code * scale.

Parity pins for every function live in tests/test_oracle_pins.py; none of them
re-types these formulas.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------
# inputs
# ----------------------------------------------------------------------------
def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored representation -> float64 (exact for fp32 and for bf16 bits)."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        bits = np.asarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32).astype(np.float64)
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def default_scale(d_h: int) -> float:
    return 1.0 / np.sqrt(float(d_h))


# ----------------------------------------------------------------------------
# 8. cache size
# ----------------------------------------------------------------------------
def cache_bytes(L: int, S: int, n_kv: int, d_h: int, b: int) -> int:
    """Bytes of a K+V cache for one sequence: two tensors (K and V) of
    L layers x S tokens x n_kv heads x d_h elements x b bytes."""
    return 2 * int(L) * int(S) * int(n_kv) * int(d_h) * int(b)


# ----------------------------------------------------------------------------
# 1-2. window probabilities and raw scores
# ----------------------------------------------------------------------------
def window_probs(q_rows: np.ndarray, k_head: np.ndarray, w: int, scale: float):
    """Softmax rows of the observation window for one (sequence, KV head).

    q_rows: [G, w, d] float64 -- the window queries of the G query heads that
            share this KV head, row i at absolute position len - w + i.
    k_head: [len, d] float64 -- every cached key of this KV head.
    Returns (pi [G, w, len], m [G, w], l [G, w]) with pi zero on masked keys;
    m is the row maximum of the visible logits and l the sum of exp(z - m).
    """
    G, w_, d = q_rows.shape
    assert w_ == w
    length = k_head.shape[0]
    z = scale * (q_rows.reshape(G * w, d) @ k_head.T).reshape(G, w, length)
    pos = (length - w) + np.arange(w)                        # absolute row positions
    visible = np.arange(length)[None, :] <= pos[:, None]     # [w, len]
    z = np.where(visible[None, :, :], z, -np.inf)
    m = z.max(axis=2)
    e = np.exp(z - m[:, :, None])                            # exp(-inf) = 0
    l = e.sum(axis=2)
    return e / l[:, :, None], m, l


def raw_scores(q_win: np.ndarray, k: np.ndarray, cu_seqlens, n_h: int, n_kv: int, w: int,
               dtype: str, scale: float | None = None) -> np.ndarray:
    """raw[h, t] for every packed token t: the softmax mass that the window rows
    of the G query heads of KV head h put on token t (window tokens included,
    where the causal mask applies).  Shape [n_kv, T], float64.

    q_win: [n_seqs * w, n_h, d] stored;  k: [T, n_kv, d] stored.
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    n_seqs = len(cu) - 1
    d = k.shape[2]
    if scale is None or scale <= 0:
        scale = default_scale(d)
    G = n_h // n_kv
    qf = to_f64(q_win, dtype)
    kf = to_f64(k, dtype)
    out = np.zeros((n_kv, int(cu[-1])), dtype=np.float64)
    for b in range(n_seqs):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        qb = qf[b * w:(b + 1) * w]                            # [w, n_h, d]
        for h in range(n_kv):
            q_rows = np.transpose(qb[:, h * G:(h + 1) * G, :], (1, 0, 2))   # [G, w, d]
            pi, _, _ = window_probs(q_rows, kf[t0:t1, h, :], w, scale)
            out[h, t0:t1] = pi.sum(axis=(0, 1))
    return out


def row_stats(q_win: np.ndarray, k: np.ndarray, cu_seqlens, n_h: int, n_kv: int, w: int,
              dtype: str, scale: float | None = None):
    """(m, l) of every window row, shapes [n_seqs, n_h, w]: m = max visible
    logit (natural-log units), l = sum over visible keys of exp(z - m)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    n_seqs = len(cu) - 1
    d = k.shape[2]
    if scale is None or scale <= 0:
        scale = default_scale(d)
    G = n_h // n_kv
    qf = to_f64(q_win, dtype)
    kf = to_f64(k, dtype)
    m_all = np.zeros((n_seqs, n_h, w))
    l_all = np.zeros((n_seqs, n_h, w))
    for b in range(n_seqs):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        qb = qf[b * w:(b + 1) * w]
        for h in range(n_kv):
            q_rows = np.transpose(qb[:, h * G:(h + 1) * G, :], (1, 0, 2))
            _, m, l = window_probs(q_rows, kf[t0:t1, h, :], w, scale)
            m_all[b, h * G:(h + 1) * G] = m
            l_all[b, h * G:(h + 1) * G] = l
    return m_all, l_all


# ----------------------------------------------------------------------------
# 3. pooling
# ----------------------------------------------------------------------------
def maxpool1d_same(x: np.ndarray, pool_k: int) -> np.ndarray:
    """out[j] = max of x[j + t] over |t| <= (pool_k - 1) / 2 with 0 <= j + t < len(x)."""
    if pool_k < 1 or pool_k % 2 == 0:
        raise ValueError("pool_k must be odd and >= 1")
    r = (pool_k - 1) // 2
    n = x.shape[0]
    out = x.copy()
    for t in range(1, r + 1):
        out[:n - t] = np.maximum(out[:n - t], x[t:])        # right neighbour j + t
        out[t:] = np.maximum(out[t:], x[:n - t])            # left neighbour j - t
    return out


def pool_prefix(raw: np.ndarray, cu_seqlens, w: int, pool_k: int) -> np.ndarray:
    """Pooled scores [n_kv, T]: on each sequence's prefix [0, P) the max-pool of
    raw over that prefix; window positions carry +inf (always retained)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    out = np.full_like(raw, np.inf)
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        P = max(t1 - t0 - w, 0)
        for h in range(raw.shape[0]):
            out[h, t0:t0 + P] = maxpool1d_same(raw[h, t0:t0 + P], pool_k)
    return out


# ----------------------------------------------------------------------------
# 4. selection
# ----------------------------------------------------------------------------
def budget_offsets(seqlens, budget: int) -> np.ndarray:
    """cu_budget: prefix sums of min(budget, len_b), int64, length n_seqs + 1."""
    kept = np.minimum(np.asarray(seqlens, dtype=np.int64), int(budget))
    out = np.zeros(len(kept) + 1, dtype=np.int64)
    out[1:] = np.cumsum(kept)
    return out


def topk_prefix(scores: np.ndarray, k_sel: int) -> np.ndarray:
    """The k_sel positions with the largest scores (ties: lower index first),
    returned in ascending position order."""
    order = np.argsort(-scores, kind="stable")               # descending score, index asc on ties
    return np.sort(order[:k_sel])


def select_one(pooled_prefix: np.ndarray, length: int, w: int, budget: int) -> np.ndarray:
    """Retained positions of one (sequence, KV head): ascending prefix winners,
    then the window P..len-1; all positions when budget >= len."""
    if budget < w:
        raise ValueError("budget must be >= w (the window is always kept)")
    if budget >= length:
        return np.arange(length, dtype=np.int64)
    P = length - w
    chosen = topk_prefix(pooled_prefix[:P], budget - w)
    return np.concatenate([chosen, np.arange(P, length, dtype=np.int64)])


def select_topk(pooled: np.ndarray, cu_seqlens, w: int, budget: int) -> np.ndarray:
    """idx [n_kv, sum_b min(budget, len_b)], int64, sequence-local positions."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = np.diff(cu)
    cb = budget_offsets(lens, budget)
    n_kv = pooled.shape[0]
    idx = np.zeros((n_kv, int(cb[-1])), dtype=np.int64)
    for b in range(len(lens)):
        t0 = int(cu[b])
        for h in range(n_kv):
            idx[h, cb[b]:cb[b + 1]] = select_one(pooled[h, t0:t0 + lens[b]], int(lens[b]), w, budget)
    return idx


# ----------------------------------------------------------------------------
# 5. gather
# ----------------------------------------------------------------------------
def gather_kv(k: np.ndarray, v: np.ndarray, idx: np.ndarray, cu_seqlens, budget: int):
    """K_c[cb_b + t, h] = K[cu_b + idx[h, cb_b + t], h] (same for V); any dtype,
    bytes copied unchanged."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = np.diff(cu)
    cb = budget_offsets(lens, budget)
    n_kv = k.shape[1]
    kc = np.empty((int(cb[-1]),) + k.shape[1:], dtype=k.dtype)
    vc = np.empty_like(kc)
    for b in range(len(lens)):
        for h in range(n_kv):
            src = cu[b] + idx[h, cb[b]:cb[b + 1]]
            kc[cb[b]:cb[b + 1], h] = k[src, h]
            vc[cb[b]:cb[b + 1], h] = v[src, h]
    return kc, vc


# ----------------------------------------------------------------------------
# 6. decode attention
# ----------------------------------------------------------------------------
def gqa_decode(q: np.ndarray, k_c: np.ndarray, v_c: np.ndarray, row_offset, kv_len,
               n_kv: int, dtype: str, scale: float | None = None, cache_dtype: str | None = None) -> np.ndarray:
    """out[b, qh] = sum_t softmax_t(scale * q[b, qh] . K_c[off_b + t, qh // G]) V_c[off_b + t, qh // G]
    over t < kv_len[b]; an empty cache gives 0.  float64 [batch, n_h, d].
    cache_dtype (default: dtype) names the stored type of k_c / v_c; "f64"
    takes them as float64 values."""
    cache_dtype = dtype if cache_dtype is None else cache_dtype
    qf = to_f64(q, dtype)
    kf = to_f64(k_c, cache_dtype)
    vf = to_f64(v_c, cache_dtype)
    batch, n_h, d = qf.shape
    if scale is None or scale <= 0:
        scale = default_scale(d)
    G = n_h // n_kv
    out = np.zeros((batch, n_h, d))
    for b in range(batch):
        o, n = int(row_offset[b]), int(kv_len[b])
        if n == 0:
            continue
        for qh in range(n_h):
            h = qh // G
            z = scale * (kf[o:o + n, h, :] @ qf[b, qh])
            e = np.exp(z - z.max())
            out[b, qh] = (e / e.sum()) @ vf[o:o + n, h, :]
    return out


# ----------------------------------------------------------------------------
# 7. FastKV token-selective propagation
# ----------------------------------------------------------------------------
def tsp_select(raw: np.ndarray, S: int, w: int, pool_k: int, k_tsp: int) -> np.ndarray:
    """One token set for the layer: the k_tsp prefix positions with the largest
    pooled head-summed score (ties: lower index), ascending, then the window.

    raw: [n_rows, S] per-head raw scores of one sequence (rows summed here)."""
    P = S - w
    if k_tsp < 0 or k_tsp > P:
        raise ValueError("k_tsp must lie in [0, S - w]")
    agg = raw[:, :P].sum(axis=0)
    pooled = maxpool1d_same(agg, pool_k)
    chosen = topk_prefix(pooled, k_tsp)
    return np.concatenate([chosen, np.arange(P, S, dtype=np.int64)])


def tsp_pooled(raw: np.ndarray, S: int, w: int, pool_k: int) -> np.ndarray:
    P = S - w
    return maxpool1d_same(raw[:, :P].sum(axis=0), pool_k)


def tsp_gather(hidden: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Propagated hidden states: hidden rows idx, bytes unchanged."""
    return hidden[np.asarray(idx, dtype=np.int64)].copy()


def rate_count(rate: float, S: int) -> int:
    """Token count of a rate applied to S tokens (reading: floor)."""
    return int(np.floor(rate * S))


# ----------------------------------------------------------------------------
# 9. quantised compact cache
# ----------------------------------------------------------------------------
def quantize_rows_int8(x: np.ndarray):
    """Symmetric int8 quantisation of every vector along the last axis.

    x: float32 values (the exact widening of the stored cache).  Returns
    (codes int8 of x's shape, scales float32 of x.shape[:-1]).  The scale is
    max|x| / 127 and the code round-half-even(x / scale), each quotient taken
    in float32; all-zero vectors get scale 0 and codes 0."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    ratio = (x / safe[..., None]).astype(np.float32)
    codes = np.clip(np.rint(ratio), -127, 127)
    codes = np.where(scale[..., None] > 0, codes, 0).astype(np.int8)
    return codes, scale


def dequantize_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """code * scale in float64 (exact: an 8-bit integer times a float32)."""
    return codes.astype(np.float64) * np.asarray(scale, dtype=np.float64)[..., None]


def gather_kv_q8(k: np.ndarray, v: np.ndarray, idx: np.ndarray, cu_seqlens, budget: int, dtype: str):
    """Gather the retained rows (as gather_kv) and quantise every (slot, head)
    vector.  Returns (kq, vq int8 [Tb, n_kv, d], ks, vs float32 [n_kv, Tb])."""
    kc, vc = gather_kv(k, v, idx, cu_seqlens, budget)
    kq, ks = quantize_rows_int8(to_f64(kc, dtype).astype(np.float32))
    vq, vs = quantize_rows_int8(to_f64(vc, dtype).astype(np.float32))
    return kq, vq, np.ascontiguousarray(ks.T), np.ascontiguousarray(vs.T)


def gqa_decode_q8(q: np.ndarray, kq: np.ndarray, vq: np.ndarray, k_scale: np.ndarray, v_scale: np.ndarray,
                  row_offset, kv_len, n_kv: int, q_dtype: str, scale: float | None = None) -> np.ndarray:
    """Decode attention (gqa_decode) over the dequantised int8 caches.
    k_scale, v_scale: [n_kv, >= rows] float32."""
    rows = kq.shape[0]
    kd = dequantize_rows(kq, np.asarray(k_scale)[:, :rows].T)
    vd = dequantize_rows(vq, np.asarray(v_scale)[:, :rows].T)
    return gqa_decode(q, kd, vd, row_offset, kv_len, n_kv, q_dtype, scale, cache_dtype="f64")


# ----------------------------------------------------------------------------
# 10. PyramidKV per-layer budgets
# ----------------------------------------------------------------------------
def pyramid_budgets(L: int, avg_budget: int, min_budget: int) -> np.ndarray:
    """Per-layer budgets falling linearly from 2 * avg - min (layer 0) to min
    (layer L - 1), integer arithmetic throughout.  int64 [L]."""
    if L < 1 or min_budget < 0 or min_budget > avg_budget:
        raise ValueError("need L >= 1 and 0 <= min_budget <= avg_budget")
    if L == 1:
        return np.array([avg_budget], dtype=np.int64)
    b_max = 2 * avg_budget - min_budget
    return np.array([b_max - ((b_max - min_budget) * l) // (L - 1) for l in range(L)], dtype=np.int64)


# ----------------------------------------------------------------------------
# 11. FreeKV decode-time retrieval with fine-grained correction
# ----------------------------------------------------------------------------
def freekv_flags(q_cur: np.ndarray, q_prev: np.ndarray, n_kv: int, tau: float, dtype: str):
    """(flags bool [batch, n_kv], cos float64 [batch, n_h]): cos of the current
    and previous query of every query head; a KV head is flagged (scored and
    selected again) when the smallest cos of its group is below tau."""
    a = to_f64(q_cur, dtype)
    b = to_f64(q_prev, dtype)
    dot = np.sum(a * b, axis=-1)
    den = np.sqrt(np.sum(a * a, axis=-1)) * np.sqrt(np.sum(b * b, axis=-1))
    cos = np.where(den > 0, dot / np.where(den > 0, den, 1.0), 0.0)
    batch, n_h = cos.shape
    G = n_h // n_kv
    return cos.reshape(batch, n_kv, G).min(axis=2) < tau, cos


def decode_query_scores(q: np.ndarray, k: np.ndarray, cu_seqlens, n_kv: int, dtype: str,
                        scale: float | None = None) -> np.ndarray:
    """raw[h, t]: for sequence b, the softmax mass that the decode queries of
    the G query heads of KV head h put on each of its len_b cached keys (the
    query follows the whole cache, so every key is visible).  [n_kv, T]."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    qf = to_f64(q, dtype)
    kf = to_f64(k, dtype)
    batch, n_h, d = qf.shape
    if scale is None or scale <= 0:
        scale = default_scale(d)
    G = n_h // n_kv
    out = np.zeros((n_kv, int(cu[-1])))
    for b in range(batch):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        for h in range(n_kv):
            z = scale * (qf[b, h * G:(h + 1) * G] @ kf[t0:t1, h].T)        # [G, len]
            e = np.exp(z - z.max(axis=1, keepdims=True))
            out[h, t0:t1] = (e / e.sum(axis=1, keepdims=True)).sum(axis=0)
    return out


def freekv_step(q_cur, q_prev, k, v, cu_seqlens, idx_prev, n_kv: int, w: int, pool_k: int, budget: int,
                tau: float, dtype: str, scale: float | None = None, flags=None):
    """One decode step.  Returns (flags, idx, k_c, v_c, out): the heads flagged
    by freekv_flags (or the given flags) get a fresh index list from
    decode_query_scores -> pool_prefix -> select_topk; the others keep
    idx_prev; k_c / v_c are the rows idx names; out is gqa_decode of q_cur over
    them."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = np.diff(cu)
    if flags is None:
        flags, _ = freekv_flags(q_cur, q_prev, n_kv, tau, dtype)
    raw = decode_query_scores(q_cur, k, cu, n_kv, dtype, scale)
    fresh = select_topk(pool_prefix(raw, cu, w, pool_k), cu, w, budget)
    idx = np.array(idx_prev, dtype=np.int64, copy=True)
    cb = budget_offsets(lens, budget)
    for b in range(len(lens)):
        for h in range(n_kv):
            if flags[b, h]:
                idx[h, cb[b]:cb[b + 1]] = fresh[h, cb[b]:cb[b + 1]]
    k_c, v_c = gather_kv(k, v, idx, cu, budget)
    out = gqa_decode(q_cur, k_c, v_c, cb[:-1], np.diff(cb), n_kv, dtype, scale)
    return flags, idx, k_c, v_c, out


# ----------------------------------------------------------------------------
# 12. xKV cross-layer factorisation and selective reconstruction
# ----------------------------------------------------------------------------
def xkv_factorize(k_layers, r: int, dtype: str):
    """k_layers: W caches [S, n_kv, d] (stored).  Returns (A [n_kv, S, r],
    Vt [n_kv, r, W * d]) in float64 with A = X_h V_r and Vt = V_r^T from the
    truncated SVD of X_h = [K_1[:, h] | ... | K_W[:, h]]."""
    X = np.concatenate([to_f64(k, dtype) for k in k_layers], axis=2)     # [S, n_kv, W d]
    S, n_kv, Wd = X.shape
    if not 1 <= r <= min(S, Wd):
        raise ValueError("need 1 <= r <= min(S, W * d)")
    A = np.zeros((n_kv, S, r))
    Vt = np.zeros((n_kv, r, Wd))
    for h in range(n_kv):
        _, _, vt = np.linalg.svd(X[:, h, :], full_matrices=False)
        Vt[h] = vt[:r]
        A[h] = X[:, h, :] @ vt[:r].T
    return A, Vt


def xkv_reconstruct(A: np.ndarray, Vt: np.ndarray, layer: int, d: int, idx: np.ndarray) -> np.ndarray:
    """Rows idx[h] of layer `layer` for every KV head: [n_sel, n_kv, d] float64,
    row t of head h = A[h, idx[h, t]] @ Vt[h][:, layer*d:(layer+1)*d]."""
    n_kv, n_sel = idx.shape
    out = np.zeros((n_sel, n_kv, d))
    for h in range(n_kv):
        out[:, h, :] = A[h][np.asarray(idx[h], dtype=np.int64)] @ Vt[h][:, layer * d:(layer + 1) * d]
    return out


def xkv_window_bytes(S: int, n_kv: int, d: int, W: int, r: int, b_basis: int, b_blocks: int) -> int:
    """Bytes one factorised window stores (per KV head: the S x r basis and the
    r x (W d) reconstruction blocks), against W * S * n_kv * d * b for the
    plain keys of the window."""
    return n_kv * (S * r * b_basis + r * W * d * b_blocks)
