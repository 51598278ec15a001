// C ABI of libkvc: argument validation, work plans, workspace layout and
// kernel launches.  Declarations and contracts are in include/kvc.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "kvc_internal.h"

namespace {

thread_local char g_err[512] = "";

kvc_status fail(kvc_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

kvc_status cuda_fail(cudaError_t e, const char *what) {
  return fail(KVC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int elem_size(kvc_dtype dt) { return dt == KVC_F32 ? 4 : dt == KVC_BF16 ? 2 : 0; }

constexpr size_t kErrWordBytes = 256;   // workspace head: device error word

// ------------------------------------------------------------ batch checks
struct Batch {
  int64_t T = 0;
  int max_len = 0;
  int min_len = 0;
};

kvc_status check_batch(int n_seqs, const int32_t *seqlens_host, int min_each, Batch *bt) {
  if (n_seqs < 1) return fail(KVC_ERR_INVALID_ARG, "n_seqs must be >= 1 (got %d)", n_seqs);
  if (!seqlens_host) return fail(KVC_ERR_INVALID_ARG, "seqlens_host is NULL");
  int64_t T = 0;
  int mx = 0, mn = INT32_MAX;
  for (int b = 0; b < n_seqs; ++b) {
    const int L = seqlens_host[b];
    if (L < min_each) return fail(KVC_ERR_INVALID_ARG, "seqlens_host[%d] = %d is below %d", b, L, min_each);
    T += L;
    mx = std::max(mx, L);
    mn = std::min(mn, L);
  }
  if (T >= (int64_t)INT32_MAX) return fail(KVC_ERR_INVALID_ARG, "total tokens %lld exceed int32", (long long)T);
  bt->T = T;
  bt->max_len = mx;
  bt->min_len = mn;
  return KVC_OK;
}

// --------------------------------------------------------- scoring plan
struct ScorePlan {
  bool tc = false, fused = false;
  int R = 0, R_pad = 0, tile = 0, keys_per_chunk = 0, n_chunks = 0;
  Batch bt;
  size_t off_sync = 0, off_hist = 0, off_cnt = 0, off_part = 0, off_raw = 0, bytes = 0;
};

kvc_status plan_score(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host, int n_h, int n_kv, int d_h, int w,
                      ScorePlan *pl) {
  if (dt != KVC_F32 && dt != KVC_BF16) return fail(KVC_ERR_UNSUPPORTED, "dtype %d not supported", (int)dt);
  if (n_h < 1 || n_kv < 1 || n_h % n_kv != 0)
    return fail(KVC_ERR_INVALID_ARG, "n_h (%d) must be a positive multiple of n_kv (%d)", n_h, n_kv);
  if (d_h != 64 && d_h != 128) return fail(KVC_ERR_UNSUPPORTED, "d_h must be 64 or 128 (got %d)", d_h);
  if (w < 1) return fail(KVC_ERR_INVALID_ARG, "w must be >= 1 (got %d)", w);
  const int G = n_h / n_kv;
  if ((int64_t)G * w > 256) return fail(KVC_ERR_UNSUPPORTED, "window block G*w = %d exceeds 256 rows", G * w);
  kvc_status s = check_batch(n_seqs, seqlens_host, w, &pl->bt);
  if (s != KVC_OK) return s;
  pl->R = G * w;
  pl->tc = (dt == KVC_BF16) && pl->R <= 128;
  pl->R_pad = pl->tc ? 128 : (pl->R + 63) / 64 * 64;
  pl->tile = pl->tc ? kvc::tc_keys_per_tile() : kvc::simt_keys_per_tile();
  // chunk the keys of every (sequence, head) so that about one wave of CTAs
  // covers the batch: the smallest tiles-per-chunk whose CTA count fits
  const int target = pl->tc ? kvc::kNumSMs : 2 * kvc::kNumSMs;
  int64_t total_tiles = 0;
  int max_tiles = 0;
  std::vector<int> tiles(n_seqs);
  for (int b = 0; b < n_seqs; ++b) {
    tiles[b] = (seqlens_host[b] + pl->tile - 1) / pl->tile;
    total_tiles += (int64_t)tiles[b] * n_kv;
    max_tiles = std::max(max_tiles, tiles[b]);
  }
  int tpc = (int)std::max<int64_t>(1, (total_tiles + target - 1) / target);
  for (; tpc < max_tiles; ++tpc) {
    int64_t ctas = 0;
    for (int b = 0; b < n_seqs; ++b) ctas += (int64_t)n_kv * ((tiles[b] + tpc - 1) / tpc);
    if (ctas <= target) break;
  }
  tpc = std::max(1, std::min(tpc, std::max(1, max_tiles)));
  if (pl->tc) {
    // the grid is (n_kv, chunks of the longest sequence, n_seqs); when it
    // exceeds one CTA per SM the launch is not fused
    const int64_t grid = (int64_t)n_kv * n_seqs * ((std::max(1, max_tiles) + tpc - 1) / tpc);
    if (grid > kvc::kNumSMs) {
      // the split launches (one CTA per SM, several waves): the chunk size
      // that minimises waves x (tiles per chunk + a per-CTA setup cost of
      // about 8 tiles), so that long sequences no longer set the makespan
      auto cost = [&](int t) {
        int64_t c = 0;
        for (int b = 0; b < n_seqs; ++b) c += (int64_t)n_kv * ((tiles[b] + t - 1) / t);
        return (c + kvc::kNumSMs - 1) / kvc::kNumSMs * (int64_t)(t + 8);
      };
      int best = tpc;
      int64_t best_cost = cost(tpc);
      for (int t = 4; t < max_tiles; ++t) {
        const int64_t c = cost(t);
        if (c < best_cost) { best_cost = c; best = t; }
      }
      tpc = best;
    }
  }
  pl->keys_per_chunk = tpc * pl->tile;
  pl->n_chunks = std::max(1, (pl->bt.max_len + pl->keys_per_chunk - 1) / pl->keys_per_chunk);
  // one cooperative launch when the whole grid is resident at once (one CTA per SM)
  pl->fused = pl->tc && (int64_t)n_kv * pl->n_chunks * n_seqs <= kvc::kNumSMs;
  const size_t units = (size_t)n_seqs * n_kv;
  pl->off_sync = kErrWordBytes;
  pl->off_hist = round_up(pl->off_sync + units * kvc::tc_counters_per_unit() * sizeof(int), 256);
  pl->off_cnt = round_up(pl->off_hist + units * kvc::tc_hist_ints() * sizeof(int), 256);
  pl->off_part = round_up(pl->off_cnt + units * pl->n_chunks * kvc::tc_count_ints() * sizeof(int), 256);
  const size_t part_bytes = (size_t)n_seqs * n_kv * pl->n_chunks * pl->R_pad * sizeof(float2);
  pl->off_raw = round_up(pl->off_part + part_bytes, 256);
  pl->bytes = pl->off_raw + round_up((size_t)n_kv * pl->bt.T * sizeof(float), 256);
  return KVC_OK;
}

// --------------------------------------------------------- decode plan
struct DecodePlan {
  int chunk_rows = 0, n_chunks = 0;
  size_t off_tickets = 0, off_part = 0, bytes = 0;
};

kvc_status plan_decode(kvc_dtype dt, int batch, int n_h, int n_kv, int d_h, int max_kv_len, DecodePlan *pl) {
  if (dt != KVC_F32 && dt != KVC_BF16) return fail(KVC_ERR_UNSUPPORTED, "dtype %d not supported", (int)dt);
  if (batch < 1) return fail(KVC_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", batch);
  if (n_h < 1 || n_kv < 1 || n_h % n_kv != 0)
    return fail(KVC_ERR_INVALID_ARG, "n_h (%d) must be a positive multiple of n_kv (%d)", n_h, n_kv);
  const int G = n_h / n_kv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(KVC_ERR_UNSUPPORTED, "GQA group %d not in {1,2,4,8}", G);
  if (d_h != 64 && d_h != 128) return fail(KVC_ERR_UNSUPPORTED, "d_h must be 64 or 128 (got %d)", d_h);
  if (max_kv_len < 0) return fail(KVC_ERR_INVALID_ARG, "max_kv_len must be >= 0");
  // stream-K over warps: every (batch entry, KV head) unit gets at most
  // decode_slots(max_kv_len) partial slots
  const int64_t units = (int64_t)batch * n_kv;
  pl->chunk_rows = 0;
  pl->n_chunks = kvc::decode_slots(max_kv_len);
  pl->off_tickets = kErrWordBytes;
  pl->off_part = round_up(pl->off_tickets + (size_t)units * sizeof(int), 256);
  pl->bytes = pl->off_part + (size_t)units * pl->n_chunks * G * (d_h + 4) * sizeof(float);
  return KVC_OK;
}

}  // namespace

namespace kvc {
std::atomic<int64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

cudaError_t ensure_smem_limit(const void *fn, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<const void *, int>, int>> done;   // ((fn, device), bytes)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (auto &d : done)
    if (d.first.first == fn && d.first.second == dev && d.second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back({{fn, dev}, bytes});
  return e;
}
}  // namespace kvc

extern "C" {

int kvc_version(void) { return 100; }

int64_t kvc_launch_count(void) { return kvc::g_launches.load(std::memory_order_relaxed); }

kvc_status kvc_check_workspace(const void *ws, kvc_stream_t stream) {
  if (!aligned16(ws)) return fail(KVC_ERR_INVALID_ARG, "ws must be non-NULL and 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "waiting for the stream");
  if (word != 0) return fail(KVC_ERR_DEVICE_CHECK, "device error word is %d: a bounded wait gave up", word);
  return KVC_OK;
}

const char *kvc_status_string(int status) {
  switch (status) {
    case KVC_OK: return "KVC_OK";
    case KVC_ERR_INVALID_ARG: return "KVC_ERR_INVALID_ARG";
    case KVC_ERR_UNSUPPORTED: return "KVC_ERR_UNSUPPORTED";
    case KVC_ERR_WORKSPACE: return "KVC_ERR_WORKSPACE";
    case KVC_ERR_CUDA: return "KVC_ERR_CUDA";
    case KVC_ERR_DEVICE_CHECK: return "KVC_ERR_DEVICE_CHECK";
    default: return "KVC_ERR_UNKNOWN";
  }
}

const char *kvc_last_error(void) { return g_err; }

uint64_t kvc_cache_bytes(int L, int64_t S, int n_kv, int d_h, int b) {
  if (L < 0 || S < 0 || n_kv < 0 || d_h < 0 || b < 0) return 0;
  return 2ull * (uint64_t)L * (uint64_t)S * (uint64_t)n_kv * (uint64_t)d_h * (uint64_t)b;
}

int64_t kvc_budget_offsets(int n_seqs, const int32_t *seqlens_host, int budget, int32_t *cu_budget_host) {
  if (n_seqs < 0 || (n_seqs > 0 && !seqlens_host) || !cu_budget_host || budget < 0) return -1;
  int64_t acc = 0;
  cu_budget_host[0] = 0;
  for (int b = 0; b < n_seqs; ++b) {
    if (seqlens_host[b] < 0) return -1;
    acc += std::min(budget, seqlens_host[b]);
    if (acc >= INT32_MAX) return -1;
    cu_budget_host[b + 1] = (int32_t)acc;
  }
  return acc;
}

int64_t kvc_pyramid_budgets(int L, int avg_budget, int min_budget, int32_t *budgets_host) {
  if (L < 1 || min_budget < 0 || min_budget > avg_budget || !budgets_host) return -1;
  if (L == 1) {
    budgets_host[0] = avg_budget;
    return avg_budget;
  }
  const int64_t b_max = 2 * (int64_t)avg_budget - min_budget;
  if (b_max > INT32_MAX) return -1;
  int64_t total = 0;
  for (int l = 0; l < L; ++l) {
    budgets_host[l] = (int32_t)(b_max - ((b_max - min_budget) * l) / (L - 1));
    total += budgets_host[l];
  }
  return total;
}

size_t kvc_score_window_workspace_size(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host, int n_h, int n_kv,
                                       int d_h, int w) {
  ScorePlan pl;
  if (plan_score(dt, n_seqs, seqlens_host, n_h, n_kv, d_h, w, &pl) != KVC_OK) return 0;
  return pl.bytes;
}

}  // extern "C"

namespace {

// What kvc_compress_window adds to scoring: the selection and gather that run
// inside the fused launch when it applies.
struct SelectGather {
  const int32_t *cu_budget;
  int budget;
  int total_budget;
  int32_t *idx;
  const void *v;
  void *k_out, *v_out;
};

// Scoring (and, when sel != nullptr and the fused launch applies with every key
// chunk small enough to keep on chip, the selection and gather too).  *done_sel
// reports whether the selection and gather ran.
kvc_status score_impl(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens, int n_h,
                      int n_kv, int d_h, int w, int pool_k, float scale, const void *q_win, const void *k,
                      float *scores, float *scores_raw, void *ws, size_t ws_bytes, kvc_stream_t stream,
                      const SelectGather *sel, bool *done_sel) {
  if (done_sel) *done_sel = false;
  ScorePlan pl;
  kvc_status s = plan_score(dt, n_seqs, seqlens_host, n_h, n_kv, d_h, w, &pl);
  if (s != KVC_OK) return s;
  if (pool_k < 1 || pool_k > 31 || pool_k % 2 == 0)
    return fail(KVC_ERR_INVALID_ARG, "pool_k must be odd and in [1, 31] (got %d)", pool_k);
  if (!cu_seqlens) return fail(KVC_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (!aligned16(q_win) || !aligned16(k) || !aligned16(scores))
    return fail(KVC_ERR_INVALID_ARG, "q_win, k and scores must be non-NULL and 16-byte aligned");
  if (scores_raw && !aligned16(scores_raw)) return fail(KVC_ERR_INVALID_ARG, "scores_raw must be 16-byte aligned");
  if (!aligned16(ws) || ws_bytes < pl.bytes)
    return fail(KVC_ERR_WORKSPACE, "workspace needs %zu bytes at a 16-byte aligned address (got %zu)", pl.bytes,
                ws_bytes);
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_h);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  kvc::ScoreArgs a;
  a.dt = dt; a.n_seqs = n_seqs; a.n_h = n_h; a.n_kv = n_kv; a.d_h = d_h; a.w = w; a.scale = scale;
  a.cu_seqlens = cu_seqlens; a.q_win = q_win; a.k = k;
  a.part = reinterpret_cast<float2 *>(wsb + pl.off_part);
  a.raw = scores_raw ? scores_raw : reinterpret_cast<float *>(wsb + pl.off_raw);
  a.err = reinterpret_cast<int *>(wsb);
  a.sync = reinterpret_cast<int *>(wsb + pl.off_sync);
  a.hist = reinterpret_cast<int *>(wsb + pl.off_hist);
  a.cnt = reinterpret_cast<int *>(wsb + pl.off_cnt);
  a.scores = scores;
  a.pool_k = pool_k;
  a.fused = pl.fused;
  a.T_total = (int)pl.bt.T;
  a.n_chunks = pl.n_chunks;
  a.keys_per_chunk = pl.keys_per_chunk;
  a.R_pad = pl.R_pad;
  a.idx = nullptr; a.cu_budget = nullptr; a.v = nullptr; a.k_out = nullptr; a.v_out = nullptr;
  a.total_budget = 0; a.budget = 0;
  const bool fuse_sel = sel && pl.fused && pl.keys_per_chunk <= kvc::tc_select_max_keys(d_h);
  if (fuse_sel) {
    a.idx = sel->idx; a.cu_budget = sel->cu_budget; a.v = sel->v; a.k_out = sel->k_out; a.v_out = sel->v_out;
    a.total_budget = sel->total_budget; a.budget = sel->budget;
  }
  cudaError_t e = pl.tc ? kvc::score_window_tc(a, st) : kvc::score_window_simt(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "score kernels");
  if (done_sel) *done_sel = fuse_sel;
  if (pl.fused) return KVC_OK;   // the pool ran inside the fused launch
  e = kvc::pool_prefix(a.raw, scores, cu_seqlens, n_seqs, n_kv, a.T_total, pl.bt.max_len, w, pool_k, st);
  if (e != cudaSuccess) return cuda_fail(e, "pool kernel");
  return KVC_OK;
}

}  // namespace

extern "C" {

kvc_status kvc_score_window(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                            int n_h, int n_kv, int d_h, int w, int pool_k, float scale, const void *q_win,
                            const void *k, float *scores, float *scores_raw, void *ws, size_t ws_bytes,
                            kvc_stream_t stream) {
  return score_impl(dt, n_seqs, seqlens_host, cu_seqlens, n_h, n_kv, d_h, w, pool_k, scale, q_win, k, scores,
                    scores_raw, ws, ws_bytes, stream, nullptr, nullptr);
}

kvc_status kvc_compress_window(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                               const int32_t *cu_budget, int n_h, int n_kv, int d_h, int w, int pool_k, int budget,
                               float scale, const void *q_win, const void *k, const void *v, float *scores,
                               float *scores_raw, int32_t *idx, void *k_out, void *v_out, void *ws, size_t ws_bytes,
                               kvc_stream_t stream) {
  // validate the selection and gather arguments before anything is launched
  Batch bt;
  kvc_status s = check_batch(n_seqs, seqlens_host, w, &bt);
  if (s != KVC_OK) return s;
  if (budget < w) return fail(KVC_ERR_INVALID_ARG, "budget (%d) must be >= w (%d): the window is always kept", budget, w);
  if (!cu_budget) return fail(KVC_ERR_INVALID_ARG, "cu_budget is NULL");
  if (!aligned16(idx) || !aligned16(v) || !aligned16(k_out) || !aligned16(v_out))
    return fail(KVC_ERR_INVALID_ARG, "idx, v, k_out and v_out must be non-NULL and 16-byte aligned");
  int64_t total = 0;
  for (int b = 0; b < n_seqs; ++b) total += std::min(budget, seqlens_host[b]);
  SelectGather sel{cu_budget, budget, (int)total, idx, v, k_out, v_out};
  bool done = false;
  s = score_impl(dt, n_seqs, seqlens_host, cu_seqlens, n_h, n_kv, d_h, w, pool_k, scale, q_win, k, scores,
                 scores_raw, ws, ws_bytes, stream, &sel, &done);
  if (s != KVC_OK || done) return s;
  s = kvc_select_topk(n_seqs, seqlens_host, cu_seqlens, cu_budget, n_kv, w, budget, scores, idx, stream);
  if (s != KVC_OK) return s;
  return kvc_gather_kv(dt, n_seqs, seqlens_host, cu_seqlens, cu_budget, n_kv, d_h, budget, idx, k, v, k_out, v_out,
                       stream);
}

kvc_status kvc_select_topk(int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                           const int32_t *cu_budget, int n_kv, int w, int budget, const float *scores, int32_t *idx,
                           kvc_stream_t stream) {
  Batch bt;
  kvc_status s = check_batch(n_seqs, seqlens_host, 0, &bt);
  if (s != KVC_OK) return s;
  if (n_kv < 1) return fail(KVC_ERR_INVALID_ARG, "n_kv must be >= 1");
  if (w < 1) return fail(KVC_ERR_INVALID_ARG, "w must be >= 1 (got %d)", w);
  if (budget < w) return fail(KVC_ERR_INVALID_ARG, "budget (%d) must be >= w (%d): the window is always kept", budget, w);
  if (!cu_seqlens || !cu_budget) return fail(KVC_ERR_INVALID_ARG, "cu_seqlens / cu_budget is NULL");
  if (!aligned16(scores) || !aligned16(idx))
    return fail(KVC_ERR_INVALID_ARG, "scores and idx must be non-NULL and 16-byte aligned");
  int64_t total = 0;
  for (int b = 0; b < n_seqs; ++b) total += std::min(budget, seqlens_host[b]);
  cudaError_t e = kvc::select_topk(scores, idx, cu_seqlens, cu_budget, n_seqs, n_kv, (int)bt.T, (int)total, w, budget,
                                   std::max(bt.max_len, w), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select kernel");
  return KVC_OK;
}

kvc_status kvc_gather_kv(kvc_dtype dt, int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                         const int32_t *cu_budget, int n_kv, int d_h, int budget, const int32_t *idx, const void *k,
                         const void *v, void *k_out, void *v_out, kvc_stream_t stream) {
  const int es = elem_size(dt);
  if (!es) return fail(KVC_ERR_UNSUPPORTED, "dtype %d not supported", (int)dt);
  Batch bt;
  kvc_status s = check_batch(n_seqs, seqlens_host, 0, &bt);
  if (s != KVC_OK) return s;
  if (n_kv < 1 || d_h < 1) return fail(KVC_ERR_INVALID_ARG, "n_kv and d_h must be >= 1");
  if ((d_h * es) % 16 != 0) return fail(KVC_ERR_UNSUPPORTED, "d_h * element size must be a multiple of 16 bytes");
  if (budget < 0) return fail(KVC_ERR_INVALID_ARG, "budget must be >= 0");
  if (!cu_seqlens || !cu_budget) return fail(KVC_ERR_INVALID_ARG, "cu_seqlens / cu_budget is NULL");
  if (!aligned16(idx) || !aligned16(k) || !aligned16(v) || !aligned16(k_out) || !aligned16(v_out))
    return fail(KVC_ERR_INVALID_ARG, "idx, k, v, k_out and v_out must be non-NULL and 16-byte aligned");
  int64_t total = 0;
  int max_kept = 0;
  for (int b = 0; b < n_seqs; ++b) {
    const int kept = std::min(budget, seqlens_host[b]);
    total += kept;
    max_kept = std::max(max_kept, kept);
  }
  if (total == 0) return KVC_OK;
  cudaError_t e = kvc::gather_rows_kv(k, v, k_out, v_out, idx, cu_seqlens, cu_budget, n_seqs, n_kv, d_h * es,
                                      (int)total, max_kept, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gather kernel");
  return KVC_OK;
}

kvc_status kvc_gather_kv_q8(int n_seqs, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                            const int32_t *cu_budget, int n_kv, int d_h, int budget, const int32_t *idx, const void *k,
                            const void *v, int8_t *k_q, int8_t *v_q, float *k_scale, float *v_scale,
                            int64_t scale_pitch, kvc_stream_t stream) {
  Batch bt;
  kvc_status s = check_batch(n_seqs, seqlens_host, 0, &bt);
  if (s != KVC_OK) return s;
  if (n_kv < 1) return fail(KVC_ERR_INVALID_ARG, "n_kv must be >= 1");
  if (d_h != 64 && d_h != 128) return fail(KVC_ERR_UNSUPPORTED, "d_h must be 64 or 128 (got %d)", d_h);
  if (budget < 0) return fail(KVC_ERR_INVALID_ARG, "budget must be >= 0");
  if (!cu_seqlens || !cu_budget) return fail(KVC_ERR_INVALID_ARG, "cu_seqlens / cu_budget is NULL");
  if (!aligned16(idx) || !aligned16(k) || !aligned16(v) || !aligned16(k_q) || !aligned16(v_q) ||
      !aligned16(k_scale) || !aligned16(v_scale))
    return fail(KVC_ERR_INVALID_ARG, "idx, k, v, k_q, v_q, k_scale and v_scale must be non-NULL and 16-byte aligned");
  int64_t total = 0;
  int max_kept = 0;
  for (int b = 0; b < n_seqs; ++b) {
    const int kept = std::min(budget, seqlens_host[b]);
    total += kept;
    max_kept = std::max(max_kept, kept);
  }
  if (scale_pitch < total) return fail(KVC_ERR_INVALID_ARG, "scale_pitch (%lld) must be >= the %lld compact rows",
                                       (long long)scale_pitch, (long long)total);
  if (total == 0) return KVC_OK;
  cudaError_t e = kvc::gather_rows_kv_q8(k, v, k_q, v_q, k_scale, v_scale, scale_pitch, idx, cu_seqlens, cu_budget,
                                         n_seqs, n_kv, d_h, (int)total, max_kept, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gather-and-quantise kernel");
  return KVC_OK;
}

size_t kvc_tsp_workspace_size(int S, int w) {
  if (S < 1 || w < 1 || w > S) return 0;
  return kErrWordBytes + round_up((size_t)(S - w) * sizeof(float), 256);
}

kvc_status kvc_tsp_select_gather(kvc_dtype dt, int S, int n_rows, int w, int pool_k, int k_tsp,
                                 const float *scores_raw, const void *hidden, int D, int32_t *idx_out,
                                 void *hidden_out, void *ws, size_t ws_bytes, kvc_stream_t stream) {
  const int es = elem_size(dt);
  if (!es) return fail(KVC_ERR_UNSUPPORTED, "dtype %d not supported", (int)dt);
  if (S < 1 || w < 1 || w > S) return fail(KVC_ERR_INVALID_ARG, "need 1 <= w <= S (w=%d, S=%d)", w, S);
  if (n_rows < 1) return fail(KVC_ERR_INVALID_ARG, "n_rows must be >= 1");
  if (pool_k < 1 || pool_k > 31 || pool_k % 2 == 0)
    return fail(KVC_ERR_INVALID_ARG, "pool_k must be odd and in [1, 31] (got %d)", pool_k);
  if (k_tsp < 0 || k_tsp > S - w) return fail(KVC_ERR_INVALID_ARG, "k_tsp must lie in [0, S - w] (got %d)", k_tsp);
  if (D < 1 || ((int64_t)D * es) % 16 != 0)
    return fail(KVC_ERR_UNSUPPORTED, "D * element size must be a positive multiple of 16 bytes");
  if (!aligned16(scores_raw) || !aligned16(hidden) || !aligned16(idx_out) || !aligned16(hidden_out))
    return fail(KVC_ERR_INVALID_ARG, "scores_raw, hidden, idx_out and hidden_out must be 16-byte aligned");
  const size_t need = kvc_tsp_workspace_size(S, w);
  if (!aligned16(ws) || ws_bytes < need)
    return fail(KVC_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, ws_bytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float *pooled = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kErrWordBytes);
  cudaError_t e = kvc::tsp_pool(scores_raw, n_rows, S, w, pool_k, pooled, st);
  if (e != cudaSuccess) return cuda_fail(e, "tsp pool kernel");
  e = kvc::tsp_select(pooled, S, w, k_tsp, idx_out, st);
  if (e != cudaSuccess) return cuda_fail(e, "tsp select kernel");
  e = kvc::gather_hidden(hidden, hidden_out, idx_out, k_tsp + w, D * es, S, st);
  if (e != cudaSuccess) return cuda_fail(e, "hidden gather kernel");
  return KVC_OK;
}

size_t kvc_gqa_decode_workspace_size(int batch, int n_h, int n_kv, int d_h, int max_kv_len) {
  DecodePlan pl;
  if (plan_decode(KVC_BF16, batch, n_h, n_kv, d_h, max_kv_len, &pl) != KVC_OK) return 0;
  return pl.bytes;
}

kvc_status kvc_gqa_decode_attn(kvc_dtype dt, int batch, int n_h, int n_kv, int d_h, float scale, const void *q,
                               const void *k_c, const void *v_c, int64_t cache_rows, const int64_t *kv_row_offset,
                               const int32_t *kv_len, int max_kv_len, float *out, void *ws, size_t ws_bytes,
                               kvc_stream_t stream) {
  DecodePlan pl;
  kvc_status s = plan_decode(dt, batch, n_h, n_kv, d_h, max_kv_len, &pl);
  if (s != KVC_OK) return s;
  if (!aligned16(q) || !aligned16(k_c) || !aligned16(v_c) || !aligned16(out))
    return fail(KVC_ERR_INVALID_ARG, "q, k_c, v_c and out must be non-NULL and 16-byte aligned");
  if (!kv_row_offset || !kv_len) return fail(KVC_ERR_INVALID_ARG, "kv_row_offset / kv_len is NULL");
  if (cache_rows < 1 || cache_rows > INT32_MAX)
    return fail(KVC_ERR_INVALID_ARG, "cache_rows must lie in [1, 2^31) (got %lld)", (long long)cache_rows);
  if (!aligned16(ws) || ws_bytes < pl.bytes)
    return fail(KVC_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", pl.bytes, ws_bytes);
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_h);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  kvc::DecodeArgs a;
  a.dt = dt; a.batch = batch; a.n_h = n_h; a.n_kv = n_kv; a.d_h = d_h; a.scale = scale;
  a.q = q; a.k_c = k_c; a.v_c = v_c; a.row_off = kv_row_offset; a.kv_len = kv_len; a.out = out;
  a.tickets = reinterpret_cast<int *>(wsb + pl.off_tickets);
  a.err = reinterpret_cast<int *>(wsb);
  a.cache_rows = cache_rows;
  a.part = reinterpret_cast<float *>(wsb + pl.off_part);
  a.n_chunks = pl.n_chunks;
  a.chunk_rows = pl.chunk_rows;
  cudaError_t e = kvc::gqa_decode(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel");
  return KVC_OK;
}

kvc_status kvc_gqa_decode_attn_q8(int batch, int n_h, int n_kv, int d_h, float scale, const void *q,
                                  const int8_t *k_q, const int8_t *v_q, const float *k_scale, const float *v_scale,
                                  int64_t scale_pitch, int64_t cache_rows, const int64_t *kv_row_offset,
                                  const int32_t *kv_len, int max_kv_len, float *out, void *ws, size_t ws_bytes,
                                  kvc_stream_t stream) {
  DecodePlan pl;
  kvc_status s = plan_decode(KVC_BF16, batch, n_h, n_kv, d_h, max_kv_len, &pl);
  if (s != KVC_OK) return s;
  if (!aligned16(q) || !aligned16(k_q) || !aligned16(v_q) || !aligned16(out) || !aligned16(k_scale) ||
      !aligned16(v_scale))
    return fail(KVC_ERR_INVALID_ARG, "q, k_q, v_q, k_scale, v_scale and out must be non-NULL and 16-byte aligned");
  if (!kv_row_offset || !kv_len) return fail(KVC_ERR_INVALID_ARG, "kv_row_offset / kv_len is NULL");
  if (cache_rows < 1 || cache_rows > INT32_MAX)
    return fail(KVC_ERR_INVALID_ARG, "cache_rows must lie in [1, 2^31) (got %lld)", (long long)cache_rows);
  if (scale_pitch < cache_rows)
    return fail(KVC_ERR_INVALID_ARG, "scale_pitch (%lld) must be >= cache_rows (%lld)", (long long)scale_pitch,
                (long long)cache_rows);
  if (!aligned16(ws) || ws_bytes < pl.bytes)
    return fail(KVC_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", pl.bytes, ws_bytes);
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_h);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  kvc::DecodeArgs a;
  a.dt = KVC_BF16; a.batch = batch; a.n_h = n_h; a.n_kv = n_kv; a.d_h = d_h; a.scale = scale;
  a.q = q; a.k_c = k_q; a.v_c = v_q; a.row_off = kv_row_offset; a.kv_len = kv_len; a.out = out;
  a.tickets = reinterpret_cast<int *>(wsb + pl.off_tickets);
  a.err = reinterpret_cast<int *>(wsb);
  a.cache_rows = cache_rows;
  a.part = reinterpret_cast<float *>(wsb + pl.off_part);
  a.n_chunks = pl.n_chunks;
  a.chunk_rows = pl.chunk_rows;
  a.k_scale = k_scale; a.v_scale = v_scale; a.scale_pitch = scale_pitch;
  cudaError_t e = kvc::gqa_decode_tc(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "int8 decode kernel");
  return KVC_OK;
}

// ------------------------------------------------------------------ FreeKV
namespace {
struct FreeKvPlan {
  DecodePlan dec;
  int n_chunks = 0, G = 0, max_kept = 0;
  int64_t zpitch = 0, total_kept = 0;
  Batch bt;
  size_t off_dec = 0, off_flags = 0, off_doff = 0, off_dlen = 0, off_part = 0, off_scores = 0, off_z = 0, bytes = 0;
};

kvc_status plan_freekv(int batch, const int32_t *seqlens_host, int n_h, int n_kv, int d_h, int w, int budget,
                       FreeKvPlan *pl) {
  kvc_status s = check_batch(batch, seqlens_host, w, &pl->bt);
  if (s != KVC_OK) return s;
  if (w < 1) return fail(KVC_ERR_INVALID_ARG, "w must be >= 1 (got %d)", w);
  if (budget < w) return fail(KVC_ERR_INVALID_ARG, "budget (%d) must be >= w (%d): the window is always kept", budget, w);
  int64_t total = 0;
  int max_kept = 0;
  for (int b = 0; b < batch; ++b) {
    const int kept = std::min(budget, seqlens_host[b]);
    total += kept;
    max_kept = std::max(max_kept, kept);
  }
  s = plan_decode(KVC_BF16, batch, n_h, n_kv, d_h, max_kept, &pl->dec);
  if (s != KVC_OK) return s;
  pl->G = n_h / n_kv;
  pl->max_kept = max_kept;
  pl->total_kept = total;
  pl->n_chunks = (pl->bt.max_len + kvc::freekv_chunk_keys() - 1) / kvc::freekv_chunk_keys();
  pl->zpitch = (int64_t)round_up((size_t)pl->bt.max_len, 4);
  const size_t units = (size_t)batch * n_kv;
  pl->off_dec = 0;                                             // the decode workspace (error word first)
  pl->off_flags = round_up(pl->dec.bytes, 256);
  pl->off_doff = round_up(pl->off_flags + units * sizeof(int), 256);
  pl->off_dlen = round_up(pl->off_doff + (size_t)batch * sizeof(int64_t), 256);
  pl->off_part = round_up(pl->off_dlen + (size_t)batch * sizeof(int), 256);
  pl->off_scores = round_up(pl->off_part + units * pl->n_chunks * pl->G * sizeof(float2), 256);
  pl->off_z = round_up(pl->off_scores + (size_t)n_kv * pl->bt.T * sizeof(float), 256);
  pl->bytes = pl->off_z + units * pl->G * (size_t)pl->zpitch * sizeof(float);
  return KVC_OK;
}
}  // namespace

size_t kvc_freekv_workspace_size(int batch, const int32_t *seqlens_host, int n_h, int n_kv, int d_h, int w,
                                 int budget) {
  FreeKvPlan pl;
  if (plan_freekv(batch, seqlens_host, n_h, n_kv, d_h, w, budget, &pl) != KVC_OK) return 0;
  return pl.bytes;
}

kvc_status kvc_freekv_step(int batch, const int32_t *seqlens_host, const int32_t *cu_seqlens,
                           const int32_t *cu_budget, int n_h, int n_kv, int d_h, int w, int pool_k, int budget,
                           float tau, float scale, const void *q_cur, const void *q_prev, const void *k,
                           const void *v, int32_t *idx, void *k_c, void *v_c, int32_t *reselected, float *out,
                           void *ws, size_t ws_bytes, kvc_stream_t stream) {
  FreeKvPlan pl;
  kvc_status s = plan_freekv(batch, seqlens_host, n_h, n_kv, d_h, w, budget, &pl);
  if (s != KVC_OK) return s;
  if (pool_k < 1 || pool_k > 31 || pool_k % 2 == 0)
    return fail(KVC_ERR_INVALID_ARG, "pool_k must be odd and in [1, 31] (got %d)", pool_k);
  if (!cu_seqlens || !cu_budget) return fail(KVC_ERR_INVALID_ARG, "cu_seqlens / cu_budget is NULL");
  if (!aligned16(q_cur) || !aligned16(q_prev) || !aligned16(k) || !aligned16(v) || !aligned16(idx) ||
      !aligned16(k_c) || !aligned16(v_c) || !aligned16(reselected) || !aligned16(out))
    return fail(KVC_ERR_INVALID_ARG, "q_cur, q_prev, k, v, idx, k_c, v_c, reselected and out must be non-NULL "
                "and 16-byte aligned");
  if (!aligned16(ws) || ws_bytes < pl.bytes)
    return fail(KVC_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", pl.bytes, ws_bytes);
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d_h);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  kvc::FreeKvArgs f;
  f.q_cur = static_cast<const __nv_bfloat16 *>(q_cur);
  f.q_prev = static_cast<const __nv_bfloat16 *>(q_prev);
  f.k = static_cast<const __nv_bfloat16 *>(k);
  f.cu_seqlens = cu_seqlens;
  f.cu_budget = cu_budget;
  f.flags = reselected;
  f.dec_off = reinterpret_cast<int64_t *>(wsb + pl.off_doff);
  f.dec_len = reinterpret_cast<int *>(wsb + pl.off_dlen);
  f.z = reinterpret_cast<float *>(wsb + pl.off_z);
  f.part = reinterpret_cast<float2 *>(wsb + pl.off_part);
  f.scores = reinterpret_cast<float *>(wsb + pl.off_scores);
  f.batch = batch; f.n_h = n_h; f.n_kv = n_kv; f.d_h = d_h; f.w = w; f.pool_r = pool_k / 2;
  f.n_chunks = pl.n_chunks; f.T_total = (int)pl.bt.T; f.zpitch = pl.zpitch;
  f.c = scale * 1.4426950408889634f;
  f.tau = tau;
  cudaError_t e = kvc::freekv_rescore(f, st);
  if (e != cudaSuccess) return cuda_fail(e, "FreeKV re-scoring kernels");
  e = kvc::select_topk(f.scores, idx, cu_seqlens, cu_budget, batch, n_kv, (int)pl.bt.T, (int)pl.total_kept, w, budget,
                       std::max(pl.bt.max_len, w), st, reselected);
  if (e != cudaSuccess) return cuda_fail(e, "FreeKV select kernel");
  e = kvc::gather_rows_kv(k, v, k_c, v_c, idx, cu_seqlens, cu_budget, batch, n_kv, d_h * 2, (int)pl.total_kept,
                          pl.max_kept, st, reselected);
  if (e != cudaSuccess) return cuda_fail(e, "FreeKV gather kernel");
  kvc::DecodeArgs a;
  a.dt = KVC_BF16; a.batch = batch; a.n_h = n_h; a.n_kv = n_kv; a.d_h = d_h; a.scale = scale;
  a.q = q_cur; a.k_c = k_c; a.v_c = v_c; a.row_off = f.dec_off; a.kv_len = f.dec_len; a.out = out;
  a.tickets = reinterpret_cast<int *>(wsb + pl.off_dec + pl.dec.off_tickets);
  a.err = reinterpret_cast<int *>(wsb);
  a.cache_rows = std::max<int64_t>(1, pl.total_kept);
  a.part = reinterpret_cast<float *>(wsb + pl.off_dec + pl.dec.off_part);
  a.n_chunks = pl.dec.n_chunks;
  a.chunk_rows = pl.dec.chunk_rows;
  e = kvc::gqa_decode(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "FreeKV decode kernel");
  return KVC_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Token-selective propagation with library-owned scratch.
//
// For callers that cannot allocate device memory for a workspace -- code
// running where the process' allocator must not be touched (inside another
// library's memory pool or out-of-memory handler, or a latency-critical
// serving loop that forbids allocation) -- this entry point keeps its only
// scratch, the pooled head-summed scores of the prefix, in a fixed array
// compiled into the library.  Every GPU that loads the library holds the
// array (1 MiB) until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr int kStaticTspMaxPrefix = 262144;   // S - w limit of the static variant (floats)
static __device__ __align__(256) float g_tsp_static_scratch[kStaticTspMaxPrefix];

// Device address of the array on the current device, resolved once per
// device (host code only sees a host-side stand-in under the array's name).
kvc_status static_scratch(float **out) {
  static std::mutex mu;
  static std::vector<std::pair<int, float *>> resolved;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(mu);
  for (auto &r : resolved)
    if (r.first == dev) { *out = r.second; return KVC_OK; }
  float *p = nullptr;
  e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_tsp_static_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static TSP scratch");
  resolved.push_back({dev, p});
  *out = p;
  return KVC_OK;
}

}  // namespace

extern "C" kvc_status kvc_tsp_select_gather_static(kvc_dtype dt, int S, int n_rows, int w, int pool_k, int k_tsp,
                                                   const float *scores_raw, const void *hidden, int D,
                                                   int32_t *idx_out, void *hidden_out, kvc_stream_t stream) {
  const int es = elem_size(dt);
  if (!es) return fail(KVC_ERR_UNSUPPORTED, "dtype %d not supported", (int)dt);
  if (S < 1 || w < 1 || w > S) return fail(KVC_ERR_INVALID_ARG, "need 1 <= w <= S (w=%d, S=%d)", w, S);
  if (S - w > kStaticTspMaxPrefix)
    return fail(KVC_ERR_UNSUPPORTED, "the static-scratch variant takes S - w <= %d (got %d); use "
                "kvc_tsp_select_gather with a workspace", kStaticTspMaxPrefix, S - w);
  if (n_rows < 1) return fail(KVC_ERR_INVALID_ARG, "n_rows must be >= 1");
  if (pool_k < 1 || pool_k > 31 || pool_k % 2 == 0)
    return fail(KVC_ERR_INVALID_ARG, "pool_k must be odd and in [1, 31] (got %d)", pool_k);
  if (k_tsp < 0 || k_tsp > S - w) return fail(KVC_ERR_INVALID_ARG, "k_tsp must lie in [0, S - w] (got %d)", k_tsp);
  if (D < 1 || ((int64_t)D * es) % 16 != 0)
    return fail(KVC_ERR_UNSUPPORTED, "D * element size must be a positive multiple of 16 bytes");
  if (!aligned16(scores_raw) || !aligned16(hidden) || !aligned16(idx_out) || !aligned16(hidden_out))
    return fail(KVC_ERR_INVALID_ARG, "scores_raw, hidden, idx_out and hidden_out must be 16-byte aligned");
  float *pooled = nullptr;
  kvc_status s = static_scratch(&pooled);
  if (s != KVC_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the pooled scores are fully rewritten before they are read: nothing to clear
  cudaError_t e = kvc::tsp_pool(scores_raw, n_rows, S, w, pool_k, pooled, st);
  if (e != cudaSuccess) return cuda_fail(e, "tsp pool kernel");
  e = kvc::tsp_select(pooled, S, w, k_tsp, idx_out, st);
  if (e != cudaSuccess) return cuda_fail(e, "tsp select kernel");
  e = kvc::gather_hidden(hidden, hidden_out, idx_out, k_tsp + w, D * es, S, st);
  if (e != cudaSuccess) return cuda_fail(e, "hidden gather kernel");
  return KVC_OK;
}

// ----------------------------------------------------------------- xKV
namespace {
struct XkvPlan {
  int F = 0;
  size_t off_gram = 0, off_y = 0, off_va = 0, off_vb = 0, off_c = 0, off_m = 0, bytes = 0;
};

kvc_status check_xkv_shape(int S, int n_kv, int d_h, int W, int r) {
  if (S < 1 || n_kv < 1) return fail(KVC_ERR_INVALID_ARG, "S and n_kv must be >= 1 (S=%d, n_kv=%d)", S, n_kv);
  if (n_kv > 65535) return fail(KVC_ERR_UNSUPPORTED, "n_kv must be <= 65535");
  if (d_h != 64 && d_h != 128) return fail(KVC_ERR_UNSUPPORTED, "d_h must be 64 or 128 (got %d)", d_h);
  if (W < 1 || W > kvc::kXkvMaxW) return fail(KVC_ERR_UNSUPPORTED, "W must be in [1, %d] (got %d)", kvc::kXkvMaxW, W);
  const int F = W * d_h;
  if (F > 512) return fail(KVC_ERR_UNSUPPORTED, "W * d_h must be <= 512 (got %d)", F);
  if (r != 16 && r != 32 && r != 64) return fail(KVC_ERR_UNSUPPORTED, "r must be 16, 32 or 64 (got %d)", r);
  if (r > S || r > F) return fail(KVC_ERR_INVALID_ARG, "r (%d) must be <= min(S, W * d_h) = %d", r, std::min(S, F));
  return KVC_OK;
}

kvc_status plan_xkv(int S, int n_kv, int d_h, int W, int r, XkvPlan *pl) {
  kvc_status s = check_xkv_shape(S, n_kv, d_h, W, r);
  if (s != KVC_OK) return s;
  pl->F = W * d_h;
  const size_t nk = (size_t)n_kv;
  pl->off_gram = kErrWordBytes;
  pl->off_y = round_up(pl->off_gram + nk * pl->F * pl->F * sizeof(float), 256);
  pl->off_va = round_up(pl->off_y + nk * pl->F * r * sizeof(float), 256);
  pl->off_vb = round_up(pl->off_va + nk * pl->F * r * sizeof(float), 256);
  pl->off_c = round_up(pl->off_vb + nk * pl->F * r * sizeof(float), 256);
  pl->off_m = round_up(pl->off_c + nk * r * r * sizeof(double), 256);
  pl->bytes = round_up(pl->off_m + nk * r * r * sizeof(double), 256);
  return KVC_OK;
}
}  // namespace

extern "C" size_t kvc_xkv_workspace_size(int S, int n_kv, int d_h, int W, int r) {
  XkvPlan pl;
  return plan_xkv(S, n_kv, d_h, W, r, &pl) == KVC_OK ? pl.bytes : 0;
}

extern "C" kvc_status kvc_xkv_factorize(int S, int n_kv, int d_h, int W, int r, int iters,
                                        const void *const *k_layers, const float *v0, kvc_dtype basis_dt,
                                        void *basis, float *blocks, void *ws, size_t ws_bytes,
                                        kvc_stream_t stream) {
  XkvPlan pl;
  kvc_status s = plan_xkv(S, n_kv, d_h, W, r, &pl);
  if (s != KVC_OK) return s;
  if (iters < 1 || iters > 1000) return fail(KVC_ERR_INVALID_ARG, "iters must be in [1, 1000] (got %d)", iters);
  if (basis_dt != KVC_F32 && basis_dt != KVC_BF16)
    return fail(KVC_ERR_UNSUPPORTED, "basis dtype %d not supported", (int)basis_dt);
  if (!k_layers) return fail(KVC_ERR_INVALID_ARG, "k_layers is NULL");
  for (int l = 0; l < W; ++l)
    if (!aligned16(k_layers[l])) return fail(KVC_ERR_INVALID_ARG, "k_layers[%d] must be non-NULL and 16-byte aligned", l);
  if (!aligned16(v0) || !aligned16(basis) || !aligned16(blocks))
    return fail(KVC_ERR_INVALID_ARG, "v0, basis and blocks must be non-NULL and 16-byte aligned");
  if (!aligned16(ws)) return fail(KVC_ERR_WORKSPACE, "ws must be non-NULL and 16-byte aligned");
  if (ws_bytes < pl.bytes)
    return fail(KVC_ERR_WORKSPACE, "workspace of %zu bytes is below the %zu required", ws_bytes, pl.bytes);
  char *w = static_cast<char *>(ws);
  kvc::XkvArgs a = {};
  a.S = S; a.n_kv = n_kv; a.d_h = d_h; a.W = W; a.r = r; a.iters = iters;
  for (int l = 0; l < W; ++l) a.k_layers[l] = k_layers[l];
  a.v0 = v0;
  a.gram = reinterpret_cast<float *>(w + pl.off_gram);
  a.y = reinterpret_cast<float *>(w + pl.off_y);
  a.v_a = reinterpret_cast<float *>(w + pl.off_va);
  a.v_b = reinterpret_cast<float *>(w + pl.off_vb);
  a.c = reinterpret_cast<double *>(w + pl.off_c);
  a.m = reinterpret_cast<double *>(w + pl.off_m);
  a.blocks = blocks;
  a.basis = basis;
  a.basis_bf16 = basis_dt == KVC_BF16;
  cudaError_t e = kvc::xkv_factorize(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "xKV factorisation kernels");
  return KVC_OK;
}

extern "C" kvc_status kvc_xkv_reconstruct(int S, int n_kv, int d_h, int W, int r, int layer, int n_sel,
                                          kvc_dtype basis_dt, const void *basis, const float *blocks,
                                          const int32_t *idx, void *out, kvc_stream_t stream) {
  kvc_status s = check_xkv_shape(S, n_kv, d_h, W, r);
  if (s != KVC_OK) return s;
  if (layer < 0 || layer >= W) return fail(KVC_ERR_INVALID_ARG, "layer must be in [0, W) (got %d)", layer);
  if (n_sel < 0) return fail(KVC_ERR_INVALID_ARG, "n_sel must be >= 0");
  if (n_sel > INT32_MAX - 64) return fail(KVC_ERR_UNSUPPORTED, "n_sel too large");
  if (basis_dt != KVC_F32 && basis_dt != KVC_BF16)
    return fail(KVC_ERR_UNSUPPORTED, "basis dtype %d not supported", (int)basis_dt);
  if (!aligned16(basis) || !aligned16(blocks) || !aligned16(idx) || !aligned16(out))
    return fail(KVC_ERR_INVALID_ARG, "basis, blocks, idx and out must be non-NULL and 16-byte aligned");
  if (n_sel == 0) return KVC_OK;
  kvc::XkvArgs a = {};
  a.S = S; a.n_kv = n_kv; a.d_h = d_h; a.W = W; a.r = r; a.layer = layer; a.n_sel = n_sel;
  a.basis = const_cast<void *>(basis);
  a.blocks = const_cast<float *>(blocks);
  a.basis_bf16 = basis_dt == KVC_BF16;
  a.idx = idx;
  a.out = out;
  cudaError_t e = kvc::xkv_reconstruct(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "xKV reconstruction kernel");
  return KVC_OK;
}
