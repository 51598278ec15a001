// Max-pool of the raw window scores, and the budgeted radix top-k.
//
// Pool (the pages leave the details open; reading: stride 1, same length,
// neighbours outside the prefix [0, P) ignored, window positions +inf so they
// are always retained -- a sliding window keeps its recent region,
// "Variantes de l'attention et compression du cache KV", section "Compresser
// un cache existant").
//
// Select: per (sequence, KV head) the k largest pooled prefix scores, lowest
// position first among equal scores, written in ascending position order
// (original positions are kept, section "Quand la reutilisation est-elle
// exacte ?" of the same page), then the window positions.  One 1024-thread
// block per (sequence, head): MSB-first radix select on order-preserving
// 32-bit keys in digits of 12, 10 and 10 bits finds the k-th largest key T and
// how many keys equal to T are taken; one ordered pass then writes
// position = (#keys > T before it) + min(#keys == T before it, taken).
#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kPoolTile = 1024;
constexpr int kPoolThreads = 256;
constexpr int kMaxPoolRadius = 15;

// ------------------------------------------------------------------ pooling
__global__ void __launch_bounds__(kPoolThreads)
pool_prefix_kernel(const float *__restrict__ raw, float *__restrict__ scores, const int *__restrict__ cu_seqlens,
                   int T_total, int w, int r) {
  const int h = blockIdx.y, b = blockIdx.z;
  const int t0 = cu_seqlens[b], len = cu_seqlens[b + 1] - t0;
  const int j0 = blockIdx.x * kPoolTile;
  if (j0 >= len) return;
  const int P = len - w;
  __shared__ float sv[kPoolTile + 2 * kMaxPoolRadius];
  const float *src = raw + (size_t)h * T_total + t0;
  for (int e = threadIdx.x; e < kPoolTile + 2 * r; e += kPoolThreads) {
    const int j = j0 - r + e;
    sv[e] = (j >= 0 && j < P) ? src[j] : kNegInf;
  }
  __syncthreads();
  float *dst = scores + (size_t)h * T_total + t0;
  for (int e = threadIdx.x; e < kPoolTile; e += kPoolThreads) {
    const int j = j0 + e;
    if (j >= len) break;
    float v = kPosInf;
    if (j < P) {
      v = sv[e + r];
      for (int t = 1; t <= r; ++t) v = fmaxf(v, fmaxf(sv[e + r - t], sv[e + r + t]));
    }
    dst[j] = v;
  }
}

// TSP: agg[j] = sum over score rows, then the same pool; output on [0, P).
__global__ void __launch_bounds__(kPoolThreads)
tsp_pool_kernel(const float *__restrict__ raw, int n_rows, int S, int w, int r, float *__restrict__ pooled) {
  const int j0 = blockIdx.x * kPoolTile;
  const int P = S - w;
  __shared__ float sv[kPoolTile + 2 * kMaxPoolRadius];
  for (int e = threadIdx.x; e < kPoolTile + 2 * r; e += kPoolThreads) {
    const int j = j0 - r + e;
    float a = kNegInf;
    if (j >= 0 && j < P) {
      a = 0.f;
      for (int q = 0; q < n_rows; ++q) a += raw[(size_t)q * S + j];
    }
    sv[e] = a;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kPoolTile; e += kPoolThreads) {
    const int j = j0 + e;
    if (j >= P) break;
    float v = sv[e + r];
    for (int t = 1; t <= r; ++t) v = fmaxf(v, fmaxf(sv[e + r - t], sv[e + r + t]));
    pooled[j] = v;
  }
}

// ---------------------------------------------------------------- selection
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSmemKeysMax = 40960;   // keys cached in shared memory (160 KB)

// float -> uint32 with the same order (negatives below positives, NaN on top)
KVC_DEVINL uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelSmem {
  int hist[4096];
  int wsum[kSelWarps];
  int bcast[4];
};

// Block-wide exclusive prefix sum of one int per thread; returns the
// exclusive value and writes the block total to *total.
KVC_DEVINL int block_exclusive_scan(int v, SelSmem &sm, int *total) {
  const int lane = lane_id(), wid = warp_id();
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm.wsum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = sm.wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sm.wsum[lane] = s;   // inclusive warp prefix
  }
  __syncthreads();
  const int before = (wid == 0) ? 0 : sm.wsum[wid - 1];
  *total = sm.wsum[kSelWarps - 1];
  const int ex = before + x - v;
  __syncthreads();
  return ex;
}

// Writes the ascending positions of the k largest of src[0..n) (lowest index
// first among equal keys) to out[0..k).  0 <= k <= n.
KVC_DEVINL void block_topk_ascending(const float *__restrict__ src, int n, int k, int32_t *__restrict__ out,
                                     uint32_t *cache, int cache_cap, SelSmem &sm) {
  if (k <= 0) return;
  const bool cached = (n <= cache_cap);
  if (k >= n) {
    for (int i = threadIdx.x; i < n; i += kSelThreads) out[i] = i;
    return;
  }
  if (cached)
    for (int i = threadIdx.x; i < n; i += kSelThreads) cache[i] = order_key(src[i]);
  // cache writes are ordered before the first histogram read by the syncs below
  uint32_t prefix = 0, pmask = 0;
  int k_rem = k;
  const int shifts[3] = {20, 10, 0};
  const int widths[3] = {12, 10, 10};
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass], nb = 1 << widths[pass];
    for (int i = threadIdx.x; i < nb; i += kSelThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kSelThreads) {
      const uint32_t u = cached ? cache[i] : order_key(src[i]);
      if ((u & pmask) == prefix) atomicAdd(&sm.hist[(u >> shift) & (nb - 1)], 1);
    }
    __syncthreads();
    // suffix counts: thread t owns bins [t*per, (t+1)*per) counted from the top
    const int per = nb / kSelThreads;   // 4 or 1
    int own = 0;
    for (int q = 0; q < per; ++q) own += sm.hist[nb - 1 - (threadIdx.x * per + q)];
    int tot;
    const int above = block_exclusive_scan(own, sm, &tot);   // keys in higher bins
    int run = above;
    for (int q = 0; q < per; ++q) {
      const int bin = nb - 1 - (threadIdx.x * per + q);
      const int cnt = sm.hist[bin];
      if (run < k_rem && run + cnt >= k_rem) {
        sm.bcast[0] = bin;
        sm.bcast[1] = run;
      }
      run += cnt;
    }
    __syncthreads();
    const int bin = sm.bcast[0];
    k_rem -= sm.bcast[1];
    prefix |= (uint32_t)bin << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;   // key of the k-th largest element; take k_rem of the keys == T
  int run_gt = 0, run_eq = 0;
  for (int base = 0; base < n; base += kSelThreads) {
    const int i = base + threadIdx.x;
    int gt = 0, eq = 0;
    if (i < n) {
      const uint32_t u = cached ? cache[i] : order_key(src[i]);
      gt = u > T;
      eq = u == T;
    }
    int tot;
    const int ex = block_exclusive_scan(gt | (eq << 16), sm, &tot);
    const int ex_gt = ex & 0xffff, ex_eq = ex >> 16;
    const int eq_before = run_eq + ex_eq;
    if (gt || (eq && eq_before < k_rem)) out[run_gt + ex_gt + min(eq_before, k_rem)] = i;
    run_gt += tot & 0xffff;
    run_eq += tot >> 16;
  }
}

__global__ void __launch_bounds__(kSelThreads)
select_topk_kernel(const float *__restrict__ scores, int32_t *__restrict__ idx, const int *__restrict__ cu_seqlens,
                   const int *__restrict__ cu_budget, int T_total, int total_budget, int w, int budget,
                   int cache_cap) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int t0 = cu_seqlens[b], len = cu_seqlens[b + 1] - t0;
  int32_t *dst = idx + (size_t)h * total_budget + cu_budget[b];
  if (budget >= len) {
    for (int t = threadIdx.x; t < len; t += kSelThreads) dst[t] = t;
    return;
  }
  const int P = len - w, k_sel = budget - w;
  extern __shared__ uint32_t sel_cache[];
  __shared__ SelSmem sm;
  block_topk_ascending(scores + (size_t)h * T_total + t0, P, k_sel, dst, sel_cache, cache_cap, sm);
  for (int t = threadIdx.x; t < w; t += kSelThreads) dst[k_sel + t] = P + t;
}

__global__ void __launch_bounds__(kSelThreads)
tsp_select_kernel(const float *__restrict__ pooled, int S, int w, int k_tsp, int32_t *__restrict__ idx_out,
                  int cache_cap) {
  const int P = S - w;
  extern __shared__ uint32_t sel_cache[];
  __shared__ SelSmem sm;
  block_topk_ascending(pooled, P, k_tsp, idx_out, sel_cache, cache_cap, sm);
  for (int t = threadIdx.x; t < w; t += kSelThreads) idx_out[k_tsp + t] = P + t;
}

}  // namespace

cudaError_t pool_prefix(const float *raw, float *scores, const int32_t *cu_seqlens, int n_seqs, int n_kv,
                        int T_total, int max_len, int w, int pool_k, cudaStream_t st) {
  dim3 grid((max_len + kPoolTile - 1) / kPoolTile, n_kv, n_seqs);
  pool_prefix_kernel<<<grid, kPoolThreads, 0, st>>>(raw, scores, cu_seqlens, T_total, w, (pool_k - 1) / 2);
  return cudaGetLastError();
}

cudaError_t tsp_pool(const float *raw, int n_rows, int S, int w, int pool_k, float *pooled, cudaStream_t st) {
  const int P = S - w;
  if (P <= 0) return cudaSuccess;
  tsp_pool_kernel<<<(P + kPoolTile - 1) / kPoolTile, kPoolThreads, 0, st>>>(raw, n_rows, S, w, (pool_k - 1) / 2,
                                                                            pooled);
  return cudaGetLastError();
}

static cudaError_t set_sel_smem(const void *fn, int n, int *cap, size_t *bytes) {
  *cap = n <= kSmemKeysMax ? n : 0;
  *bytes = (size_t)(*cap) * sizeof(uint32_t);
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(kSmemKeysMax * 4));
}

cudaError_t select_topk(const float *scores, int32_t *idx, const int32_t *cu_seqlens, const int32_t *cu_budget,
                        int n_seqs, int n_kv, int T_total, int total_budget, int w, int budget, int max_len,
                        cudaStream_t st) {
  int cap;
  size_t bytes;
  cudaError_t e = set_sel_smem((const void *)select_topk_kernel, max_len - w, &cap, &bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(n_kv, n_seqs);
  select_topk_kernel<<<grid, kSelThreads, bytes, st>>>(scores, idx, cu_seqlens, cu_budget, T_total, total_budget, w,
                                                       budget, cap);
  return cudaGetLastError();
}

cudaError_t tsp_select(const float *pooled, int S, int w, int k_tsp, int32_t *idx_out, cudaStream_t st) {
  int cap;
  size_t bytes;
  cudaError_t e = set_sel_smem((const void *)tsp_select_kernel, S - w, &cap, &bytes);
  if (e != cudaSuccess) return e;
  tsp_select_kernel<<<1, kSelThreads, bytes, st>>>(pooled, S, w, k_tsp, idx_out, cap);
  return cudaGetLastError();
}

}  // namespace kvc
