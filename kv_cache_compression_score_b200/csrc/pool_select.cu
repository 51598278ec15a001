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
constexpr int kSmemKeysMax = 40960;   // keys cached in shared memory (+1 pad word per 32: 165 KB)

// float -> uint32 with the same order (negatives below positives, NaN on top)
KVC_DEVINL uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelSmem {
  int hist[2048];
  int wsum[kSelWarps];
  int wsum2[kSelWarps];
  int bcast[4];
};

// Block-wide exclusive prefix sum of an int2 per thread (two counters at once).
KVC_DEVINL int2 block_exclusive_scan2(int2 v, SelSmem &sm, int2 *total) {
  const int lane = lane_id(), wid = warp_id();
  int x = v.x, y = v.y;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, x, o), b = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) { x += a; y += b; }
  }
  if (lane == 31) { sm.wsum[wid] = x; sm.wsum2[wid] = y; }
  __syncthreads();
  if (wid == 0) {
    int a = sm.wsum[lane], b = sm.wsum2[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int c = __shfl_up_sync(0xffffffffu, a, o), d = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) { a += c; b += d; }
    }
    sm.wsum[lane] = a;
    sm.wsum2[lane] = b;
  }
  __syncthreads();
  const int bx = wid ? sm.wsum[wid - 1] : 0, by = wid ? sm.wsum2[wid - 1] : 0;
  *total = make_int2(sm.wsum[kSelWarps - 1], sm.wsum2[kSelWarps - 1]);
  __syncthreads();
  return make_int2(bx + x - v.x, by + y - v.y);
}

// Writes the ascending positions of the k largest of src[0..n) (lowest index
// first among equal keys) to out[0..k).  0 <= k <= n.
//
// Thread t owns the contiguous run [t*E, (t+1)*E), E = ceil(n / threads), so
// index order is (thread, position in run).  Keys are cached in shared memory
// with one pad word per 32 (conflict-free strided reads) when n fits the
// cache, else re-read from global memory (L2-resident).  Radix digits of 11
// bits start at the highest bit where the keys of the array differ, so the
// first histogram spreads over the occupied range.
KVC_DEVINL void block_topk_ascending(const float *__restrict__ src, int n, int k, int32_t *__restrict__ out,
                                     uint32_t *cache, int cache_cap, SelSmem &sm) {
  if (k <= 0) return;
  if (k >= n) {
    for (int i = threadIdx.x; i < n; i += kSelThreads) out[i] = i;
    return;
  }
  const bool cached = (n <= cache_cap);
  const int E = (n + kSelThreads - 1) / kSelThreads;
  const int beg = min(n, (int)threadIdx.x * E), end = min(n, beg + E);
  auto key_at = [&](int i) -> uint32_t { return cached ? cache[i + (i >> 5)] : order_key(src[i]); };
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  if (cached) {
    for (int i = threadIdx.x; i < n; i += kSelThreads) cache[i + (i >> 5)] = order_key(src[i]);
    __syncthreads();
  }
  for (int i = beg; i < end; ++i) {
    const uint32_t u = key_at(i);
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  }
  // block min / max
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane_id() == 0) { sm.wsum[warp_id()] = (int)kmin; sm.wsum2[warp_id()] = (int)kmax; }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0xffffffffu, b = 0u;
    for (int q = 0; q < kSelWarps; ++q) { a = min(a, (uint32_t)sm.wsum[q]); b = max(b, (uint32_t)sm.wsum2[q]); }
    sm.bcast[2] = (int)a;
    sm.bcast[3] = (int)b;
  }
  __syncthreads();
  kmin = (uint32_t)sm.bcast[2];
  kmax = (uint32_t)sm.bcast[3];
  __syncthreads();

  uint32_t prefix = kmin, pmask = 0u;        // bits above `top` are common to every key
  int k_rem = k;
  if (kmin != kmax) {
    const int top = 31 - __clz(kmin ^ kmax);  // highest differing bit
    pmask = (top == 31) ? 0u : (0xffffffffu << (top + 1));
    prefix = kmin & pmask;
    for (int hi = top; hi >= 0; hi -= 11) {
      const int width = min(11, hi + 1), shift = hi + 1 - width, nb = 1 << width;
      for (int i = threadIdx.x; i < nb; i += kSelThreads) sm.hist[i] = 0;
      __syncthreads();
      for (int i = beg; i < end; ++i) {
        const uint32_t u = key_at(i);
        if ((u & pmask) == prefix) atomicAdd(&sm.hist[(u >> shift) & (nb - 1)], 1);
      }
      __syncthreads();
      // suffix counts from the top bin down: thread t owns bins nb-1-(t*per + q)
      const int per = (nb + kSelThreads - 1) / kSelThreads;
      int own = 0;
      for (int q = 0; q < per; ++q) {
        const int bin = nb - 1 - ((int)threadIdx.x * per + q);
        if (bin >= 0) own += sm.hist[bin];
      }
      int2 tot;
      const int above = block_exclusive_scan2(make_int2(own, 0), sm, &tot).x;
      int run = above;
      for (int q = 0; q < per; ++q) {
        const int bin = nb - 1 - ((int)threadIdx.x * per + q);
        if (bin < 0) break;
        const int cnt = sm.hist[bin];
        if (run < k_rem && run + cnt >= k_rem) { sm.bcast[0] = bin; sm.bcast[1] = run; }
        run += cnt;
      }
      __syncthreads();
      k_rem -= sm.bcast[1];
      prefix |= (uint32_t)sm.bcast[0] << shift;
      pmask |= (uint32_t)(nb - 1) << shift;
      __syncthreads();
    }
  }
  const uint32_t T = prefix;   // key of the k-th largest; take the first k_rem keys equal to T
  int gt = 0, eq = 0;
  for (int i = beg; i < end; ++i) {
    const uint32_t u = key_at(i);
    gt += u > T;
    eq += u == T;
  }
  int2 tot;
  const int2 ex = block_exclusive_scan2(make_int2(gt, eq), sm, &tot);
  int g_before = ex.x, e_before = ex.y;
  for (int i = beg; i < end; ++i) {
    const uint32_t u = key_at(i);
    if (u > T) {
      out[g_before + min(e_before, k_rem)] = i;
      ++g_before;
    } else if (u == T) {
      if (e_before < k_rem) out[g_before + e_before] = i;
      ++e_before;
    }
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
  *bytes = (size_t)(*cap + *cap / 32 + 1) * sizeof(uint32_t);
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)((kSmemKeysMax + kSmemKeysMax / 32 + 1) * 4));
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
