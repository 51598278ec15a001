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
// exacte ?" of the same page), then the window positions.  A cluster of 8
// CTAs per (sequence, head) runs an MSB-first radix select on order-preserving
// 32-bit keys: 11-bit digits starting at the highest bit where the keys
// differ, per-CTA histograms summed through distributed shared memory, so it
// finds the k-th largest key T and how many keys equal to T are taken; one
// ordered pass then writes position = (#keys > T before it) + min(#keys == T
// before it, taken).
#include <cooperative_groups.h>

#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace cg = cooperative_groups;

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
// float -> uint32 with the same order (negatives below positives, NaN on top)
KVC_DEVINL uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------- cluster selection
// One thread-block cluster of kClu CTAs per (sequence, head).  CTA r owns the
// contiguous slice r of the n keys (so index order is (rank, thread run,
// position)); the radix histograms are built per CTA and summed by every CTA
// through distributed shared memory, so all CTAs take identical decisions.
constexpr int kClu = 8;
constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;
constexpr int kCBins = 2048;
constexpr int kCCacheMax = 40960;     // keys per CTA slice cached in shared memory

constexpr int kCandLocal = kCThreads;           // candidate keys one CTA may contribute
constexpr int kCandTotal = kClu * kCandLocal;   // candidate keys of the whole cluster

struct __align__(16) CSel {
  int hist[2][kCBins];
  uint32_t cand[kCandLocal];     // this CTA's keys in the threshold bucket
  uint32_t all[kCandTotal];      // every CTA's candidates, in rank order
  int wsum[kCWarps];
  int wsum2[kCWarps];
  int bcast[4];
  unsigned int kmm[2];   // this CTA's min / max key
  int cnt[2];            // this CTA's (#keys > T, #keys == T)
  int ncand;             // candidates collected by this CTA (> kCandLocal: overflow)
  int sel[4];            // threshold decision shared by the block
};

KVC_DEVINL void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
KVC_DEVINL uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// `p` (in this CTA's shared memory) as seen in CTA `rank` of the cluster;
// plain loads through the mapped pointer, ordered by the cluster barriers
template <typename T> KVC_DEVINL T *remote(T *p, uint32_t rank) {
  return cg::this_cluster().map_shared_rank(p, rank);
}

KVC_DEVINL int2 cblock_scan2(int2 v, CSel &sm, int2 *total) {
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
    int a = lane < kCWarps ? sm.wsum[lane] : 0, b = lane < kCWarps ? sm.wsum2[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int c = __shfl_up_sync(0xffffffffu, a, o), d = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) { a += c; b += d; }
    }
    if (lane < kCWarps) { sm.wsum[lane] = a; sm.wsum2[lane] = b; }
  }
  __syncthreads();
  const int bx = wid ? sm.wsum[wid - 1] : 0, by = wid ? sm.wsum2[wid - 1] : 0;
  *total = make_int2(sm.wsum[kCWarps - 1], sm.wsum2[kCWarps - 1]);
  __syncthreads();
  return make_int2(bx + x - v.x, by + y - v.y);
}

// Adaptive multi-pass radix select (the general path): 11-bit digits from the
// highest bit where the keys differ, one cluster-wide histogram per digit.
// Same contract as cluster_topk_ascending.
KVC_DEVINL void cluster_topk_adaptive(const float *__restrict__ src, int n, int k, int32_t *__restrict__ out,
                                      uint32_t *cache, CSel &sm) {
  const uint32_t rank = cluster_rank();
  const int tid = threadIdx.x;
  const int per = (n + kClu - 1) / kClu;
  const int s0 = min(n, (int)rank * per), ns = min(n, s0 + per) - s0;
  const bool cached = ns <= kCCacheMax;
  const int E = (ns + kCThreads - 1) / kCThreads;
  const int beg = min(ns, tid * E), end = min(ns, beg + E);
  auto key_at = [&](int i) -> uint32_t { return cached ? cache[i + (i >> 5)] : order_key(src[s0 + i]); };

  uint32_t kmin = 0xffffffffu, kmax = 0u;
  if (cached) {
    for (int i = tid; i < ns; i += kCThreads) cache[i + (i >> 5)] = order_key(src[s0 + i]);
    __syncthreads();
  }
  for (int i = beg; i < end; ++i) {
    const uint32_t u = key_at(i);
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane_id() == 0) { sm.wsum[warp_id()] = (int)kmin; sm.wsum2[warp_id()] = (int)kmax; }
  __syncthreads();
  if (tid == 0) {
    uint32_t a = 0xffffffffu, b = 0u;
    for (int q = 0; q < kCWarps; ++q) { a = min(a, (uint32_t)sm.wsum[q]); b = max(b, (uint32_t)sm.wsum2[q]); }
    sm.kmm[0] = a;
    sm.kmm[1] = b;
  }
  cluster_sync_all();
  if (tid == 0) {
    uint32_t a = 0xffffffffu, b = 0u;
    for (uint32_t r = 0; r < kClu; ++r) {
      a = min(a, *remote(&sm.kmm[0], r));
      b = max(b, *remote(&sm.kmm[1], r));
    }
    sm.bcast[2] = (int)a;
    sm.bcast[3] = (int)b;
  }
  __syncthreads();
  kmin = (uint32_t)sm.bcast[2];
  kmax = (uint32_t)sm.bcast[3];

  uint32_t prefix = kmin, pmask = 0u;
  int k_rem = k;
  if (kmin != kmax) {
    const int top = 31 - __clz(kmin ^ kmax);
    pmask = (top == 31) ? 0u : (0xffffffffu << (top + 1));
    prefix = kmin & pmask;
    int pass = 0;
    for (int hi = top; hi >= 0; hi -= 11, ++pass) {
      const int width = min(11, hi + 1), shift = hi + 1 - width, nb = 1 << width;
      int *H = sm.hist[pass & 1];
      for (int i = tid; i < nb; i += kCThreads) H[i] = 0;
      __syncthreads();
      for (int i = beg; i < end; ++i) {
        const uint32_t u = key_at(i);
        if ((u & pmask) == prefix) atomicAdd(&H[(u >> shift) & (nb - 1)], 1);
      }
      cluster_sync_all();   // every CTA's histogram of this pass is complete
      // global counts of the bins this thread owns, from the top bin down
      const int bper = (nb + kCThreads - 1) / kCThreads;
      int cnt[4], own = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        cnt[q] = 0;
        const int bin = nb - 1 - (tid * bper + q);
        if (q < bper && bin >= 0) {
          int v[kClu];
#pragma unroll
          for (uint32_t r = 0; r < kClu; ++r) v[r] = *remote(&H[bin], r);   // independent remote loads
#pragma unroll
          for (uint32_t r = 0; r < kClu; ++r) cnt[q] += v[r];
          own += cnt[q];
        }
      }
      int2 tot;
      int run = cblock_scan2(make_int2(own, 0), sm, &tot).x;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int bin = nb - 1 - (tid * bper + q);
        if (q < bper && bin >= 0) {
          if (run < k_rem && run + cnt[q] >= k_rem) { sm.bcast[0] = bin; sm.bcast[1] = run; }
          run += cnt[q];
        }
      }
      __syncthreads();
      k_rem -= sm.bcast[1];
      prefix |= (uint32_t)sm.bcast[0] << shift;
      pmask |= (uint32_t)(nb - 1) << shift;
      __syncthreads();
    }
  }
  const uint32_t T = prefix;
  int gt = 0, eq = 0;
  for (int i = beg; i < end; ++i) {
    const uint32_t u = key_at(i);
    gt += u > T;
    eq += u == T;
  }
  int2 tot;
  const int2 ex = cblock_scan2(make_int2(gt, eq), sm, &tot);
  if (tid == 0) { sm.cnt[0] = tot.x; sm.cnt[1] = tot.y; }
  cluster_sync_all();
  if (tid == 0) {
    int g0 = 0, e0 = 0;
    for (uint32_t r = 0; r < rank; ++r) {
      g0 += *remote(&sm.cnt[0], r);
      e0 += *remote(&sm.cnt[1], r);
    }
    sm.bcast[0] = g0;
    sm.bcast[1] = e0;
  }
  __syncthreads();
  int g_before = sm.bcast[0] + ex.x, e_before = sm.bcast[1] + ex.y;
  for (int i = beg; i < end; ++i) {
    const uint32_t u = key_at(i);
    if (u > T) {
      out[g_before + min(e_before, k_rem)] = s0 + i;
      ++g_before;
    } else if (u == T) {
      if (e_before < k_rem) out[g_before + e_before] = s0 + i;
      ++e_before;
    }
  }
  cluster_sync_all();   // no CTA leaves while another may still read its shared memory
}


// Block-wide radix select over keys[0..n) in shared memory (one CTA): the
// k-th largest key T and how many keys equal to T are among the k largest.
KVC_DEVINL void block_kth_largest(const uint32_t *keys, int n, int k, CSel &sm, uint32_t *T_out, int *take_eq,
                                  int hi_bit = 31, uint32_t prefix = 0u, uint32_t pmask = 0u) {
  const int tid = threadIdx.x;
  int k_rem = k;
  for (int hi = hi_bit; hi >= 0; hi -= 11) {
    const int width = min(11, hi + 1), shift = hi + 1 - width, nb = 1 << width;
    int *H = sm.hist[1];
    for (int i = tid; i < nb; i += kCThreads) H[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kCThreads)
      if ((keys[i] & pmask) == prefix) atomicAdd(&H[(keys[i] >> shift) & (nb - 1)], 1);
    __syncthreads();
    const int bper = (nb + kCThreads - 1) / kCThreads;
    int own = 0;
    for (int q = 0; q < bper; ++q) {
      const int bin = nb - 1 - (tid * bper + q);
      if (bin >= 0) own += H[bin];
    }
    int2 tot;
    int run = cblock_scan2(make_int2(own, 0), sm, &tot).x;
    for (int q = 0; q < bper; ++q) {
      const int bin = nb - 1 - (tid * bper + q);
      if (bin < 0) break;
      const int c = H[bin];
      if (run < k_rem && run + c >= k_rem) { sm.sel[0] = bin; sm.sel[1] = run; }
      run += c;
    }
    __syncthreads();
    k_rem -= sm.sel[1];
    prefix |= (uint32_t)sm.sel[0] << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    __syncthreads();
  }
  *T_out = prefix;
  *take_eq = k_rem;
}

// First-level bucket of a key: 32 sub-bins per binade for scores in
// [2^-30, 2^34), lower scores (and negative ones) in bin 0, higher in bin 2047.
// Monotone in the key, so whole buckets above the threshold bucket are
// selected and whole buckets below are not.
KVC_DEVINL constexpr int top_digit_lo() { return (int)((0x80000000u | (97u << 23)) >> 18); }   // key of 2^-30 / 2^18
KVC_DEVINL int top_digit(uint32_t u) {
  const int d = (int)(u >> 18) - top_digit_lo();
  return d < 0 ? 0 : (d > kCBins - 1 ? kCBins - 1 : d);
}

// Ascending positions of the k largest of src[0..n) (ties: lower index) to
// out[0..k), computed by the whole cluster.  0 < k < n.  Every thread of every
// CTA of the cluster must call it.
//
// One histogram of a 2048-bucket log-scale digit of the score locates the
// bucket holding the k-th largest key; the keys of
// that bucket (the candidates) are gathered from every CTA and the exact
// threshold is found locally.  Buckets too full for the candidate buffers
// fall back to the adaptive multi-pass select.
KVC_DEVINL void cluster_topk_ascending(const float *__restrict__ src, int n, int k, int32_t *__restrict__ out,
                                       uint32_t *cache, CSel &sm) {
  const uint32_t rank = cluster_rank();
  const int tid = threadIdx.x;
  const int per = (n + kClu - 1) / kClu;
  const int s0 = min(n, (int)rank * per), ns = min(n, s0 + per) - s0;
  if (per > kCCacheMax) {          // uniform across the cluster (slices are at most `per` long)
    cluster_topk_adaptive(src, n, k, out, cache, sm);
    return;
  }
  const int E = (ns + kCThreads - 1) / kCThreads;
  const int beg = min(ns, tid * E), end = min(ns, beg + E);
  int *H = sm.hist[0];
  for (int i = tid; i < kCBins; i += kCThreads) H[i] = 0;
  if (tid == 0) sm.ncand = 0;
  // keys into shared memory (one pad word per 32: conflict-free runs)
  {
    constexpr int U = 8;
    for (int i0 = tid; i0 < ns; i0 += U * kCThreads) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kCThreads;
        v[u] = i < ns ? src[s0 + i] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * kCThreads;
        if (i < ns) cache[i + (i >> 5)] = order_key(v[u]);
      }
    }
  }
  __syncthreads();
  for (int i = beg; i < end; ++i) atomicAdd(&H[top_digit(cache[i + (i >> 5)])], 1);
  cluster_sync_all();                                   // (1) every CTA's histogram is complete

  // cluster histogram of the 4 bins this thread owns (from the top), one int4 per CTA
  const int b_lo = kCBins - 4 - 4 * tid;                // bins b_lo .. b_lo + 3
  int4 hv[kClu];
#pragma unroll
  for (uint32_t r = 0; r < kClu; ++r) hv[r] = *remote(reinterpret_cast<int4 *>(H + b_lo), r);
  int c4[4] = {0, 0, 0, 0};
#pragma unroll
  for (uint32_t r = 0; r < kClu; ++r) { c4[0] += hv[r].w; c4[1] += hv[r].z; c4[2] += hv[r].y; c4[3] += hv[r].x; }
  int2 tot;
  int run = cblock_scan2(make_int2(c4[0] + c4[1] + c4[2] + c4[3], 0), sm, &tot).x;
#pragma unroll
  for (int q = 0; q < 4; ++q) {                         // bins b_lo + 3 - q, descending
    if (run < k && run + c4[q] >= k) { sm.sel[0] = b_lo + 3 - q; sm.sel[1] = run; }
    run += c4[q];
  }
  __syncthreads();
  const int bstar = sm.sel[0], above = sm.sel[1];      // keys in bins > bstar (whole cluster)
  // this CTA's candidates: its keys in bucket bstar
  // (one shared atomic per warp and step: the lanes holding a candidate take
  // consecutive slots)
  for (int q = 0; q < E; ++q) {
    const int i = beg + q;
    const uint32_t u = i < end ? cache[i + (i >> 5)] : 0u;
    const bool c = i < end && top_digit(u) == bstar;
    const uint32_t m = __ballot_sync(0xffffffffu, c);
    if (m) {
      int base = 0;
      if (lane_id() == __ffs(m) - 1) base = atomicAdd(&sm.ncand, __popc(m));
      base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
      if (c) {
        const int slot = base + __popc(m & ((1u << lane_id()) - 1u));
        if (slot < kCandLocal) sm.cand[slot] = u;
      }
    }
  }
  cluster_sync_all();                                   // (2) every CTA's candidates are listed
  // counts and candidate blocks of every CTA in one round of remote loads;
  // blocks are fixed-size, only the first nc[r] entries are meaningful
  int nc[kClu], total = 0;
  bool overflow = false;
#pragma unroll
  for (uint32_t r = 0; r < kClu; ++r) nc[r] = *remote(&sm.ncand, r);
  {
    uint32_t v[kClu];
    const int i = tid;                                  // kCandLocal == kCThreads
#pragma unroll
    for (uint32_t r = 0; r < kClu; ++r) v[r] = *remote(&sm.cand[i], r);
#pragma unroll
    for (uint32_t r = 0; r < kClu; ++r) sm.all[r * kCandLocal + i] = v[r];
  }
#pragma unroll
  for (uint32_t r = 0; r < kClu; ++r) {
    overflow |= nc[r] > kCandLocal;
    total += nc[r];
  }
  if (overflow) {                                       // uniform decision: every CTA read the same counts
    cluster_sync_all();                                 // nobody still reads this pass's buffers
    cluster_topk_adaptive(src, n, k, out, cache, sm);
    return;
  }
  __syncthreads();
  // compact the blocks (rank order) into sm.all[0..total)
  {
    uint32_t v[kClu];
    const int i = tid;
#pragma unroll
    for (uint32_t r = 0; r < kClu; ++r) v[r] = sm.all[r * kCandLocal + i];
    __syncthreads();
    int base = 0;
#pragma unroll
    for (uint32_t r = 0; r < kClu; ++r) {
      if (i < nc[r]) sm.all[base + i] = v[r];
      base += nc[r];
    }
  }
  __syncthreads();
  uint32_t T;
  int take_eq;
  const int k_rem = k - above;
  if (total <= kCThreads) {
    // small candidate set: exact rank of each candidate by counting
    if (tid == 0) sm.sel[2] = 0;
    __syncthreads();
    if (tid < total) {
      const uint32_t mine = sm.all[tid];
      int gtc = 0, eqc = 0;
      for (int j = 0; j < total; ++j) {
        const uint32_t o = sm.all[j];
        gtc += o > mine;
        eqc += o == mine;
      }
      if (gtc < k_rem && gtc + eqc >= k_rem) { sm.sel[2] = (int)mine; sm.sel[3] = k_rem - gtc; }
    }
    __syncthreads();
    T = (uint32_t)sm.sel[2];
    take_eq = sm.sel[3];
  } else if (bstar > 0 && bstar < kCBins - 1) {
    // every candidate has the 14 key bits 31..18 of bucket bstar
    const uint32_t hi14 = ((uint32_t)(bstar + top_digit_lo()) << 18);
    block_kth_largest(sm.all, total, k_rem, sm, &T, &take_eq, 17, hi14, 0xfffc0000u);
  } else {
    block_kth_largest(sm.all, total, k_rem, sm, &T, &take_eq);
  }
  // (#keys > T, #keys == T) in each CTA before this one: bins above bstar plus
  // candidates above / equal to T
  int g_rank = 0, e_rank = 0;
  {
    int base = 0;
    for (uint32_t r = 0; r < rank; ++r) {
      for (int i = tid; i < nc[r]; i += kCThreads) {
        const uint32_t u = sm.all[base + i];
        g_rank += u > T;
        e_rank += u == T;
      }
      base += nc[r];
    }
    // bins above bstar held by lower ranks
    int above_lower = 0;
#pragma unroll
    for (uint32_t r = 0; r < kClu; ++r) {
      if (r >= rank) break;
      const int hb[4] = {hv[r].w, hv[r].z, hv[r].y, hv[r].x};
#pragma unroll
      for (int q = 0; q < 4; ++q) above_lower += (b_lo + 3 - q > bstar) ? hb[q] : 0;
    }
    g_rank += above_lower;
  }
  const int2 pre = cblock_scan2(make_int2(g_rank, e_rank), sm, &tot);   // only totals used
  const int gt_before_cta = tot.x, eq_before_cta = tot.y;
  (void)pre;
  // this thread's run
  int gt = 0, eq = 0;
  for (int i = beg; i < end; ++i) {
    const uint32_t u = cache[i + (i >> 5)];
    gt += u > T;
    eq += u == T;
  }
  const int2 ex = cblock_scan2(make_int2(gt, eq), sm, &tot);
  int g_before = gt_before_cta + ex.x, e_before = eq_before_cta + ex.y;
  for (int i = beg; i < end; ++i) {
    const uint32_t u = cache[i + (i >> 5)];
    if (u > T) {
      out[g_before + min(e_before, take_eq)] = s0 + i;
      ++g_before;
    } else if (u == T) {
      if (e_before < take_eq) out[g_before + e_before] = s0 + i;
      ++e_before;
    }
  }
  cluster_sync_all();   // (3) no CTA leaves while another may still read its shared memory
}

__global__ void __launch_bounds__(kCThreads)
select_topk_cluster(const float *__restrict__ scores, int32_t *__restrict__ idx, const int *__restrict__ cu_seqlens,
                    const int *__restrict__ cu_budget, int T_total, int total_budget, int w, int budget,
                    const int *__restrict__ mask) {
  grid_dependency_wait();
  allow_dependents();
  const int h = blockIdx.x / kClu, b = blockIdx.y;
  if (mask && !mask[b * (gridDim.x / kClu) + h]) return;   // the same decision in every CTA of the cluster
  const uint32_t rank = cluster_rank();
  const int t0 = cu_seqlens[b], len = cu_seqlens[b + 1] - t0;
  int32_t *dst = idx + (size_t)h * total_budget + cu_budget[b];
  if (budget >= len) {           // identical decision in every CTA of the cluster
    for (int t = rank * kCThreads + threadIdx.x; t < len; t += kClu * kCThreads) dst[t] = t;
    return;
  }
  const int P = len - w, k_sel = budget - w;
  extern __shared__ uint32_t csel_cache[];
  __shared__ CSel sm;
  if (k_sel > 0) cluster_topk_ascending(scores + (size_t)h * T_total + t0, P, k_sel, dst, csel_cache, sm);
  if (rank == 0)
    for (int t = threadIdx.x; t < w; t += kCThreads) dst[k_sel + t] = P + t;
}

__global__ void __launch_bounds__(kCThreads)
tsp_select_cluster(const float *__restrict__ pooled, int S, int w, int k_tsp, int32_t *__restrict__ idx_out) {
  grid_dependency_wait();
  allow_dependents();
  const uint32_t rank = cluster_rank();
  const int P = S - w;
  extern __shared__ uint32_t csel_cache[];
  __shared__ CSel sm;
  if (k_tsp >= P) {
    for (int t = rank * kCThreads + threadIdx.x; t < P; t += kClu * kCThreads) idx_out[t] = t;
  } else if (k_tsp > 0) {
    cluster_topk_ascending(pooled, P, k_tsp, idx_out, csel_cache, sm);
  }
  if (rank == 0)
    for (int t = threadIdx.x; t < w; t += kCThreads) idx_out[k_tsp + t] = P + t;
}

}  // namespace

cudaError_t pool_prefix(const float *raw, float *scores, const int32_t *cu_seqlens, int n_seqs, int n_kv,
                        int T_total, int max_len, int w, int pool_k, cudaStream_t st) {
  dim3 grid((max_len + kPoolTile - 1) / kPoolTile, n_kv, n_seqs);
  pool_prefix_kernel<<<grid, kPoolThreads, 0, st>>>(raw, scores, cu_seqlens, T_total, w, (pool_k - 1) / 2);
  count_launch();
  return cudaGetLastError();
}

cudaError_t tsp_pool(const float *raw, int n_rows, int S, int w, int pool_k, float *pooled, cudaStream_t st) {
  const int P = S - w;
  if (P <= 0) return cudaSuccess;
  tsp_pool_kernel<<<(P + kPoolTile - 1) / kPoolTile, kPoolThreads, 0, st>>>(raw, n_rows, S, w, (pool_k - 1) / 2,
                                                                            pooled);
  count_launch();
  return cudaGetLastError();
}

static cudaError_t launch_cluster(const void *fn, dim3 grid, size_t smem, cudaStream_t st, void **args) {
  cudaError_t e = ensure_smem_limit((const void *)fn, (int)((kCCacheMax + kCCacheMax / 32 + 1) * 4));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kCThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClu;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  return cudaLaunchKernelExC(&cfg, fn, args);
}

static size_t cluster_cache_bytes(int n) {
  const int per = (n + kClu - 1) / kClu;
  const int cap = per <= kCCacheMax ? per : 0;
  return (size_t)(cap + cap / 32 + 1) * sizeof(uint32_t);
}

cudaError_t select_topk(const float *scores, int32_t *idx, const int32_t *cu_seqlens, const int32_t *cu_budget,
                        int n_seqs, int n_kv, int T_total, int total_budget, int w, int budget, int max_len,
                        cudaStream_t st, const int32_t *mask) {
  void *args[] = {(void *)&scores, (void *)&idx, (void *)&cu_seqlens, (void *)&cu_budget, (void *)&T_total,
                  (void *)&total_budget, (void *)&w, (void *)&budget, (void *)&mask};
  return launch_cluster((const void *)select_topk_cluster, dim3(kClu * n_kv, n_seqs), cluster_cache_bytes(max_len - w),
                        st, args);
}

cudaError_t tsp_select(const float *pooled, int S, int w, int k_tsp, int32_t *idx_out, cudaStream_t st) {
  void *args[] = {(void *)&pooled, (void *)&S, (void *)&w, (void *)&k_tsp, (void *)&idx_out};
  return launch_cluster((const void *)tsp_select_cluster, dim3(kClu), cluster_cache_bytes(S - w), st, args);
}

}  // namespace kvc
