// FreeKV decode-time retrieval with fine-grained correction (FreeKV, technical
// summary 2.A, "Récupération Spéculative" and "Correction Fine").  A decode
// step reuses the tokens retrieved for the previous step; a KV head whose
// query drifted (cosine similarity of the current and previous query below
// tau, for any query head of its group) is scored again with the current
// query and its tokens are selected and gathered again before attention.
//
// Kernels of one step (all flagged work is decided on the device, so the
// host never waits):
//   fk_flags       one warp per (sequence, KV head): G cosines, the flag, and
//                  the decode offsets / lengths of the compact caches;
//   fk_logits      flagged heads only, 1024 keys per CTA: the logits of the G
//                  query heads against every cached key as a tensor-core
//                  product in the transposed orientation (S^T = K . Q^T,
//                  mma.sync m16n8k16, the G heads on the N = 8 side, K rows
//                  staged per warp with cp.async into a swizzled tile), written
//                  in log2 units, plus each chunk's (max, sum of 2^(z - max));
//   fk_raw_pool    flagged heads only: merges the chunk statistics into the
//                  offset m + log2(l) of each query head, forms raw[j] =
//                  sum_g 2^(z_gj - off_g) on the chunk and its halo and
//                  max-pools it over the prefix (the window keeps +inf);
// then the cluster select and the compact gather of the standalone calls,
// restricted to the flagged heads, and decode attention over every head.
#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kFkWarps = 4;
constexpr int kFkThreads = kFkWarps * 32;
constexpr int kFkChunk = 1024;            // keys per CTA of the logit / pool passes
constexpr int kFkMaxR = 15;               // largest pool radius

template <int D, int G>
__global__ void __launch_bounds__(kFkThreads)
fk_flags_kernel(FreeKvArgs p) {
  grid_dependency_wait();
  const int u = blockIdx.x * kFkWarps + warp_id(), lane = lane_id();
  if (u >= p.batch * p.n_kv) return;
  const int b = u / p.n_kv, h = u % p.n_kv;
  float cmin = kPosInf;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const size_t row = ((size_t)b * p.n_h + (size_t)h * G + g) * D;
    float dot = 0.f, na = 0.f, nb = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float x = __bfloat162float(p.q_cur[row + d]), y = __bfloat162float(p.q_prev[row + d]);
      dot = fmaf(x, y, dot);
      na = fmaf(x, x, na);
      nb = fmaf(y, y, nb);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      dot += __shfl_xor_sync(0xffffffffu, dot, o);
      na += __shfl_xor_sync(0xffffffffu, na, o);
      nb += __shfl_xor_sync(0xffffffffu, nb, o);
    }
    const float den = sqrtf(na) * sqrtf(nb);
    cmin = fminf(cmin, den > 0.f ? dot / den : 0.f);
  }
  if (lane == 0) {
    p.flags[u] = cmin < p.tau ? 1 : 0;
    if (h == 0) {
      p.dec_off[b] = p.cu_budget[b];
      p.dec_len[b] = p.cu_budget[b + 1] - p.cu_budget[b];
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kFkThreads)
fk_logits_kernel(FreeKvArgs p) {
  grid_dependency_wait();
  constexpr int NKS = D / 16;
  constexpr int kTileB = 16 * D * 2;                 // 16 key rows of one head (bf16)
  __shared__ __align__(1024) uint8_t sk[kFkWarps][2][kTileB];
  __shared__ float2 sml[kFkWarps][8];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (!p.flags[b * p.n_kv + h]) return;
  const int t0 = p.cu_seqlens[b], len = p.cu_seqlens[b + 1] - t0;
  const int k0 = c * kFkChunk;
  if (k0 >= len) return;
  const int k1 = min(len, k0 + kFkChunk);
  const int warp = warp_id(), lane = lane_id();
  const int g = lane >> 2, t = lane & 3, lr = lane & 7, li = lane >> 3;

  uint32_t qf[NKS][2];
  {
    const __nv_bfloat16 *qb = p.q_cur + ((size_t)b * p.n_h + (size_t)h * G + g) * D;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      qf[ks][0] = g < G ? __ldg(reinterpret_cast<const uint32_t *>(qb + 16 * ks + 2 * t)) : 0u;
      qf[ks][1] = g < G ? __ldg(reinterpret_cast<const uint32_t *>(qb + 16 * ks + 8 + 2 * t)) : 0u;
    }
  }
  float m0 = kNegInf, m1 = kNegInf, l0 = 0.f, l1 = 0.f;   // heads 2t, 2t+1 of this lane
  float *zb = p.z + (size_t)(b * p.n_kv + h) * G * p.zpitch;
  const int n_groups = (k1 - k0 + 15) / 16;
  auto issue = [&](int gi, int buf) {
    const int key0 = k0 + gi * 16;
    for (int e = lane; e < 16 * (D / 8); e += 32) {
      const int r = e / (D / 8), ch = e % (D / 8);
      const bool ok = key0 + r < k1;
      const __nv_bfloat16 *src = p.k + ((size_t)(t0 + (ok ? key0 + r : k0)) * p.n_kv + h) * D + ch * 8;
      cp_async16(sk[warp][buf] + swz<128, 16>(r, ch), src, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  int buf = 0;
  if (warp < n_groups) issue(warp, 0);
  for (int gi = warp; gi < n_groups; gi += kFkWarps) {
    if (gi + kFkWarps < n_groups) {
      issue(gi + kFkWarps, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t base = smem_u32(sk[warp][buf]);
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      uint32_t a[4];
      ldsm_x4(base + swz<128, 16>(lr + (li & 1) * 8, 2 * ks + (li >> 1)), a);
      mma_bf16(sc, a, qf[ks][0], qf[ks][1]);
    }
    const int key0 = k0 + gi * 16;
    const bool v0 = key0 + g < k1, v1 = key0 + g + 8 < k1;
    const float z0 = v0 ? sc[0] * p.c : kNegInf, z1 = v0 ? sc[1] * p.c : kNegInf;
    const float z2 = v1 ? sc[2] * p.c : kNegInf, z3 = v1 ? sc[3] * p.c : kNegInf;
    if (2 * t < G) {
      if (v0) zb[(size_t)(2 * t) * p.zpitch + key0 + g] = z0;
      if (v1) zb[(size_t)(2 * t) * p.zpitch + key0 + g + 8] = z2;
    }
    if (2 * t + 1 < G) {
      if (v0) zb[(size_t)(2 * t + 1) * p.zpitch + key0 + g] = z1;
      if (v1) zb[(size_t)(2 * t + 1) * p.zpitch + key0 + g + 8] = z3;
    }
    float tm0 = fmaxf(z0, z2), tm1 = fmaxf(z1, z3);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o));
      tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o));
    }
    if (tm0 > m0) { l0 *= (m0 == kNegInf) ? 0.f : fast_exp2(m0 - tm0); m0 = tm0; }
    if (tm1 > m1) { l1 *= (m1 == kNegInf) ? 0.f : fast_exp2(m1 - tm1); m1 = tm1; }
    l0 += (v0 ? fast_exp2(z0 - m0) : 0.f) + (v1 ? fast_exp2(z2 - m0) : 0.f);
    l1 += (v0 ? fast_exp2(z1 - m1) : 0.f) + (v1 ? fast_exp2(z3 - m1) : 0.f);
    __syncwarp();                                   // the buffer is refilled by the next issue
    buf ^= 1;
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (g == 0) {
    sml[warp][2 * t] = make_float2(m0, l0);
    sml[warp][2 * t + 1] = make_float2(m1, l1);
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int hd = threadIdx.x;
    float M = kNegInf, Ls = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kFkWarps; ++w2) M = fmaxf(M, sml[w2][hd].x);
    if (M != kNegInf)
#pragma unroll
      for (int w2 = 0; w2 < kFkWarps; ++w2)
        if (sml[w2][hd].x != kNegInf) Ls += sml[w2][hd].y * fast_exp2(sml[w2][hd].x - M);
    p.part[((size_t)(b * p.n_kv + h) * p.n_chunks + c) * G + hd] = make_float2(M, Ls);
  }
}

template <int G>
__global__ void __launch_bounds__(256)
fk_raw_pool_kernel(FreeKvArgs p) {
  grid_dependency_wait();
  __shared__ float off[8];
  __shared__ float sraw[kFkChunk + 2 * kFkMaxR];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (!p.flags[b * p.n_kv + h]) return;
  const int t0 = p.cu_seqlens[b], len = p.cu_seqlens[b + 1] - t0;
  const int j0 = c * kFkChunk;
  if (j0 >= len) return;
  const int j1 = min(len, j0 + kFkChunk);
  const int P = len - p.w, r = p.pool_r;
  const int nc = (len + kFkChunk - 1) / kFkChunk;
  if (threadIdx.x < G) {
    const float2 *pp = p.part + (size_t)(b * p.n_kv + h) * p.n_chunks * G + threadIdx.x;
    float M = kNegInf, Ls = 0.f;
    for (int cc = 0; cc < nc; ++cc) {
      const float2 v = pp[(size_t)cc * G];
      const float mn = fmaxf(M, v.x);
      if (mn == kNegInf) continue;
      Ls = Ls * (M == kNegInf ? 0.f : fast_exp2(M - mn)) + (v.x == kNegInf ? 0.f : v.y * fast_exp2(v.x - mn));
      M = mn;
    }
    off[threadIdx.x] = M + __log2f(Ls);
  }
  __syncthreads();
  const float *zb = p.z + (size_t)(b * p.n_kv + h) * G * p.zpitch;
  const int n_halo = j1 - j0 + 2 * r;
  for (int e = threadIdx.x; e < n_halo; e += blockDim.x) {
    const int j = j0 - r + e;
    float a = kNegInf;                              // outside the prefix: ignored by the pool
    if (j >= 0 && j < P) {
      a = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) a += fast_exp2(zb[(size_t)g * p.zpitch + j] - off[g]);
    }
    sraw[e] = a;
  }
  __syncthreads();
  float *dst = p.scores + (size_t)h * p.T_total + t0;
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
    float v = kPosInf;                              // the window is always kept
    if (j < P) {
      const float *cptr = sraw + (j - j0 + r);
      v = cptr[0];
      for (int q = 1; q <= r; ++q) v = fmaxf(v, fmaxf(cptr[-q], cptr[q]));
    }
    dst[j] = v;
  }
}

template <int D, int G>
cudaError_t launch_fk(const FreeKvArgs &a, cudaStream_t st) {
  cudaError_t e;
  const int units = a.batch * a.n_kv;
  count_launch();
  if ((e = launch_pdl(fk_flags_kernel<D, G>, dim3((units + kFkWarps - 1) / kFkWarps), dim3(kFkThreads), 0, st, a)))
    return e;
  const dim3 grid(a.n_chunks, a.n_kv, a.batch);
  count_launch();
  if ((e = launch_pdl(fk_logits_kernel<D, G>, grid, dim3(kFkThreads), 0, st, a))) return e;
  count_launch();
  return launch_pdl(fk_raw_pool_kernel<G>, grid, dim3(256), 0, st, a);
}

template <int D>
cudaError_t by_group(const FreeKvArgs &a, cudaStream_t st) {
  switch (a.n_h / a.n_kv) {
    case 1: return launch_fk<D, 1>(a, st);
    case 2: return launch_fk<D, 2>(a, st);
    case 4: return launch_fk<D, 4>(a, st);
    default: return launch_fk<D, 8>(a, st);
  }
}

}  // namespace

int freekv_chunk_keys() { return kFkChunk; }

cudaError_t freekv_rescore(const FreeKvArgs &a, cudaStream_t st) {
  return a.d_h == 64 ? by_group<64>(a, st) : by_group<128>(a, st);
}

}  // namespace kvc
