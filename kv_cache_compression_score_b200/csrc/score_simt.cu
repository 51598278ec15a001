// Observation-window saliency scores on the CUDA cores (float32 inputs, and
// bf16 window blocks whose row count the tensor-core kernels do not take).
//
// Exact two-pass softmax (SnapKV-style observation-window scoring, "Variantes
// de l'attention et compression du cache KV", section "Compresser un cache
// existant"; causal offset of the window rows from section "Quand la
// reutilisation est-elle exacte ?"):
//   pass 1 (stats):  per window row, running max m and sum l of 2^(y - m) over
//                    the visible keys of one key chunk, y = log2(e) * scale * q.k;
//   pass 2 (score):  the chunk partials are merged per row into
//                    off = m + log2(l); each key j gets
//                    raw[j] = sum over rows of 2^(y_rj - off_r).
// Rows r = g * w + i (query head g of the KV head's group, window row i at
// absolute position P + i); a key j is visible to row r when j <= P + i.
//
// Tiles: 64 rows x 64 keys per step, 256 threads, each thread a 4x4 block of
// logits; operands staged transposed in shared memory (d-major) so the inner
// product reads two broadcast-free float4 per 16 FMAs.
#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kTK = 64;    // keys per tile
constexpr int kTR = 64;    // rows per row block
constexpr int kThreads = 256;
constexpr int kMaxRB = 4;  // up to 256 rows

struct SimtShape {
  int n_kv, n_h, G, w, R, R_pad, n_chunks, keys_per_chunk;
  float c;  // scale * log2(e)
};

template <typename T, int D>
struct SimtSmem {
  static constexpr int kQStride(int R_pad) { return R_pad + 4; }
  static size_t bytes(int R_pad) {
    return sizeof(float) * ((size_t)D * (R_pad + 4) + (size_t)D * (kTK + 4) + (size_t)R_pad + 16 * kTK);
  }
};

// Stage the whole window block of (b, h) transposed: Qs[d][r].
template <typename T, int D>
KVC_DEVINL void load_q_transposed(float *Qs, int qstride, const T *q_win, int b, int h, const SimtShape &s) {
  constexpr int V = Elem<T>::kPerVec;
  const int nvec = D / V;
  for (int e = threadIdx.x; e < s.R_pad * nvec; e += kThreads) {
    int r = e / nvec, dv = (e % nvec) * V;
    float f[8];
    if (r < s.R) {
      int g = r / s.w, i = r % s.w;
      const T *src = q_win + ((size_t)(b * s.w + i) * s.n_h + (size_t)h * s.G + g) * D + dv;
      Elem<T>::unpack(*reinterpret_cast<const uint4 *>(src), f);
    } else {
#pragma unroll
      for (int x = 0; x < V; ++x) f[x] = 0.f;
    }
#pragma unroll
    for (int x = 0; x < V; ++x) Qs[(dv + x) * qstride + r] = f[x];
  }
}

template <typename T, int D>
KVC_DEVINL void load_k_tile(float *Ks, const T *k, int t0, int key0, int len, int h, int n_kv) {
  constexpr int V = Elem<T>::kPerVec;
  constexpr int nvec = D / V;
  for (int e = threadIdx.x; e < kTK * nvec; e += kThreads) {
    int j = e / nvec, dv = (e % nvec) * V;
    float f[8];
    if (key0 + j < len) {
      const T *src = k + ((size_t)(t0 + key0 + j) * n_kv + h) * D + dv;
      Elem<T>::unpack(ld_nc16(src), f);
    } else {
#pragma unroll
      for (int x = 0; x < V; ++x) f[x] = 0.f;
    }
#pragma unroll
    for (int x = 0; x < V; ++x) Ks[(dv + x) * (kTK + 4) + j] = f[x];
  }
}

// acc[a][b] = sum_d Qs[d][row0 + ty*4 + a] * Ks[d][tx*4 + b]
template <int D>
KVC_DEVINL void tile_dot(const float *Qs, int qstride, int row0, const float *Ks, float acc[4][4]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 8
  for (int d = 0; d < D; ++d) {
    float4 qa = *reinterpret_cast<const float4 *>(Qs + d * qstride + row0 + ty * 4);
    float4 kb = *reinterpret_cast<const float4 *>(Ks + d * (kTK + 4) + tx * 4);
    float qv[4] = {qa.x, qa.y, qa.z, qa.w}, kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qv[a], kv[b], acc[a][b]);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
score_stats_simt(const T *__restrict__ q_win, const T *__restrict__ k, const int *__restrict__ cu_seqlens,
                 SimtShape s, float2 *__restrict__ part) {
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = cu_seqlens[b], len = cu_seqlens[b + 1] - t0;
  const int key_begin = c * s.keys_per_chunk;
  if (key_begin >= len) return;
  const int key_end = min(len, key_begin + s.keys_per_chunk);
  const int P = len - s.w;

  extern __shared__ float4 smem_f4[];
  float *Qs = reinterpret_cast<float *>(smem_f4);
  const int qstride = s.R_pad + 4;
  float *Ks = Qs + (size_t)D * qstride;

  load_q_transposed<T, D>(Qs, qstride, q_win, b, h, s);

  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int n_rb = s.R_pad / kTR;
  float m[kMaxRB][4], l[kMaxRB][4];
#pragma unroll
  for (int rb = 0; rb < kMaxRB; ++rb)
#pragma unroll
    for (int a = 0; a < 4; ++a) { m[rb][a] = kNegInf; l[rb][a] = 0.f; }

  for (int key0 = key_begin; key0 < key_end; key0 += kTK) {
    __syncthreads();
    load_k_tile<T, D>(Ks, k, t0, key0, len, h, s.n_kv);
    __syncthreads();
#pragma unroll
    for (int rb = 0; rb < kMaxRB; ++rb) {
      if (rb >= n_rb) break;
      float acc[4][4];
      tile_dot<D>(Qs, qstride, rb * kTR, Ks, acc);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int r = rb * kTR + ty * 4 + a;
        const int pos = P + (r % s.w);          // absolute position of the row
        float y[4], tmax = kNegInf;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const int j = key0 + tx * 4 + bb;
          y[bb] = (j < key_end && j <= pos) ? acc[a][bb] * s.c : kNegInf;
          tmax = fmaxf(tmax, y[bb]);
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        const float mn = fmaxf(m[rb][a], tmax);
        const float ms = (mn == kNegInf) ? 0.f : mn;   // nothing visible yet: keep l = 0
        float ps = 0.f;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) ps += fast_exp2(y[bb] - ms);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l[rb][a] = l[rb][a] * fast_exp2(m[rb][a] - ms) + ps;
        m[rb][a] = mn;
      }
    }
  }
  if (tx == 0) {
    float2 *dst = part + ((size_t)(b * s.n_kv + h) * s.n_chunks + c) * s.R_pad;
#pragma unroll
    for (int rb = 0; rb < kMaxRB; ++rb) {
      if (rb >= n_rb) break;
#pragma unroll
      for (int a = 0; a < 4; ++a) dst[rb * kTR + ty * 4 + a] = make_float2(m[rb][a], l[rb][a]);
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
score_raw_simt(const T *__restrict__ q_win, const T *__restrict__ k, const int *__restrict__ cu_seqlens,
               SimtShape s, const float2 *__restrict__ part, float *__restrict__ raw, int T_total) {
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = cu_seqlens[b], len = cu_seqlens[b + 1] - t0;
  const int key_begin = c * s.keys_per_chunk;
  if (key_begin >= len) return;
  const int key_end = min(len, key_begin + s.keys_per_chunk);
  const int P = len - s.w;
  const int n_chunks_b = (len + s.keys_per_chunk - 1) / s.keys_per_chunk;

  extern __shared__ float4 smem_f4[];
  float *Qs = reinterpret_cast<float *>(smem_f4);
  const int qstride = s.R_pad + 4;
  float *Ks = Qs + (size_t)D * qstride;
  float *off = Ks + (size_t)D * (kTK + 4);
  float *red = off + s.R_pad;                 // [16][kTK]

  // merge the chunk partials of every row: off = M + log2(L)
  const float2 *pp = part + (size_t)(b * s.n_kv + h) * s.n_chunks * s.R_pad;
  for (int r = threadIdx.x; r < s.R_pad; r += kThreads) {
    float o = kPosInf;
    if (r < s.R) {
      float M = kNegInf;
      for (int cc = 0; cc < n_chunks_b; ++cc) M = fmaxf(M, pp[(size_t)cc * s.R_pad + r].x);
      float L = 0.f;
      for (int cc = 0; cc < n_chunks_b; ++cc) {
        float2 v = pp[(size_t)cc * s.R_pad + r];
        if (v.x != kNegInf) L += v.y * fast_exp2(v.x - M);
      }
      o = M + __log2f(L);
    }
    off[r] = o;
  }
  load_q_transposed<T, D>(Qs, qstride, q_win, b, h, s);

  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int n_rb = s.R_pad / kTR;
  for (int key0 = key_begin; key0 < key_end; key0 += kTK) {
    __syncthreads();
    load_k_tile<T, D>(Ks, k, t0, key0, len, h, s.n_kv);
    __syncthreads();
    float col[4] = {0.f, 0.f, 0.f, 0.f};
    for (int rb = 0; rb < n_rb; ++rb) {
      float acc[4][4];
      tile_dot<D>(Qs, qstride, rb * kTR, Ks, acc);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int r = rb * kTR + ty * 4 + a;
        const int pos = P + (r % s.w);
        const float o = off[r];
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const int j = key0 + tx * 4 + bb;
          if (j <= pos) col[bb] += fast_exp2(fmaf(acc[a][bb], s.c, -o));
        }
      }
    }
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) red[ty * kTK + tx * 4 + bb] = col[bb];
    __syncthreads();
    if (threadIdx.x < kTK) {
      const int j = key0 + threadIdx.x;
      float sum = 0.f;
#pragma unroll
      for (int t = 0; t < 16; ++t) sum += red[t * kTK + threadIdx.x];
      if (j < key_end) raw[(size_t)h * T_total + t0 + j] = sum;
    }
  }
}

}  // namespace

template <typename T, int D>
static cudaError_t launch_simt(const ScoreArgs &a, cudaStream_t st) {
  SimtShape s;
  s.n_kv = a.n_kv; s.n_h = a.n_h; s.G = a.n_h / a.n_kv; s.w = a.w;
  s.R = s.G * a.w;
  s.R_pad = a.R_pad;   // multiple of the row block, >= R
  s.n_chunks = a.n_chunks;
  s.keys_per_chunk = a.keys_per_chunk;
  s.c = a.scale * kLog2e;
  const size_t smem = SimtSmem<T, D>::bytes(s.R_pad);
  cudaError_t e;
  e = ensure_smem_limit((const void *)score_stats_simt<T, D>, (int)smem);
  if (e != cudaSuccess) return e;
  e = ensure_smem_limit((const void *)score_raw_simt<T, D>, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_chunks, a.n_kv, a.n_seqs);
  score_stats_simt<T, D><<<grid, kThreads, smem, st>>>(
      static_cast<const T *>(a.q_win), static_cast<const T *>(a.k), a.cu_seqlens, s, a.part);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  score_raw_simt<T, D><<<grid, kThreads, smem, st>>>(
      static_cast<const T *>(a.q_win), static_cast<const T *>(a.k), a.cu_seqlens, s, a.part, a.raw, a.T_total);
  count_launch();
  return cudaGetLastError();
}

int simt_keys_per_tile() { return kTK; }

cudaError_t score_window_simt(const ScoreArgs &a, cudaStream_t st) {
  if (a.dt == KVC_F32) {
    if (a.d_h == 64) return launch_simt<float, 64>(a, st);
    return launch_simt<float, 128>(a, st);
  }
  if (a.d_h == 64) return launch_simt<__nv_bfloat16, 64>(a, st);
  return launch_simt<__nv_bfloat16, 128>(a, st);
}

}  // namespace kvc
