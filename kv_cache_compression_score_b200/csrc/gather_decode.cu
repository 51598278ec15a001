// Compact-cache gather, hidden-state gather (FastKV token-selective
// propagation, FastKV section 2.A) and split-K GQA decode attention over the
// compact cache.  All three are HBM streams: 16-byte vector loads and stores,
// no shared-memory staging needed for the gathers.
#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

// ------------------------------------------------------------------- gathers
constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 4;

// One 16-byte vector of one (slot t, head h) row per work item.
__global__ void __launch_bounds__(kGatherThreads)
gather_kv_kernel(const uint8_t *__restrict__ k, const uint8_t *__restrict__ v, uint8_t *__restrict__ k_out,
                 uint8_t *__restrict__ v_out, const int32_t *__restrict__ idx, const int *__restrict__ cu_seqlens,
                 const int *__restrict__ cu_budget, int n_kv, int vec_per_head, int total_budget) {
  const int b = blockIdx.y;
  const int t0 = cu_seqlens[b], len = cu_seqlens[b + 1] - t0;
  const int cb = cu_budget[b], kept = cu_budget[b + 1] - cb;
  const int row_vecs = n_kv * vec_per_head;
  const long long n_items = (long long)kept * row_vecs;
  const size_t head_bytes = (size_t)vec_per_head * 16;
  for (long long base = (long long)blockIdx.x * kGatherThreads * kGatherUnroll + threadIdx.x; base < n_items;
       base += (long long)gridDim.x * kGatherThreads * kGatherUnroll) {
    uint4 kv_k[kGatherUnroll], kv_v[kGatherUnroll];
    size_t dst_off[kGatherUnroll];
    bool ok[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const long long e = base + (long long)u * kGatherThreads;
      ok[u] = e < n_items;
      if (ok[u]) {
        const int t = (int)(e / row_vecs);
        const int rem = (int)(e - (long long)t * row_vecs);
        const int h = rem / vec_per_head, c = rem - h * vec_per_head;
        const int src_t = idx[(size_t)h * total_budget + cb + t];
        dst_off[u] = ((size_t)(cb + t) * n_kv + h) * head_bytes + (size_t)c * 16;
        if (src_t >= 0 && src_t < len) {
          const size_t src_off = ((size_t)(t0 + src_t) * n_kv + h) * head_bytes + (size_t)c * 16;
          kv_k[u] = ld_stream16(k + src_off);
          kv_v[u] = ld_stream16(v + src_off);
        } else {   // index outside the sequence: zero row, no out-of-bounds read
          kv_k[u] = make_uint4(0, 0, 0, 0);
          kv_v[u] = make_uint4(0, 0, 0, 0);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      if (ok[u]) {
        st_stream16(k_out + dst_off[u], kv_k[u]);
        st_stream16(v_out + dst_off[u], kv_v[u]);
      }
    }
  }
}

__global__ void __launch_bounds__(kGatherThreads)
gather_hidden_kernel(const uint8_t *__restrict__ hidden, uint8_t *__restrict__ out, const int32_t *__restrict__ idx,
                     int n_rows, int vec_per_row, int n_src) {
  const long long n_items = (long long)n_rows * vec_per_row;
  for (long long base = (long long)blockIdx.x * kGatherThreads * kGatherUnroll + threadIdx.x; base < n_items;
       base += (long long)gridDim.x * kGatherThreads * kGatherUnroll) {
    uint4 val[kGatherUnroll];
    size_t dst_off[kGatherUnroll];
    bool ok[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const long long e = base + (long long)u * kGatherThreads;
      ok[u] = e < n_items;
      if (ok[u]) {
        const int t = (int)(e / vec_per_row), c = (int)(e - (long long)t * vec_per_row);
        const size_t row_bytes = (size_t)vec_per_row * 16;
        dst_off[u] = (size_t)t * row_bytes + (size_t)c * 16;
        const int src = idx[t];
        val[u] = (src >= 0 && src < n_src) ? ld_stream16(hidden + (size_t)src * row_bytes + (size_t)c * 16)
                                           : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u)
      if (ok[u]) st_stream16(out + dst_off[u], val[u]);
  }
}

// ------------------------------------------------------------ decode (GQA)
// CTA = (chunk of cache rows, KV head h, batch entry b); 4 warps.  A row of
// d_h elements is split over LPR = d_h / 16 lanes (16 elements each), so a
// warp covers 32 / LPR rows per step.  The G query heads of h live in
// registers (pre-scaled to log2 units); logits are reduced over the LPR lanes
// of a row with xor-shuffles, then each row group keeps an online softmax
// (m, l, acc).  Row groups, warps and chunks are merged with the usual
// rescaling; the last CTA of a (b, h) to finish (atomic ticket, no waiting)
// merges the chunk partials and writes the output.
constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;

template <typename T> struct RowSlice;
template <> struct RowSlice<__nv_bfloat16> {   // 16 bf16 = 2 x 16 B
  uint4 a, b;
  KVC_DEVINL void load(const __nv_bfloat16 *p) { a = ld_stream16(p); b = ld_stream16(p + 8); }
  KVC_DEVINL void to_f32(float *f) const { Elem<__nv_bfloat16>::unpack(a, f); Elem<__nv_bfloat16>::unpack(b, f + 8); }
};
template <> struct RowSlice<float> {           // 16 fp32 = 4 x 16 B
  uint4 a, b, c, d;
  KVC_DEVINL void load(const float *p) {
    a = ld_stream16(p); b = ld_stream16(p + 4); c = ld_stream16(p + 8); d = ld_stream16(p + 12);
  }
  KVC_DEVINL void to_f32(float *f) const {
    Elem<float>::unpack(a, f); Elem<float>::unpack(b, f + 4); Elem<float>::unpack(c, f + 8); Elem<float>::unpack(d, f + 12);
  }
};

// merge (m2, l2, a2) into (m, l, a) -- log2-domain maxima
KVC_DEVINL void merge_scale(float m, float m2, float &s1, float &s2, float &mn) {
  mn = fmaxf(m, m2);
  if (mn == kNegInf) { s1 = 0.f; s2 = 0.f; return; }
  s1 = fast_exp2(m - mn);
  s2 = fast_exp2(m2 - mn);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecThreads)
gqa_decode_kernel(const T *__restrict__ q, const T *__restrict__ kc, const T *__restrict__ vc,
                  const int64_t *__restrict__ row_off, const int *__restrict__ kv_len, int n_h, int n_kv, float c,
                  int chunk_rows, int n_chunks, float *__restrict__ out, float *__restrict__ part,
                  int *__restrict__ tickets) {
  constexpr int LPR = D / 16;          // lanes per row
  constexpr int RPW = 32 / LPR;        // rows per warp step
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int len = kv_len[b];
  const int n_active = (len + chunk_rows - 1) / chunk_rows;
  const int lane = lane_id(), wid = warp_id();
  if (len == 0) {
    if (chunk == 0)
      for (int e = threadIdx.x; e < G * D; e += kDecThreads)
        out[((size_t)b * n_h + (size_t)h * G) * D + e] = 0.f;
    return;
  }
  if (chunk >= n_active) return;

  const int rg = lane / LPR, sl = lane % LPR;
  const int r_begin = chunk * chunk_rows, r_end = min(len, r_begin + chunk_rows);
  const int64_t o = row_off[b];

  float qr[G][16];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    RowSlice<T> s;
    s.load(q + ((size_t)b * n_h + (size_t)h * G + g) * D + sl * 16);
    s.to_f32(qr[g]);
#pragma unroll
    for (int e = 0; e < 16; ++e) qr[g][e] *= c;
  }
  float acc[G][16], m[G], l[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = kNegInf; l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[g][e] = 0.f;
  }

  const size_t row_stride = (size_t)n_kv * D;
  const T *kbase = kc + ((size_t)o * n_kv + h) * D + sl * 16;
  const T *vbase = vc + ((size_t)o * n_kv + h) * D + sl * 16;
  constexpr int kStep = kDecWarps * RPW;
  int row = r_begin + wid * RPW + rg;
  RowSlice<T> kn, vn;
  if (row < r_end) { kn.load(kbase + (size_t)row * row_stride); vn.load(vbase + (size_t)row * row_stride); }
  for (int base = r_begin; base < r_end; base += kStep) {
    const bool valid = row < r_end;
    RowSlice<T> kcur = kn, vcur = vn;
    const int nxt = row + kStep;
    if (nxt < r_end) { kn.load(kbase + (size_t)nxt * row_stride); vn.load(vbase + (size_t)nxt * row_stride); }
    float kf[16], vf[16];
    kcur.to_f32(kf);
    float s[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int e = 0; e < 16; e += 2) { a0 = fmaf(qr[g][e], kf[e], a0); a1 = fmaf(qr[g][e + 1], kf[e + 1], a1); }
      s[g] = a0 + a1;
    }
#pragma unroll
    for (int off = 1; off < LPR; off <<= 1)
#pragma unroll
      for (int g = 0; g < G; ++g) s[g] += __shfl_xor_sync(0xffffffffu, s[g], off);
    if (valid) {
      vcur.to_f32(vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (s[g] > m[g]) {
          const float a = fast_exp2(m[g] - s[g]);
          l[g] *= a;
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[g][e] *= a;
          m[g] = s[g];
        }
        const float p = fast_exp2(s[g] - m[g]);
        l[g] += p;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[g][e] = fmaf(p, vf[e], acc[g][e]);
      }
    }
    row = nxt;
  }

  // merge the row groups of the warp (lanes with the same slice)
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m[g], off);
      const float l2 = __shfl_xor_sync(0xffffffffu, l[g], off);
      float s1, s2, mn;
      merge_scale(m[g], m2, s1, s2, mn);
      l[g] = l[g] * s1 + l2 * s2;
      m[g] = mn;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a2 = __shfl_xor_sync(0xffffffffu, acc[g][e], off);
        acc[g][e] = acc[g][e] * s1 + a2 * s2;
      }
    }
  }

  // merge the warps through shared memory: [warp][g] -> (m, l), acc[D]
  __shared__ float sm_ml[kDecWarps][G][2];
  __shared__ float sm_acc[kDecWarps][G][D];
  if (rg == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (sl == 0) { sm_ml[wid][g][0] = m[g]; sm_ml[wid][g][1] = l[g]; }
#pragma unroll
      for (int e = 0; e < 16; ++e) sm_acc[wid][g][sl * 16 + e] = acc[g][e];
    }
  }
  __syncthreads();
  float *my_part = part + (((size_t)b * n_kv + h) * n_chunks + chunk) * (size_t)(G * (D + 2));
  for (int e = threadIdx.x; e < G * D; e += kDecThreads) {
    const int g = e / D, d = e % D;
    float M = kNegInf;
#pragma unroll
    for (int wv = 0; wv < kDecWarps; ++wv) M = fmaxf(M, sm_ml[wv][g][0]);
    float L = 0.f, A = 0.f;
#pragma unroll
    for (int wv = 0; wv < kDecWarps; ++wv) {
      const float mw = sm_ml[wv][g][0];
      if (mw == kNegInf) continue;
      const float sc = fast_exp2(mw - M);
      L = fmaf(sm_ml[wv][g][1], sc, L);
      A = fmaf(sm_acc[wv][g][d], sc, A);
    }
    if (n_active == 1) {
      out[((size_t)b * n_h + (size_t)h * G + g) * D + d] = A / L;
    } else {
      my_part[g * (D + 2) + 2 + d] = A;
      if (d == 0) { my_part[g * (D + 2)] = M; my_part[g * (D + 2) + 1] = L; }
    }
  }
  if (n_active == 1) return;

  // completion ticket: the last chunk CTA of (b, h) merges every chunk
  __shared__ int sm_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int t = atomicAdd(&tickets[b * n_kv + h], 1);
    sm_last = (t == n_active - 1);
  }
  __syncthreads();
  if (!sm_last) return;
  __threadfence();
  const float *pp = part + ((size_t)b * n_kv + h) * n_chunks * (size_t)(G * (D + 2));
  for (int e = threadIdx.x; e < G * D; e += kDecThreads) {
    const int g = e / D, d = e % D;
    float M = kNegInf;
    for (int cc = 0; cc < n_active; ++cc) M = fmaxf(M, __ldcg(pp + (size_t)cc * G * (D + 2) + g * (D + 2)));
    float L = 0.f, A = 0.f;
    for (int cc = 0; cc < n_active; ++cc) {
      const float *q0 = pp + (size_t)cc * G * (D + 2) + g * (D + 2);
      const float sc = fast_exp2(__ldcg(q0) - M);
      L = fmaf(__ldcg(q0 + 1), sc, L);
      A = fmaf(__ldcg(q0 + 2 + d), sc, A);
    }
    out[((size_t)b * n_h + (size_t)h * G + g) * D + d] = A / L;
  }
  if (threadIdx.x == 0) tickets[b * n_kv + h] = 0;   // leave the counter zeroed for the next call
}

template <typename T, int D, int G>
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
  dim3 grid(a.n_chunks, a.n_kv, a.batch);
  gqa_decode_kernel<T, D, G><<<grid, kDecThreads, 0, st>>>(
      static_cast<const T *>(a.q), static_cast<const T *>(a.k_c), static_cast<const T *>(a.v_c), a.row_off, a.kv_len,
      a.n_h, a.n_kv, a.scale * kLog2e, a.chunk_rows, a.n_chunks, a.out, a.part, a.tickets);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t decode_g(const DecodeArgs &a, cudaStream_t st) {
  switch (a.n_h / a.n_kv) {
    case 1: return launch_decode<T, D, 1>(a, st);
    case 2: return launch_decode<T, D, 2>(a, st);
    case 4: return launch_decode<T, D, 4>(a, st);
    default: return launch_decode<T, D, 8>(a, st);
  }
}

}  // namespace

cudaError_t gather_rows_kv(const void *k, const void *v, void *k_out, void *v_out, const int32_t *idx,
                           const int32_t *cu_seqlens, const int32_t *cu_budget, int n_seqs, int n_kv,
                           int row_bytes_per_head, int total_budget, int max_kept, cudaStream_t st) {
  const int vph = row_bytes_per_head / 16;
  const long long items = (long long)max_kept * n_kv * vph;
  long long blocks = (items + kGatherThreads * kGatherUnroll - 1) / (kGatherThreads * kGatherUnroll);
  if (blocks < 1) blocks = 1;
  if (blocks > 65535) blocks = 65535;
  dim3 grid((unsigned)blocks, n_seqs);
  gather_kv_kernel<<<grid, kGatherThreads, 0, st>>>(
      static_cast<const uint8_t *>(k), static_cast<const uint8_t *>(v), static_cast<uint8_t *>(k_out),
      static_cast<uint8_t *>(v_out), idx, cu_seqlens, cu_budget, n_kv, vph, total_budget);
  return cudaGetLastError();
}

cudaError_t gather_hidden(const void *hidden, void *out, const int32_t *idx, int n_rows, int row_bytes, int n_src,
                          cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const int vpr = row_bytes / 16;
  const long long items = (long long)n_rows * vpr;
  long long blocks = (items + kGatherThreads * kGatherUnroll - 1) / (kGatherThreads * kGatherUnroll);
  if (blocks > 65535) blocks = 65535;
  gather_hidden_kernel<<<(unsigned)blocks, kGatherThreads, 0, st>>>(
      static_cast<const uint8_t *>(hidden), static_cast<uint8_t *>(out), idx, n_rows, vpr, n_src);
  return cudaGetLastError();
}

cudaError_t gqa_decode(const DecodeArgs &a, cudaStream_t st) {
  if (a.dt == KVC_F32) {
    if (a.d_h == 64) return decode_g<float, 64>(a, st);
    return decode_g<float, 128>(a, st);
  }
  if (a.d_h == 64) return decode_g<__nv_bfloat16, 64>(a, st);
  return decode_g<__nv_bfloat16, 128>(a, st);
}

}  // namespace kvc
