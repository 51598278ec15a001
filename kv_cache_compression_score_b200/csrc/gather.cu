// Compact-cache gather (SnapKV keeps the chosen subset of past keys and
// values, "Variantes de l'attention et compression du cache KV", section
// "Compresser un cache existant") and hidden-state gather (FastKV token-
// selective propagation, FastKV section 2.A).  Both are HBM streams of
// 16-byte vector loads and stores; an index outside its sequence yields a
// zero row instead of an out-of-bounds read.
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
                 const int *__restrict__ cu_budget, int n_kv, int vec_per_head, int total_budget,
                 const int *__restrict__ mask) {
  grid_dependency_wait();
  allow_dependents();
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
        if (mask && !mask[b * n_kv + h]) { ok[u] = false; continue; }   // this head keeps its rows
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
  grid_dependency_wait();
  allow_dependents();
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

// Gather-and-quantise: one (slot t, head h) row of K and of V per group of
// LPR = D / 8 lanes (16 bytes = 8 bf16 per lane).  Per row: amax = max |x|,
// scale = amax / 127, code = round-half-even(x / scale) clipped to +-127,
// both quotients IEEE float32 divisions (a zero row gets scale 0 and codes 0).
// Codes go to the int8 caches in the NHD layout of the compact cache; scales
// to [n_kv, scale_pitch].
template <int D>
__global__ void __launch_bounds__(kGatherThreads)
gather_q8_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v, int8_t *__restrict__ kq,
                 int8_t *__restrict__ vq, float *__restrict__ ks, float *__restrict__ vs, int64_t scale_pitch,
                 const int32_t *__restrict__ idx, const int *__restrict__ cu_seqlens, const int *__restrict__ cu_budget,
                 int n_kv, int total_budget) {
  grid_dependency_wait();
  allow_dependents();
  constexpr int LPR = D / 8;
  constexpr int RPW = 32 / LPR;                         // rows per warp
  const int b = blockIdx.y;
  const int t0 = cu_seqlens[b], len = cu_seqlens[b + 1] - t0;
  const int cb = cu_budget[b], kept = cu_budget[b + 1] - cb;
  const int lane = lane_id(), sl = lane % LPR, rg = lane / LPR;
  const long long n_rows = (long long)kept * n_kv;
  const long long warps = (long long)gridDim.x * (kGatherThreads / 32);
  for (long long r = ((long long)blockIdx.x * (kGatherThreads / 32) + warp_id()) * RPW + rg; r - rg < n_rows;
       r += warps * RPW) {
    const bool active = r < n_rows;
    const int t = active ? (int)(r / n_kv) : 0, h = active ? (int)(r % n_kv) : 0;
    const int src_t = active ? idx[(size_t)h * total_budget + cb + t] : -1;
    const bool in = src_t >= 0 && src_t < len;
    uint4 rk = make_uint4(0, 0, 0, 0), rv = make_uint4(0, 0, 0, 0);
    if (in) {
      const size_t src = ((size_t)(t0 + src_t) * n_kv + h) * D + (size_t)sl * 8;
      rk = ld_stream16(k + src);
      rv = ld_stream16(v + src);
    }
    float xk[8], xv[8];
    Elem<__nv_bfloat16>::unpack(rk, xk);
    Elem<__nv_bfloat16>::unpack(rv, xv);
    float ak = 0.f, av = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) { ak = fmaxf(ak, fabsf(xk[i])); av = fmaxf(av, fabsf(xv[i])); }
#pragma unroll
    for (int o = 1; o < LPR; o <<= 1) {
      ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, o));
      av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, o));
    }
    const float sk = __fdiv_rn(ak, 127.f), sv = __fdiv_rn(av, 127.f);
    uint32_t ck[2] = {0u, 0u}, cv[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int qk = sk > 0.f ? max(-127, min(127, __float2int_rn(__fdiv_rn(xk[i], sk)))) : 0;
      const int qv = sv > 0.f ? max(-127, min(127, __float2int_rn(__fdiv_rn(xv[i], sv)))) : 0;
      ck[i >> 2] |= (uint32_t)(qk & 0xff) << (8 * (i & 3));
      cv[i >> 2] |= (uint32_t)(qv & 0xff) << (8 * (i & 3));
    }
    if (active) {
      const size_t dst = ((size_t)(cb + t) * n_kv + h) * D + (size_t)sl * 8;
      *reinterpret_cast<uint2 *>(kq + dst) = make_uint2(ck[0], ck[1]);
      *reinterpret_cast<uint2 *>(vq + dst) = make_uint2(cv[0], cv[1]);
      if (sl == 0) {
        ks[(size_t)h * scale_pitch + cb + t] = sk;
        vs[(size_t)h * scale_pitch + cb + t] = sv;
      }
    }
  }
}

}  // namespace

cudaError_t gather_rows_kv_q8(const void *k, const void *v, int8_t *kq, int8_t *vq, float *ks, float *vs,
                              int64_t scale_pitch, const int32_t *idx, const int32_t *cu_seqlens,
                              const int32_t *cu_budget, int n_seqs, int n_kv, int d_h, int total_budget, int max_kept,
                              cudaStream_t st) {
  const long long rows = (long long)max_kept * n_kv;
  const int rpb = (kGatherThreads / 32) * (32 / (d_h / 8));
  long long blocks = (rows + rpb - 1) / rpb;
  if (blocks < 1) blocks = 1;
  if (blocks > 65535) blocks = 65535;
  dim3 grid((unsigned)blocks, n_seqs);
  count_launch();
  const auto *kb = static_cast<const __nv_bfloat16 *>(k);
  const auto *vb = static_cast<const __nv_bfloat16 *>(v);
  if (d_h == 64)
    return launch_pdl(gather_q8_kernel<64>, grid, dim3(kGatherThreads), 0, st, kb, vb, kq, vq, ks, vs, scale_pitch,
                      idx, cu_seqlens, cu_budget, n_kv, total_budget);
  return launch_pdl(gather_q8_kernel<128>, grid, dim3(kGatherThreads), 0, st, kb, vb, kq, vq, ks, vs, scale_pitch, idx,
                    cu_seqlens, cu_budget, n_kv, total_budget);
}

cudaError_t gather_rows_kv(const void *k, const void *v, void *k_out, void *v_out, const int32_t *idx,
                           const int32_t *cu_seqlens, const int32_t *cu_budget, int n_seqs, int n_kv,
                           int row_bytes_per_head, int total_budget, int max_kept, cudaStream_t st,
                           const int32_t *mask) {
  const int vph = row_bytes_per_head / 16;
  const long long items = (long long)max_kept * n_kv * vph;
  long long blocks = (items + kGatherThreads * kGatherUnroll - 1) / (kGatherThreads * kGatherUnroll);
  if (blocks < 1) blocks = 1;
  if (blocks > 65535) blocks = 65535;
  dim3 grid((unsigned)blocks, n_seqs);
  count_launch();
  return launch_pdl(gather_kv_kernel, grid, dim3(kGatherThreads), 0, st, static_cast<const uint8_t *>(k),
                    static_cast<const uint8_t *>(v), static_cast<uint8_t *>(k_out), static_cast<uint8_t *>(v_out), idx,
                    cu_seqlens, cu_budget, n_kv, vph, total_budget, mask);
}

cudaError_t gather_hidden(const void *hidden, void *out, const int32_t *idx, int n_rows, int row_bytes, int n_src,
                          cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const int vpr = row_bytes / 16;
  const long long items = (long long)n_rows * vpr;
  long long blocks = (items + kGatherThreads * kGatherUnroll - 1) / (kGatherThreads * kGatherUnroll);
  if (blocks > 65535) blocks = 65535;
  count_launch();
  return launch_pdl(gather_hidden_kernel, dim3((unsigned)blocks), dim3(kGatherThreads), 0, st,
                    static_cast<const uint8_t *>(hidden), static_cast<uint8_t *>(out), idx, n_rows, vpr, n_src);
}

}  // namespace kvc
