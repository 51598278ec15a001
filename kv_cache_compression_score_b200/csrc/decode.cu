// GQA decode attention over compact caches: out[b, qh] = softmax(scale *
// q[b, qh] . Kc[o_b + t, h]) . Vc[o_b + t, h], h = qh / G.  Decode streams
// the whole retained cache every step, so the kernel is an HBM stream (FastKV
// section 1; "Variantes de l'attention et compression du cache KV",
// introduction).
//
// Persistent CTAs (2 per SM) walk the work items (batch entry, KV head, chunk
// of rows) grid-stride.  Warp 4 is a TMA producer: for every 32-row tile of
// an item it loads the head's K and V rows (NHD layout, 3-D tensor maps, no
// swizzle, no multicast) into a ring of shared-memory stages.  Warps 0-3
// consume: a row of d_h elements is split over LPR = d_h / 16 lanes (16
// elements each, read as 16-byte chunks that are contiguous across a quarter
// warp), the G query heads of h sit in registers pre-scaled to log2 units,
// logits are reduced over the LPR lanes with xor-shuffles and every row group
// keeps an online softmax.  At the end of an item row groups and warps are
// merged; the item's partial (m, l, acc) goes to the workspace, and the last
// item of a (b, h) to finish (atomic ticket, no waiting) merges all partials.
#include <cuda.h>

#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kConsumers = 4;                       // consumer warps
constexpr int kThreadsDec = (kConsumers + 1) * 32;  // + one producer warp
constexpr int kRS = 32;                             // rows per tile

template <typename T, int D>
struct DecLayout {
  static constexpr int kEsz = sizeof(T);
  static constexpr int kTile = kRS * D * kEsz;                    // K or V tile bytes
  static constexpr int kStages = (96 * 1024) / (2 * kTile) < 6 ? (96 * 1024) / (2 * kTile) : 6;
  static constexpr int kOffBar = kStages * 2 * kTile;
  static constexpr int kOffMl = kOffBar + 2 * 8 * 8;              // up to 8 stages x 2 barriers
  static constexpr int kBytesTiles = kOffMl;
};

struct DecParams {
  const void *q;
  const int64_t *row_off;
  const int *kv_len;
  float *out;
  float *part;
  int *tickets;
  int *err;
  int batch, n_h, n_kv, n_chunks, chunk_rows;
  float c;   // scale * log2(e)
};

KVC_DEVINL void merge_scale(float m, float m2, float &s1, float &s2, float &mn) {
  mn = fmaxf(m, m2);
  if (mn == kNegInf) { s1 = 0.f; s2 = 0.f; return; }
  s1 = fast_exp2(m - mn);
  s2 = fast_exp2(m2 - mn);
}

template <typename T> KVC_DEVINL void unpack16(const uint4 &v, float *o);
template <> KVC_DEVINL void unpack16<__nv_bfloat16>(const uint4 &v, float *o) { Elem<__nv_bfloat16>::unpack(v, o); }
template <> KVC_DEVINL void unpack16<float>(const uint4 &v, float *o) { Elem<float>::unpack(v, o); }

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreadsDec)
gqa_decode_tma(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv, DecParams p) {
  using L = DecLayout<T, D>;
  constexpr int LPR = D / 16;                 // lanes per row
  constexpr int RPW = 32 / LPR;               // rows per warp step
  constexpr int kSteps = kRS / (kConsumers * RPW);
  constexpr int EPC = 16 / L::kEsz;           // elements per 16-byte chunk
  constexpr int NCH = 16 / EPC;               // chunks per lane (16 elements)
  static_assert(kSteps >= 1 && kRS % (kConsumers * RPW) == 0, "tile rows");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *empty = full + 8;
  float *sm_ml = reinterpret_cast<float *>(smem + L::kOffMl);            // [warps][G][2]
  float *sm_acc = sm_ml + kConsumers * G * 2;                            // [warps][G][D]
  int *sm_flag = reinterpret_cast<int *>(sm_acc + kConsumers * G * D);   // [0] last, [1] error

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kConsumers); }
    sm_flag[1] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  __syncthreads();

  const int n_items = p.batch * p.n_kv * p.n_chunks;
  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int t = 0;
      volatile int *vflag = sm_flag;
      for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
        const int c = it % p.n_chunks, bh = it / p.n_chunks, h = bh % p.n_kv, b = bh / p.n_kv;
        const int len = p.kv_len[b], r0 = c * p.chunk_rows;
        if (r0 >= len) continue;
        const int r1 = min(len, r0 + p.chunk_rows);
        const int64_t o = p.row_off[b];
        for (int row = r0; row < r1; row += kRS, ++t) {
          const int s = t % L::kStages;
          if (!vflag[1] && !mbar_wait(&empty[s], ((t / L::kStages) & 1) ^ 1)) vflag[1] = 1;
          mbar_expect_tx(&full[s], 2 * L::kTile);
          uint8_t *ks = smem + s * 2 * L::kTile;
          tma_load_3d(ks, &tmk, &full[s], 0, h, (int)(o + row));
          tma_load_3d(ks + L::kTile, &tmv, &full[s], 0, h, (int)(o + row));
        }
      }
      for (int u = max(0, t - L::kStages); u < t; ++u)      // drain copies in flight
        if (!mbar_wait(&full[u % L::kStages], (u / L::kStages) & 1)) { vflag[1] = 1; break; }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int rg = lane / LPR, sl = lane % LPR;
    volatile int *vflag = sm_flag;
    int t = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      const int c = it % p.n_chunks, bh = it / p.n_chunks, h = bh % p.n_kv, b = bh / p.n_kv;
      const int len = p.kv_len[b], r0 = c * p.chunk_rows;
      const int n_active = (len + p.chunk_rows - 1) / p.chunk_rows;
      float *outp = p.out + ((size_t)b * p.n_h + (size_t)h * G) * D;
      if (len == 0) {
        if (c == 0)
          for (int e = threadIdx.x; e < G * D; e += kConsumers * 32) outp[e] = 0.f;
        continue;
      }
      if (r0 >= len) continue;
      const int r1 = min(len, r0 + p.chunk_rows);

      // query slices: element d = j * (LPR * EPC) + sl * EPC + i of chunk j
      float qr[G][16];
      const T *qb = static_cast<const T *>(p.q) + ((size_t)b * p.n_h + (size_t)h * G) * D;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          unpack16<T>(ld_nc16(qb + (size_t)g * D + j * (LPR * EPC) + sl * EPC), &qr[g][j * EPC]);
#pragma unroll
          for (int i = 0; i < EPC; ++i) qr[g][j * EPC + i] *= p.c;
        }
      float acc[G][16], m[G], l[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = kNegInf;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[g][e] = 0.f;
      }

      for (int row = r0; row < r1; row += kRS, ++t) {
        const int s = t % L::kStages;
        // after a give-up anywhere in the CTA nobody waits again: the loops
        // still run to their end (results flagged invalid), so every warp
        // reaches the named barriers below
        const bool got = vflag[1] ? true : mbar_wait(&full[s], (t / L::kStages) & 1);
        if (!__all_sync(0xffffffffu, got) && lane == 0) vflag[1] = 1;
        const uint8_t *ks = smem + s * 2 * L::kTile;
        const uint8_t *vs = ks + L::kTile;
#pragma unroll
        for (int st = 0; st < kSteps; ++st) {
          const int lr = st * (kConsumers * RPW) + warp * RPW + rg;
          const bool valid = row + lr < r1;
          float kf[16];
          const uint8_t *krow = ks + lr * D * L::kEsz + sl * 16;
#pragma unroll
          for (int j = 0; j < NCH; ++j) unpack16<T>(*reinterpret_cast<const uint4 *>(krow + j * LPR * 16), &kf[j * EPC]);
          float sc[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              a0 = fmaf(qr[g][e], kf[e], a0);
              a1 = fmaf(qr[g][e + 1], kf[e + 1], a1);
            }
            sc[g] = a0 + a1;
          }
#pragma unroll
          for (int off = 1; off < LPR; off <<= 1)
#pragma unroll
            for (int g = 0; g < G; ++g) sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], off);
          if (valid) {
            float vf[16];
            const uint8_t *vrow = vs + lr * D * L::kEsz + sl * 16;
#pragma unroll
            for (int j = 0; j < NCH; ++j)
              unpack16<T>(*reinterpret_cast<const uint4 *>(vrow + j * LPR * 16), &vf[j * EPC]);
#pragma unroll
            for (int g = 0; g < G; ++g) {
              if (sc[g] > m[g]) {
                const float a = fast_exp2(m[g] - sc[g]);
                l[g] *= a;
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[g][e] *= a;
                m[g] = sc[g];
              }
              const float pr = fast_exp2(sc[g] - m[g]);
              l[g] += pr;
#pragma unroll
              for (int e = 0; e < 16; ++e) acc[g][e] = fmaf(pr, vf[e], acc[g][e]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // merge the row groups of the warp (lanes holding the same slice)
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1)
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
      // merge the consumer warps through shared memory
      if (rg == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (sl == 0) { sm_ml[(warp * G + g) * 2] = m[g]; sm_ml[(warp * G + g) * 2 + 1] = l[g]; }
#pragma unroll
          for (int j = 0; j < NCH; ++j)
#pragma unroll
            for (int i = 0; i < EPC; ++i)
              sm_acc[(warp * G + g) * D + j * (LPR * EPC) + sl * EPC + i] = acc[g][j * EPC + i];
        }
      }
      asm volatile("bar.sync 1, %0;" :: "n"(kConsumers * 32) : "memory");
      float *my_part = p.part + ((size_t)bh * p.n_chunks + c) * (size_t)(G * (D + 2));
      for (int e = threadIdx.x; e < G * D; e += kConsumers * 32) {
        const int g = e / D, d = e % D;
        float M = kNegInf;
#pragma unroll
        for (int wv = 0; wv < kConsumers; ++wv) M = fmaxf(M, sm_ml[(wv * G + g) * 2]);
        float Ls = 0.f, A = 0.f;
#pragma unroll
        for (int wv = 0; wv < kConsumers; ++wv) {
          const float mw = sm_ml[(wv * G + g) * 2];
          if (mw == kNegInf) continue;
          const float sc = fast_exp2(mw - M);
          Ls = fmaf(sm_ml[(wv * G + g) * 2 + 1], sc, Ls);
          A = fmaf(sm_acc[(wv * G + g) * D + d], sc, A);
        }
        if (n_active == 1) {
          outp[e] = A / Ls;
        } else {
          my_part[g * (D + 2) + 2 + d] = A;
          if (d == 0) { my_part[g * (D + 2)] = M; my_part[g * (D + 2) + 1] = Ls; }
        }
      }
      if (n_active > 1) {
        __threadfence();
        asm volatile("bar.sync 1, %0;" :: "n"(kConsumers * 32) : "memory");
        if (threadIdx.x == 0) sm_flag[0] = (atomicAdd(&p.tickets[bh], 1) == n_active - 1);
        asm volatile("bar.sync 1, %0;" :: "n"(kConsumers * 32) : "memory");
        if (sm_flag[0]) {
          __threadfence();
          const float *pp = p.part + (size_t)bh * p.n_chunks * (size_t)(G * (D + 2));
          for (int e = threadIdx.x; e < G * D; e += kConsumers * 32) {
            const int g = e / D, d = e % D;
            float M = kNegInf;
            for (int cc = 0; cc < n_active; ++cc) M = fmaxf(M, __ldcg(pp + (size_t)cc * G * (D + 2) + g * (D + 2)));
            float Ls = 0.f, A = 0.f;
            for (int cc = 0; cc < n_active; ++cc) {
              const float *q0 = pp + (size_t)cc * G * (D + 2) + g * (D + 2);
              const float sc = fast_exp2(__ldcg(q0) - M);
              Ls = fmaf(__ldcg(q0 + 1), sc, Ls);
              A = fmaf(__ldcg(q0 + 2 + d), sc, A);
            }
            outp[e] = A / Ls;
          }
          if (threadIdx.x == 0) p.tickets[bh] = 0;   // leave the counter zeroed for the next call
        }
      }
      asm volatile("bar.sync 1, %0;" :: "n"(kConsumers * 32) : "memory");   // smem reuse by the next item
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && sm_flag[1]) atomicCAS(p.err, 0, 2);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                     const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                     CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                     CUtensorMapFloatOOBfill);

PFN_encodeTiled encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(ptr);
  }
  return fn;
}

// cache [rows, n_kv, D] -> boxes of D elements x 1 head x kRS rows (rows past
// the cache read as zero)
bool cache_map(CUtensorMap *m, const void *base, int64_t rows, int n_kv, int D, bool bf16) {
  PFN_encodeTiled enc = encode_fn();
  if (!enc) return false;
  const int esz = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)n_kv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * esz, (cuuint64_t)n_kv * D * esz};
  cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)kRS};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, int G>
cudaError_t launch(const DecodeArgs &a, cudaStream_t st) {
  using L = DecLayout<T, D>;
  CUtensorMap mk, mv;
  const bool bf = a.dt == KVC_BF16;
  if (!cache_map(&mk, a.k_c, a.cache_rows, a.n_kv, D, bf) || !cache_map(&mv, a.v_c, a.cache_rows, a.n_kv, D, bf))
    return cudaErrorInvalidValue;
  DecParams p;
  p.q = a.q; p.row_off = a.row_off; p.kv_len = a.kv_len; p.out = a.out; p.part = a.part; p.tickets = a.tickets;
  p.err = a.err; p.batch = a.batch; p.n_h = a.n_h; p.n_kv = a.n_kv; p.n_chunks = a.n_chunks;
  p.chunk_rows = a.chunk_rows; p.c = a.scale * kLog2e;
  const int smem = 1024 + L::kBytesTiles + (kConsumers * G * 2 + kConsumers * G * D + 4) * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(gqa_decode_tma<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int items = a.batch * a.n_kv * a.n_chunks;
  const int grid = items < 2 * kNumSMs ? items : 2 * kNumSMs;
  gqa_decode_tma<T, D, G><<<grid, kThreadsDec, smem, st>>>(mk, mv, p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t by_group(const DecodeArgs &a, cudaStream_t st) {
  switch (a.n_h / a.n_kv) {
    case 1: return launch<T, D, 1>(a, st);
    case 2: return launch<T, D, 2>(a, st);
    case 4: return launch<T, D, 4>(a, st);
    default: return launch<T, D, 8>(a, st);
  }
}

}  // namespace

int decode_tile_rows() { return kRS; }

cudaError_t gqa_decode(const DecodeArgs &a, cudaStream_t st) {
  if (a.dt == KVC_F32) return a.d_h == 64 ? by_group<float, 64>(a, st) : by_group<float, 128>(a, st);
  return a.d_h == 64 ? by_group<__nv_bfloat16, 64>(a, st) : by_group<__nv_bfloat16, 128>(a, st);
}

}  // namespace kvc
