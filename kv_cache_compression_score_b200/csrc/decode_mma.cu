// GQA decode attention over compact caches on the tensor cores, fed by TMA:
//   out[b, qh] = softmax_t(scale * q[b, qh] . Kc[o_b + t, h]) . Vc[o_b + t, h],
//   h = qh / G.
// Decode streams the whole retained cache every step (FastKV section 1;
// "Variantes de l'attention et compression du cache KV", introduction), so the
// kernel is built to keep HBM busy with as few instructions per cache byte as
// possible:
//
//  * Work split (stream-K): the rows of all (batch entry, KV head) units are
//    laid end to end and every CTA (one per SM) takes an equal contiguous
//    slice, cut into tiles of up to 64 rows of one unit.
//  * Warp 4 is the producer: per tile one thread issues 2-D tensor-map copies
//    (cp.async.bulk.tensor, no multicast) of the head's K and V rows into a
//    ring of shared-memory stages (128-byte swizzle), completion counted in
//    bytes on the stage's mbarrier.  Rows past the cache read as zero.
//  * Warps 0-3 consume 16 rows of every tile each, with mma.sync m16n8k16
//    (bf16 in, fp32 accumulate) in the transposed orientation, so the G <= 8
//    query heads of a KV head fill the N = 8 side and no M rows are wasted:
//        S^T[key][head] = K[key][:] . Q[head][:]          (A = K via ldmatrix)
//        O^T[dim][head] += V^T[dim][key] . P^T[key][head] (A = V via ldmatrix.trans)
//    The S^T accumulator turns into the P^T operand with one movmatrix per
//    8x8 block.  P is split into two bf16 terms (p = hi + lo, |lo| <= 2^-9 p)
//    so the product keeps ~16 bits of every weight; the sum l of the weights
//    is accumulated from the fp32 values.
//  * Online softmax in log2 units: the reference max of a head moves only when
//    a tile's logit exceeds it by more than kSlack (every weight <= 2^kSlack),
//    so rescaling is rare; it is uniform over the lanes of a head.
//  * At the end of a unit segment the four warps merge through shared memory;
//    a unit split over several CTAs leaves (m, l, acc) partials and the last
//    CTA to finish it (atomic ticket, no waiting) merges them.
//
// The int8 variant reads caches quantised per (row, head) with a float32
// scale (K_c = s_k * q_k, V_c = s_v * q_v): int8 tiles are widened exactly to
// bf16 in a per-warp staging area, the K scale multiplies the logits of its
// row and the V scale the weight of its row, so the products are those of the
// dequantised cache.
//
// Every wait is bounded: a wait that gives up sets the workspace error word;
// the producer still waits (bounded) for its copies in flight before exiting.
#include <cuda.h>

#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kCons = 4;                  // consumer warps
constexpr int kThr = (kCons + 1) * 32;    // + one producer warp
constexpr int kTR = 64;                   // cache rows per tile (16 per consumer warp)
constexpr int kRingBytes = 192 * 1024;
constexpr float kSlackM = 8.f;

template <int D, bool Q8>
struct MmaLayout {
  static constexpr int kEsz = Q8 ? 1 : 2;
  static constexpr int kRowB = D * kEsz;                        // one head row of K (or V)
  static constexpr int kBoxB = kRowB < 128 ? kRowB : 128;       // TMA box inner bytes = swizzle span
  static constexpr int kBoxes = kRowB / kBoxB;                  // boxes per tile per tensor
  static constexpr int kBoxBytes = kTR * kBoxB;
  static constexpr int kTileB = kTR * kRowB;                    // K (or V) bytes of one tile
  static constexpr int kStageB = 2 * kTileB;                    // K and V tiles of one stage
  static constexpr int kStagesRaw = (Q8 ? kRingBytes * 2 / 3 : kRingBytes) / kStageB;
  static constexpr int kStages = kStagesRaw > 16 ? 16 : kStagesRaw;
  // int8: per stage the K and V scales of the tile's rows (2 x kTR floats)
  static constexpr int kOffScale = kStages * kStageB;
  static constexpr int kOffBar = kOffScale + (Q8 ? kStages * 2 * kTR * 4 : 0);   // full[16], empty[16]
  static constexpr int kOffMerge = kOffBar + 2 * 16 * 8;
  // merge area: per consumer warp, 8 heads x (m, l) + 8 heads x D accumulators
  static constexpr int kMergeFloats = kCons * 8 * 2 + kCons * 8 * D;
  static constexpr int kOffFlag = kOffMerge + kMergeFloats * 4;
  static constexpr int kOffStg = (kOffFlag + 16 + 1023) / 1024 * 1024;
  // Q8 staging: per consumer warp 16 rows of K and of V widened to bf16
  static constexpr int kStgWarp = Q8 ? 2 * 16 * 2 * D : 0;
  static constexpr int kBytes = kOffStg + kCons * kStgWarp;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kStageB % 1024 == 0, "swizzled boxes need 1 KB alignment");
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

struct MmaParams {
  const __nv_bfloat16 *q;
  const int64_t *row_off;
  const int *kv_len;
  const float *k_scale, *v_scale;   // int8 caches: [n_kv, scale_pitch]
  int64_t scale_pitch;
  float *out;
  float *part;
  int *tickets;
  int *err;
  int batch, n_h, n_kv, slots;
  int64_t cache_rows;
  float c;                          // scale * log2(e)
};

// ------------------------------------------------------------ PTX wrappers
KVC_DEVINL void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
KVC_DEVINL void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      :: "r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y) : "memory");
}
KVC_DEVINL void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(map) : "memory");
}
KVC_DEVINL void cp_async4(void *dst, const void *src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;"
               :: "r"(smem_u32(dst)), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
KVC_DEVINL void cp_async_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}
KVC_DEVINL void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
KVC_DEVINL void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
KVC_DEVINL void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
               "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
KVC_DEVINL uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// (lo, hi) -> bf16x2 with lo in the low half, round to nearest even
KVC_DEVINL uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// byte offset of 16-byte chunk `ch` of row `r` inside a tile whose rows are
// cut into boxes of BoxB bytes (BoxB-byte swizzle: the chunk index is XORed
// with address bits 7.. of the row start)
template <int BoxB, int Rows>
KVC_DEVINL uint32_t swz(int r, int ch) {
  constexpr int kCh = BoxB / 16;                    // chunks per box row
  const int box = ch / kCh, c = ch % kCh;
  const int x = BoxB == 128 ? (r & 7) : ((r >> 1) & 3);
  return (uint32_t)(box * Rows * BoxB + r * BoxB + ((c ^ x) << 4));
}

template <int D, bool Q8, int G>
__global__ void __launch_bounds__(kThr, 1)
gqa_decode_mma(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv, MmaParams p) {
  using L = MmaLayout<D, Q8>;
  constexpr int NKS = D / 16;        // k-steps of the logit product = m-tiles of the value product
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *empty = full + 16;
  float *mrg = reinterpret_cast<float *>(smem + L::kOffMerge);
  float *mrg_ml = mrg;                                   // [warp][8][2]
  float *mrg_acc = mrg + kCons * 16;                     // [warp][8][D]
  volatile int *flag = reinterpret_cast<volatile int *>(smem + L::kOffFlag);   // [0] error, [1] last
  const int warp = warp_id(), lane = lane_id();

  grid_dependency_wait();
  // ---- the flattened row space and this CTA's slice
  int64_t R = 0;
  for (int b = 0; b < p.batch; ++b) R += (int64_t)p.kv_len[b] * p.n_kv;
  const int64_t NC = R > 0 ? min((int64_t)gridDim.x, max((int64_t)1, R / kTR)) : 0;
  const int cta = blockIdx.x;
  // units of empty caches produce zeros (CTA 0)
  if (cta == 0 && warp == 0)
    for (int u = 0; u < p.batch * p.n_kv; ++u)
      if (p.kv_len[u / p.n_kv] == 0)
        for (int e = lane; e < G * D; e += 32)
          p.out[((size_t)(u / p.n_kv) * p.n_h + (size_t)(u % p.n_kv) * G) * D + e] = 0.f;
  if (cta >= NC) return;
  const int64_t x_begin = cta * R / NC, x_end = (cta + 1) * R / NC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], Q8 ? 1 + 32 : 1);
      mbar_init(&empty[s], kCons);
    }
    flag[0] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  __syncthreads();

  // Tile walker shared by the producer and the consumers: from row x of the
  // flattened space, the unit (b, h), its first row u0 and length len, and
  // the tile's first unit-local row r0 and row count n.
  struct Walk {
    int b, h, len;
    int64_t base_b, x;
  };
  Walk wk;
  wk.x = x_begin;
  wk.b = 0;
  wk.base_b = 0;
  while (wk.base_b + (int64_t)p.kv_len[wk.b] * p.n_kv <= wk.x) { wk.base_b += (int64_t)p.kv_len[wk.b] * p.n_kv; ++wk.b; }
  wk.len = p.kv_len[wk.b];
  wk.h = (int)((wk.x - wk.base_b) / wk.len);
  auto advance = [&](int n) {                 // move past n rows of the current unit
    wk.x += n;
    const int64_t u_end = wk.base_b + (int64_t)(wk.h + 1) * wk.len;
    if (wk.x == u_end && wk.x < x_end) {
      if (wk.h + 1 < p.n_kv) {
        ++wk.h;
      } else {
        wk.base_b += (int64_t)wk.len * p.n_kv;
        ++wk.b;
        while (p.kv_len[wk.b] == 0) ++wk.b;   // wk.x < x_end <= R: a non-empty entry follows
        wk.len = p.kv_len[wk.b];
        wk.h = 0;
      }
    }
  };
  auto tile_rows = [&]() -> int {
    const int64_t u_end = wk.base_b + (int64_t)(wk.h + 1) * wk.len;
    return (int)min((int64_t)kTR, min(u_end, x_end) - wk.x);
  };
  auto unit_row = [&]() -> int { return (int)(wk.x - wk.base_b - (int64_t)wk.h * wk.len); };

  if (warp == kCons) {
    // ============================================================ producer
    int j = 0;
    while (wk.x < x_end) {
      const int n = tile_rows();
      const int s = j % L::kStages;
      if (j >= L::kStages && !flag[0] && !mbar_wait(&empty[s], ((j / L::kStages) - 1) & 1)) flag[0] = 1;
      if (flag[0]) break;
      const int64_t row0 = p.row_off[wk.b] + unit_row();
      uint8_t *st = smem + s * L::kStageB;
      if (lane == 0) {
        mbar_expect_tx(&full[s], 2 * L::kTileB);
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          const int xe = wk.h * D + bx * (L::kBoxB / L::kEsz);
          tma_load_2d(st + bx * L::kBoxBytes, &tmk, &full[s], xe, (int)row0);
          tma_load_2d(st + L::kTileB + bx * L::kBoxBytes, &tmv, &full[s], xe, (int)row0);
        }
      }
      if constexpr (Q8) {
        // per-row scales of the tile: 4-byte copies (the rows need not be
        // 16-byte aligned), completion counted on the same barrier
        float *sk = reinterpret_cast<float *>(smem + L::kOffScale) + s * 2 * kTR;
        const float *gk = p.k_scale + (size_t)wk.h * p.scale_pitch;
        const float *gv = p.v_scale + (size_t)wk.h * p.scale_pitch;
        for (int r = lane; r < kTR; r += 32) {
          const bool ok = r < n;
          cp_async4(sk + r, gk + (ok ? row0 + r : 0), ok);
          cp_async4(sk + kTR + r, gv + (ok ? row0 + r : 0), ok);
        }
        cp_async_arrive_noinc(&full[s]);
      }
      __syncwarp();
      advance(n);
      ++j;
    }
    // copies still in flight land before the CTA may exit
    for (int u = max(0, j - L::kStages); u < j; ++u)
      if (!mbar_wait(&full[u % L::kStages], (u / L::kStages) & 1)) { flag[0] = 1; break; }
    if constexpr (Q8) asm volatile("cp.async.wait_all;" ::: "memory");
  } else {
    // ============================================================ consumers
    const int g = lane >> 2, t = lane & 3;                 // mma fragment coordinates
    const int lr = lane & 7, li = lane >> 3;               // ldmatrix row / matrix of this lane
    uint8_t *stg = smem + L::kOffStg + warp * L::kStgWarp;
    // query fragments (B operand of the logit product): head g, dims 16ks + 2t (+8)
    uint32_t qf[NKS][2];
    float m[2], l[2], acc[NKS][4];
    int cur_b = -1, cur_h = -1;
    int64_t seg_u0 = 0;          // first flattened row of the current unit
    int j = 0;

    auto reset_unit = [&]() {
      const __nv_bfloat16 *qb = p.q + ((size_t)wk.b * p.n_h + (size_t)wk.h * G + g) * D;
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks) {
        if (g < G) {
          qf[ks][0] = __ldg(reinterpret_cast<const uint32_t *>(qb + 16 * ks + 2 * t));
          qf[ks][1] = __ldg(reinterpret_cast<const uint32_t *>(qb + 16 * ks + 8 + 2 * t));
        } else {
          qf[ks][0] = qf[ks][1] = 0u;
        }
      }
      m[0] = m[1] = kNegInf;
      l[0] = l[1] = 0.f;
#pragma unroll
      for (int i = 0; i < NKS; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
      cur_b = wk.b;
      cur_h = wk.h;
      seg_u0 = wk.base_b + (int64_t)wk.h * wk.len;
    };

    // end of a unit segment: merge the warps, then write the output or a partial
    auto finish_unit = [&](int64_t seg_x_end) {
      // heads 2t, 2t+1: l summed over the rows g of the warp
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l[0] += __shfl_xor_sync(0xffffffffu, l[0], o);
        l[1] += __shfl_xor_sync(0xffffffffu, l[1], o);
      }
      if (g == 0) {
        mrg_ml[(warp * 8 + 2 * t) * 2] = m[0];
        mrg_ml[(warp * 8 + 2 * t) * 2 + 1] = l[0];
        mrg_ml[(warp * 8 + 2 * t + 1) * 2] = m[1];
        mrg_ml[(warp * 8 + 2 * t + 1) * 2 + 1] = l[1];
      }
      float *aw = mrg_acc + warp * 8 * D;
#pragma unroll
      for (int i = 0; i < NKS; ++i) {
        aw[(2 * t) * D + 16 * i + g] = acc[i][0];
        aw[(2 * t + 1) * D + 16 * i + g] = acc[i][1];
        aw[(2 * t) * D + 16 * i + g + 8] = acc[i][2];
        aw[(2 * t + 1) * D + 16 * i + g + 8] = acc[i][3];
      }
      asm volatile("bar.sync 1, %0;" :: "n"(kCons * 32) : "memory");
      const int u = cur_b * p.n_kv + cur_h;
      const int len = p.kv_len[cur_b];
      // which CTAs share this unit
      auto owner = [&](int64_t xx) {
        int64_t c = xx * NC / R;
        while (c + 1 < NC && (c + 1) * R / NC <= xx) ++c;
        while (c > 0 && c * R / NC > xx) --c;
        return c;
      };
      const int64_t first = owner(seg_u0), last = owner(seg_u0 + len - 1);
      const int ct = threadIdx.x;                        // 0 .. 127
      float *outp = p.out + ((size_t)cur_b * p.n_h + (size_t)cur_h * G) * D;
      constexpr int REC = D + 4;
      float *pp = p.part + ((size_t)u * p.slots + (size_t)(cta - first)) * (size_t)(G * REC);
      for (int e = ct; e < G * D; e += kCons * 32) {
        const int hd = e / D, d = e % D;
        float M = kNegInf;
#pragma unroll
        for (int w2 = 0; w2 < kCons; ++w2) M = fmaxf(M, mrg_ml[(w2 * 8 + hd) * 2]);
        float Ls = 0.f, A = 0.f;
        if (M != kNegInf) {
#pragma unroll
          for (int w2 = 0; w2 < kCons; ++w2) {
            const float mw = mrg_ml[(w2 * 8 + hd) * 2];
            const float sc = mw == kNegInf ? 0.f : fast_exp2(mw - M);
            Ls += mrg_ml[(w2 * 8 + hd) * 2 + 1] * sc;
            A += mrg_acc[(w2 * 8 + hd) * D + d] * sc;
          }
        }
        if (first == last) {
          outp[hd * D + d] = A / Ls;
        } else {
          pp[hd * REC + 4 + d] = A;
          if (d == 0) { pp[hd * REC] = M; pp[hd * REC + 1] = Ls; }
        }
      }
      if (first != last) {
        __threadfence();
        asm volatile("bar.sync 1, %0;" :: "n"(kCons * 32) : "memory");
        if (ct == 0) flag[1] = (atomicAdd(&p.tickets[u], 1) == (int)(last - first)) ? 1 : 0;
        asm volatile("bar.sync 1, %0;" :: "n"(kCons * 32) : "memory");
        if (flag[1]) {
          __threadfence();
          const int n_seg = (int)(last - first + 1);
          const float *pu = p.part + (size_t)u * p.slots * (size_t)(G * REC);
          for (int e = ct; e < G * D; e += kCons * 32) {
            const int hd = e / D, d = e % D;
            float M = kNegInf;
            for (int sgi = 0; sgi < n_seg; ++sgi) M = fmaxf(M, __ldcg(pu + ((size_t)sgi * G + hd) * REC));
            float Ls = 0.f, A = 0.f;
            for (int sgi = 0; sgi < n_seg; ++sgi) {
              const float *rec = pu + ((size_t)sgi * G + hd) * REC;
              const float mj = __ldcg(rec);
              const float sc = (mj == kNegInf) ? 0.f : fast_exp2(mj - M);
              Ls += __ldcg(rec + 1) * sc;
              A += __ldcg(rec + 4 + d) * sc;
            }
            outp[hd * D + d] = A / Ls;
          }
          if (ct == 0) p.tickets[u] = 0;       // leave the counter zeroed for the next call
        }
      }
      asm volatile("bar.sync 1, %0;" :: "n"(kCons * 32) : "memory");
      (void)seg_x_end;
    };

    while (wk.x < x_end) {
      const int n = tile_rows();
      if (wk.b != cur_b || wk.h != cur_h) reset_unit();
      const int s = j % L::kStages;
      // After a wait gave up the warps keep walking the tiles (so that all of
      // them meet at the same named barriers) but skip the work.
      bool ok = flag[0] == 0;
      if (ok) {
        const bool got = mbar_wait(&full[s], (j / L::kStages) & 1);
        if (!__all_sync(0xffffffffu, got)) { if (lane == 0) flag[0] = 1; ok = false; }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        const uint8_t *stg_k = smem + s * L::kStageB;
        const uint8_t *stg_v = stg_k + L::kTileB;
        const int rw0 = warp * 16;                 // this warp's rows in the tile
        const bool v0 = rw0 + g < n, v1 = rw0 + g + 8 < n;   // rows g and g + 8 valid

        // ---- operands of this warp's 16 rows: bf16 K / V tiles (swizzled)
        uint32_t k_base, v_base;
        int rows_in;                               // rows of the area ldmatrix reads
        float ksc0 = 1.f, ksc1 = 1.f, vsc0 = 1.f, vsc1 = 1.f;
        if constexpr (Q8) {
          // widen this warp's 16 int8 rows of K and V to bf16 in its staging area
          const float *scl = reinterpret_cast<const float *>(smem + L::kOffScale) + s * 2 * kTR;
          ksc0 = scl[rw0 + g]; ksc1 = scl[rw0 + g + 8];
          vsc0 = scl[kTR + rw0 + g]; vsc1 = scl[kTR + rw0 + g + 8];
          constexpr int kChIn = D / 16;            // 16-byte int8 chunks per row
          for (int e = lane; e < 2 * 16 * kChIn; e += 32) {
            const int tsr = e / (16 * kChIn), rem = e % (16 * kChIn), r = rem / kChIn, ch = rem % kChIn;
            const uint8_t *src = (tsr ? stg_v : stg_k) + swz<L::kBoxB, kTR>(rw0 + r, ch);
            const uint4 raw = *reinterpret_cast<const uint4 *>(src);
            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t o[8];
  #pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const uint32_t x = wv[q4];
              o[2 * q4] = pack_bf16((float)(int8_t)(x & 0xff), (float)(int8_t)((x >> 8) & 0xff));
              o[2 * q4 + 1] = pack_bf16((float)(int8_t)((x >> 16) & 0xff), (float)(int8_t)(x >> 24));
            }
            // 16 int8 -> 32 bytes of bf16 = bf16 chunks 2ch, 2ch+1 of the row
            uint8_t *dst = stg + tsr * (16 * 2 * D);
            *reinterpret_cast<uint4 *>(dst + swz<128, 16>(r, 2 * ch)) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4 *>(dst + swz<128, 16>(r, 2 * ch + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
          }
          __syncwarp();
          k_base = smem_u32(stg);
          v_base = smem_u32(stg + 16 * 2 * D);
          rows_in = 16;
        } else {
          if (rw0 + 16 > n) {
            // rows past the segment: zero their V so that 0-weights meet finite values
            for (int e = lane; e < 16 * (D / 8); e += 32) {
              const int r = e / (D / 8), ch = e % (D / 8);
              if (rw0 + r >= n)
                *reinterpret_cast<uint4 *>(const_cast<uint8_t *>(stg_v) + swz<128, kTR>(rw0 + r, ch)) =
                    make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
          }
          k_base = smem_u32(stg_k);
          v_base = smem_u32(stg_v);
          rows_in = kTR;
        }
        const int r_off = Q8 ? 0 : rw0;            // first row of this warp inside the ldmatrix area
        auto frag_addr = [&](uint32_t base, int r, int ch) -> uint32_t {
          return base + (rows_in == 16 ? swz<128, 16>(r, ch) : swz<128, kTR>(r, ch));
        };

        // ---- S^T = K . Q^T for the warp's 16 rows
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
  #pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
          uint32_t a[4];
          // matrices: (rows 0-7, dims 0-7), (rows 8-15, dims 0-7), (rows 0-7, dims 8-15), (rows 8-15, dims 8-15)
          ldsm_x4(frag_addr(k_base, r_off + lr + (li & 1) * 8, 2 * ks + (li >> 1)), a);
          mma_bf16(sc, a, qf[ks][0], qf[ks][1]);
        }
        // logits in log2 units: (row g, heads 2t, 2t+1), (row g+8, same heads)
        float z[4];
        z[0] = v0 ? sc[0] * p.c * ksc0 : kNegInf;
        z[1] = v0 ? sc[1] * p.c * ksc0 : kNegInf;
        z[2] = v1 ? sc[2] * p.c * ksc1 : kNegInf;
        z[3] = v1 ? sc[3] * p.c * ksc1 : kNegInf;
        float tmax0 = fmaxf(z[0], z[2]), tmax1 = fmaxf(z[1], z[3]);
  #pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          tmax0 = fmaxf(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, o));
          tmax1 = fmaxf(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, o));
        }
        const bool need0 = tmax0 > m[0] + kSlackM, need1 = tmax1 > m[1] + kSlackM;
        if (__any_sync(0xffffffffu, need0 || need1)) {
          const float mn0 = need0 ? tmax0 : m[0], mn1 = need1 ? tmax1 : m[1];
          const float a0 = (m[0] == kNegInf) ? 0.f : fast_exp2(m[0] - mn0);
          const float a1 = (m[1] == kNegInf) ? 0.f : fast_exp2(m[1] - mn1);
          l[0] *= a0;
          l[1] *= a1;
  #pragma unroll
          for (int i = 0; i < NKS; ++i) { acc[i][0] *= a0; acc[i][2] *= a0; acc[i][1] *= a1; acc[i][3] *= a1; }
          m[0] = mn0;
          m[1] = mn1;
        }
        const float ms0 = m[0] == kNegInf ? 0.f : m[0], ms1 = m[1] == kNegInf ? 0.f : m[1];
        float pw[4];
        pw[0] = v0 ? fast_exp2(z[0] - ms0) : 0.f;
        pw[1] = v0 ? fast_exp2(z[1] - ms1) : 0.f;
        pw[2] = v1 ? fast_exp2(z[2] - ms0) : 0.f;
        pw[3] = v1 ? fast_exp2(z[3] - ms1) : 0.f;
        l[0] += pw[0] + pw[2];
        l[1] += pw[1] + pw[3];
        if constexpr (Q8) { pw[0] *= vsc0; pw[1] *= vsc0; pw[2] *= vsc1; pw[3] *= vsc1; }
        // P^T operand: two bf16 terms per weight, transposed per 8x8 block
        const uint32_t h01 = pack_bf16(pw[0], pw[1]), h23 = pack_bf16(pw[2], pw[3]);
        const uint32_t l01 = pack_bf16(pw[0] - __uint_as_float(h01 << 16), pw[1] - __uint_as_float(h01 & 0xffff0000u));
        const uint32_t l23 = pack_bf16(pw[2] - __uint_as_float(h23 << 16), pw[3] - __uint_as_float(h23 & 0xffff0000u));
        const uint32_t bh0 = movmatrix_t(h01), bh1 = movmatrix_t(h23);
        const uint32_t bl0 = movmatrix_t(l01), bl1 = movmatrix_t(l23);

        // ---- O^T += V^T . P^T
  #pragma unroll
        for (int i = 0; i < NKS; ++i) {
          uint32_t a[4];
          // matrices: (keys 0-7, dims 0-7), (keys 0-7, dims 8-15), (keys 8-15, dims 0-7), (keys 8-15, dims 8-15)
          ldsm_x4_t(frag_addr(v_base, r_off + lr + (li >> 1) * 8, 2 * i + (li & 1)), a);
          mma_bf16(acc[i], a, bh0, bh1);
          mma_bf16(acc[i], a, bl0, bl1);
        }
        // the stage (and, for int8, the staging area) is free again
        if (!Q8 && rw0 + 16 > n) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++j;
      const int64_t seg_end = min(x_end, wk.base_b + (int64_t)(wk.h + 1) * wk.len);
      advance(n);
      if (wk.x >= seg_end) finish_unit(seg_end);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && flag[0]) atomicCAS(p.err, 0, 3);
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

// cache [rows, n_kv, D] viewed as 2-D [rows][n_kv * D]; boxes of BoxB bytes x
// kTR rows, BoxB-byte swizzle; rows past the cache read as zero
template <int D, bool Q8>
bool cache_map(CUtensorMap *m, const void *base, int64_t rows, int n_kv) {
  using L = MmaLayout<D, Q8>;
  PFN_encodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)n_kv * D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)n_kv * D * L::kEsz};
  cuuint32_t box[2] = {(cuuint32_t)(L::kBoxB / L::kEsz), (cuuint32_t)kTR};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz_mode = L::kBoxB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(m, Q8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz_mode, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool Q8, int G>
cudaError_t launch(const DecodeArgs &a, cudaStream_t st) {
  using L = MmaLayout<D, Q8>;
  CUtensorMap mk, mv;
  if (!cache_map<D, Q8>(&mk, a.k_c, a.cache_rows, a.n_kv) || !cache_map<D, Q8>(&mv, a.v_c, a.cache_rows, a.n_kv))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit((const void *)gqa_decode_mma<D, Q8, G>, L::kAlloc);
  if (e != cudaSuccess) return e;
  MmaParams p;
  p.q = static_cast<const __nv_bfloat16 *>(a.q);
  p.row_off = a.row_off; p.kv_len = a.kv_len;
  p.k_scale = a.k_scale; p.v_scale = a.v_scale; p.scale_pitch = a.scale_pitch;
  p.out = a.out; p.part = a.part; p.tickets = a.tickets; p.err = a.err;
  p.batch = a.batch; p.n_h = a.n_h; p.n_kv = a.n_kv; p.slots = a.n_chunks;
  p.cache_rows = a.cache_rows;
  p.c = a.scale * kLog2e;
  count_launch();
  return launch_pdl(gqa_decode_mma<D, Q8, G>, dim3(kNumSMs), dim3(kThr), (size_t)L::kAlloc, st, mk, mv, p);
}

template <int D, bool Q8>
cudaError_t by_group(const DecodeArgs &a, cudaStream_t st) {
  switch (a.n_h / a.n_kv) {
    case 1: return launch<D, Q8, 1>(a, st);
    case 2: return launch<D, Q8, 2>(a, st);
    case 4: return launch<D, Q8, 4>(a, st);
    default: return launch<D, Q8, 8>(a, st);
  }
}

}  // namespace

int decode_mma_tile_rows() { return kTR; }

cudaError_t gqa_decode_tc(const DecodeArgs &a, cudaStream_t st) {
  const bool q8 = a.k_scale != nullptr;
  if (q8) return a.d_h == 64 ? by_group<64, true>(a, st) : by_group<128, true>(a, st);
  return a.d_h == 64 ? by_group<64, false>(a, st) : by_group<128, false>(a, st);
}

}  // namespace kvc
