// GQA decode attention over compact caches on the tensor cores, fed by TMA:
//   out[b, qh] = softmax_t(scale * q[b, qh] . Kc[o_b + t, h]) . Vc[o_b + t, h],
//   h = qh / G.
// Decode streams the whole retained cache every step (FastKV section 1;
// "Variantes de l'attention et compression du cache KV", introduction), so the
// kernel is built to keep HBM busy with few instructions per cache byte and
// enough independent work per SM to hide the latency of each instruction:
//
//  * Work split (stream-K): the rows of all (batch entry, KV head) units are
//    laid end to end and every CTA (one per SM) takes an equal contiguous
//    slice, cut into tiles of up to 32 rows of one unit.
//  * Warp 8 is the producer: per tile one thread issues 2-D tensor-map copies
//    (cp.async.bulk.tensor, no multicast) of the head's K and V rows into a
//    ring of shared-memory stages (128-byte swizzle), completion counted in
//    bytes on the stage's mbarrier.  Rows past the cache read as zero.
//  * Warps 0-7 consume whole tiles in turn (tile j goes to warp j % 8), as two
//    independent 16-row groups, with mma.sync m16n8k16 (bf16 in, fp32
//    accumulate) in the transposed orientation, so the G <= 8 query heads of a
//    KV head fill the N = 8 side and no M rows are wasted:
//        S^T[key][head] = K[key][:] . Q[head][:]          (A = K via ldmatrix)
//        O^T[dim][head] += V^T[dim][key] . P^T[key][head] (A = V via ldmatrix.trans)
//    The S^T accumulator turns into the P^T operand with one movmatrix per
//    8x8 block.  P is split into two bf16 terms (p = hi + lo, |lo| <= 2^-9 p)
//    so the product keeps ~16 bits of every weight; the sum l of the weights
//    is accumulated from the fp32 values.
//  * Online softmax in log2 units per warp: the reference max of a head moves
//    only when a tile's logit exceeds it by more than kSlack (every weight
//    <= 2^kSlack), so rescaling is rare; it is uniform over the lanes of a head.
//  * At the end of a unit segment the eight warps merge through shared
//    memory; a unit split over several CTAs leaves (m, l, acc) partials and the
//    last CTA to finish it (atomic ticket, no waiting) merges them.
//
// The int8 variant reads caches quantised per (row, head) with a float32
// scale (K_c = s_k * q_k, V_c = s_v * q_v).  Its codes are widened exactly to
// bf16 in registers from 32-bit shared-memory loads: the K operand takes four
// consecutive dims of a row per load (the dims of a k-step are visited in the
// order 4t, 4t+1, 4t+2, 4t+3 for lane column t, and the query fragments use
// the same order); the V^T operand takes four consecutive dims of one key per
// load (output dims of two m-tiles are interleaved so that lane row g holds
// dims 4g .. 4g+3 of each 32-dim block).  The K scale multiplies the logit of
// its row and the V scale the weight of its row, so the products are those of
// the dequantised cache.
//
// Every wait is bounded: a wait that gives up sets the workspace error word;
// the warps keep walking the tiles without work so that they all meet at the
// same named barriers, and the producer waits (bounded) for its copies in
// flight before exiting.
#include <cuda.h>

#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kCons = 8;                  // consumer warps 0-7
constexpr int kMergeWarp = kCons;         // warp 8: merges the consumers' unit states
constexpr int kProdWarp = kCons + 1;      // warp 9: issues the tensor-map copies
constexpr int kThr = (kCons + 2) * 32;
constexpr int kTR = 32;                   // cache rows per tile (two 16-row groups)
constexpr int kRingBytes = 176 * 1024;
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
  // The stage count is a multiple of the consumer count: tile j uses stage
  // j % kStages and goes to warp j % kCons, so every use of a stage is consumed
  // by the same warp, in order.  A warp therefore never waits on the parity of
  // a stage's next use while its previous use is still landing (parity waits
  // only tell adjacent phases apart).
  static constexpr int kStagesRaw = kRingBytes / kStageB;
  static constexpr int kStagesCap = kStagesRaw > 16 ? 16 : kStagesRaw;
  static constexpr int kStages = kStagesCap / kCons * kCons;
  static_assert(kStages >= kCons && kStages % kCons == 0, "stages per consumer warp");
  // int8: per stage the K and V scales of the tile's rows (2 x kTR floats)
  static constexpr int kOffScale = kStages * kStageB;
  // barriers: full[16], empty[16], dump_full[2], dump_empty[2]
  static constexpr int kOffBar = kOffScale + (Q8 ? kStages * 2 * kTR * 4 : 0);
  static constexpr int kOffDump = kOffBar + 512;
  // two dump buffers: per consumer warp and head, (m, l, acc[D])
  static constexpr int kRec = D + 2;
  static constexpr int kDumpFloats = kCons * 8 * kRec;
  static constexpr int kOffFlag = kOffDump + 2 * kDumpFloats * 4;
  static constexpr int kBytes = kOffFlag + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kBoxBytes % 512 == 0 && kStageB % 1024 == 0, "swizzled boxes need their alignment");
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

// two int8 codes -> bf16x2 (exact), lo in the low half
KVC_DEVINL uint32_t i8pair_bf16(uint32_t lo_byte_src, int lo_shift, uint32_t hi_byte_src, int hi_shift) {
  return pack_bf16((float)(int8_t)((lo_byte_src >> lo_shift) & 0xffu), (float)(int8_t)((hi_byte_src >> hi_shift) & 0xffu));
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
  uint64_t *dump_full = empty + 16, *dump_empty = dump_full + 2;
  float *dump = reinterpret_cast<float *>(smem + L::kOffDump);   // [2][kCons][8][kRec]
  volatile int *flag = reinterpret_cast<volatile int *>(smem + L::kOffFlag);   // [0] error, [1] last
  const int warp = warp_id(), lane = lane_id();

  grid_dependency_wait();
  // ---- the flattened row space and this CTA's slice
  int64_t R = 0;
  for (int b = 0; b < p.batch; ++b) R += (int64_t)p.kv_len[b] * p.n_kv;
  const int64_t NC = R > 0 ? min((int64_t)gridDim.x, max((int64_t)1, R / (2 * kTR))) : 0;
  const int cta = blockIdx.x;
  // batch entries with an empty cache produce zeros (the merger warp of CTA
  // 0: it has no work before the first unit ends, so no tile waits for it)
  if (cta == 0 && warp == kMergeWarp)
    for (int b = 0; b < p.batch; ++b)
      if (p.kv_len[b] == 0)
        for (int e = lane; e < p.n_kv * G * D; e += 32) p.out[(size_t)b * p.n_h * D + e] = 0.f;
  if (cta >= NC) return;
  const int64_t x_begin = cta * R / NC, x_end = (cta + 1) * R / NC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], Q8 ? 1 + 32 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int d = 0; d < 2; ++d) {
      mbar_init(&dump_full[d], kCons);
      mbar_init(&dump_empty[d], 1);
    }
    flag[0] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  __syncthreads();

  // Tile walker shared by the producer and the consumers: the unit (b, h)
  // holding flattened row x, its length, and the first flattened row base_b
  // of batch entry b.
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

  if (warp == kProdWarp) {
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
        const int r = lane;                   // kTR == 32: one row per lane
        const bool ok = r < n;
        cp_async4(sk + r, gk + (ok ? row0 + r : 0), ok);
        cp_async4(sk + kTR + r, gv + (ok ? row0 + r : 0), ok);
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
  } else if (warp < kCons) {
    // ============================================================ consumers
    const int g = lane >> 2, t = lane & 3;                 // mma fragment coordinates
    const int lr = lane & 7, li = lane >> 3;               // ldmatrix row / matrix of this lane
    // query fragments (B operand of the logit product): head g, k-step ks.
    // bf16 caches: dims 16ks + 2t (+1) and 16ks + 8 + 2t (+1); int8 caches:
    // dims 16ks + 4t .. 16ks + 4t + 3 (the order of the widened K codes).
    uint32_t qf[NKS][2];
    float cz0 = p.c, cz1 = p.c;  // logit factors of heads 2t, 2t+1 (int8: divided by the query's power-of-two scale)
    float m[2], l[2], acc[NKS][4];
    int cur_b = -1, cur_h = -1;
    int64_t seg_u0 = 0;          // first flattened row of the current unit
    int j = 0;

    auto reset_unit = [&]() {
      const __nv_bfloat16 *qb = p.q + ((size_t)wk.b * p.n_h + (size_t)wk.h * G + g) * D;
      if constexpr (Q8) {
        // int8 caches: the query in f16, head g scaled by a power of two so
        // that its largest element lies in [2^13, 2^14): every element within
        // 2^27 of that largest converts exactly (bf16 carries 8 significant
        // bits); the logit factor divides the scale out again
        float qv[NKS][4];
        float mx = 0.f;
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
          uint2 q2 = make_uint2(0u, 0u);
          if (g < G) q2 = __ldg(reinterpret_cast<const uint2 *>(qb + 16 * ks + 4 * t));
          qv[ks][0] = bf16_lo(q2.x); qv[ks][1] = bf16_hi(q2.x); qv[ks][2] = bf16_lo(q2.y); qv[ks][3] = bf16_hi(q2.y);
#pragma unroll
          for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qv[ks][e]));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        int ex = 0;
        if (mx > 0.f) frexpf(mx, &ex);
        const float qs = mx > 0.f ? ldexpf(1.f, 14 - ex) : 1.f;
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
          qf[ks][0] = pack_f16(qv[ks][0] * qs, qv[ks][1] * qs);
          qf[ks][1] = pack_f16(qv[ks][2] * qs, qv[ks][3] * qs);
        }
        const float qinv = 1.f / qs;     // a power of two: exact
        cz0 = p.c * __shfl_sync(0xffffffffu, qinv, 8 * t);       // head 2t lives in lanes 8t .. 8t + 3
        cz1 = p.c * __shfl_sync(0xffffffffu, qinv, 8 * t + 4);   // head 2t + 1 in lanes 8t + 4 .. 8t + 7
      } else {
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
          if (g < G) {
            qf[ks][0] = __ldg(reinterpret_cast<const uint32_t *>(qb + 16 * ks + 2 * t));
            qf[ks][1] = __ldg(reinterpret_cast<const uint32_t *>(qb + 16 * ks + 8 + 2 * t));
          } else {
            qf[ks][0] = qf[ks][1] = 0u;
          }
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
    // output dim of accumulator element acc[i][e] (rows g and g+8 of m-tile i)
    auto acc_dim = [&](int i, int hi8) -> int {
      if constexpr (Q8) return 32 * (i >> 1) + 4 * g + 2 * (i & 1) + hi8;
      else return 16 * i + g + 8 * hi8;
    };

    // End of a unit segment: the warp's (m, l, acc) go to dump buffer
    // n_ends % 2 for the merger warp, and the warp moves on at once.
    int n_ends = 0;
    auto dump_unit = [&]() {
      // heads 2t, 2t+1: l summed over the rows g of the warp
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l[0] += __shfl_xor_sync(0xffffffffu, l[0], o);
        l[1] += __shfl_xor_sync(0xffffffffu, l[1], o);
      }
      const int d = n_ends & 1;
      // the buffer's previous use has been merged (bounded wait)
      bool ok = true;
      if (n_ends >= 2 && !flag[0]) ok = mbar_wait(&dump_empty[d], ((n_ends >> 1) - 1) & 1);
      if (!__all_sync(0xffffffffu, ok) && lane == 0) flag[0] = 1;
      float *dw = dump + (size_t)d * L::kDumpFloats + (size_t)warp * 8 * L::kRec;
      const int h0 = 2 * t, h1 = 2 * t + 1;
      if (g == 0) {
        if (h0 < G) { dw[h0 * L::kRec] = m[0]; dw[h0 * L::kRec + 1] = l[0]; }
        if (h1 < G) { dw[h1 * L::kRec] = m[1]; dw[h1 * L::kRec + 1] = l[1]; }
      }
#pragma unroll
      for (int i = 0; i < NKS; ++i) {
        if (h0 < G) {
          dw[h0 * L::kRec + 2 + acc_dim(i, 0)] = acc[i][0];
          dw[h0 * L::kRec + 2 + acc_dim(i, 1)] = acc[i][2];
        }
        if (h1 < G) {
          dw[h1 * L::kRec + 2 + acc_dim(i, 0)] = acc[i][1];
          dw[h1 * L::kRec + 2 + acc_dim(i, 1)] = acc[i][3];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dump_full[d]);
      ++n_ends;
    };

    while (wk.x < x_end) {
      const int n = tile_rows();
      if (wk.b != cur_b || wk.h != cur_h) reset_unit();
      const int s = j % L::kStages;
      if (j % kCons == warp) {
        // After a wait gave up the warps keep walking the tiles (so that all
        // of them meet at the same named barriers) but skip the work.
        bool ok = flag[0] == 0;
        if (ok) {
          const bool got = mbar_wait(&full[s], (j / L::kStages) & 1);
          if (!__all_sync(0xffffffffu, got)) { if (lane == 0) flag[0] = 1; ok = false; }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          uint8_t *stg_k = smem + s * L::kStageB;
          uint8_t *stg_v = stg_k + L::kTileB;
          const uint32_t k_base = smem_u32(stg_k), v_base = smem_u32(stg_v);
          bool vr[2][2];                                // row g / g+8 of group 0 / 1 valid
#pragma unroll
          for (int gr = 0; gr < 2; ++gr) { vr[gr][0] = 16 * gr + g < n; vr[gr][1] = 16 * gr + g + 8 < n; }
          float ksc[2][2] = {{1.f, 1.f}, {1.f, 1.f}}, vsc[2][2] = {{1.f, 1.f}, {1.f, 1.f}};
          if constexpr (Q8) {
            const float *scl = reinterpret_cast<const float *>(smem + L::kOffScale) + s * 2 * kTR;
#pragma unroll
            for (int gr = 0; gr < 2; ++gr)
#pragma unroll
              for (int hr = 0; hr < 2; ++hr) {
                ksc[gr][hr] = scl[16 * gr + g + 8 * hr];
                vsc[gr][hr] = scl[kTR + 16 * gr + g + 8 * hr];
              }
          } else if (n < kTR) {
            // rows past the segment: zero their V so that 0-weights meet finite values
            for (int e = lane; e < (kTR - n) * (D / 8); e += 32) {
              const int r = n + e / (D / 8), ch = e % (D / 8);
              *reinterpret_cast<uint4 *>(stg_v + swz<128, kTR>(r, ch)) = make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
          }

          // ---- S^T = K . Q^T for the two 16-row groups
          float sc[2][4];
#pragma unroll
          for (int gr = 0; gr < 2; ++gr) sc[gr][0] = sc[gr][1] = sc[gr][2] = sc[gr][3] = 0.f;
#pragma unroll
          for (int ks = 0; ks < NKS; ++ks) {
#pragma unroll
            for (int gr = 0; gr < 2; ++gr) {
              uint32_t a[4];
              if constexpr (Q8) {
                // rows g, g+8 of the group; dims 16ks + 4t .. +3 of each
                const uint32_t w0 = *reinterpret_cast<const uint32_t *>(stg_k + swz<L::kBoxB, kTR>(16 * gr + g, ks) + 4 * t);
                const uint32_t w1 = *reinterpret_cast<const uint32_t *>(stg_k + swz<L::kBoxB, kTR>(16 * gr + g + 8, ks) + 4 * t);
                i8x4_f16(w0, a[0], a[2]);
                i8x4_f16(w1, a[1], a[3]);
                mma_f16(sc[gr], a, qf[ks][0], qf[ks][1]);
              } else {
                // matrices: (rows 0-7, dims 0-7), (rows 8-15, dims 0-7), (rows 0-7, dims 8-15), (rows 8-15, dims 8-15)
                ldsm_x4(k_base + swz<128, kTR>(16 * gr + lr + (li & 1) * 8, 2 * ks + (li >> 1)), a);
                mma_bf16(sc[gr], a, qf[ks][0], qf[ks][1]);
              }
            }
          }
          // logits in log2 units: (row g, heads 2t, 2t+1), (row g+8, same heads)
          float z[2][4];
#pragma unroll
          for (int gr = 0; gr < 2; ++gr) {
            z[gr][0] = vr[gr][0] ? sc[gr][0] * cz0 * ksc[gr][0] : kNegInf;
            z[gr][1] = vr[gr][0] ? sc[gr][1] * cz1 * ksc[gr][0] : kNegInf;
            z[gr][2] = vr[gr][1] ? sc[gr][2] * cz0 * ksc[gr][1] : kNegInf;
            z[gr][3] = vr[gr][1] ? sc[gr][3] * cz1 * ksc[gr][1] : kNegInf;
          }
          float tmax0 = fmaxf(fmaxf(z[0][0], z[0][2]), fmaxf(z[1][0], z[1][2]));
          float tmax1 = fmaxf(fmaxf(z[0][1], z[0][3]), fmaxf(z[1][1], z[1][3]));
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
          uint32_t bh[2][2], bl[2][2];
#pragma unroll
          for (int gr = 0; gr < 2; ++gr) {
            float pw[4];
            pw[0] = vr[gr][0] ? fast_exp2(z[gr][0] - ms0) : 0.f;
            pw[1] = vr[gr][0] ? fast_exp2(z[gr][1] - ms1) : 0.f;
            pw[2] = vr[gr][1] ? fast_exp2(z[gr][2] - ms0) : 0.f;
            pw[3] = vr[gr][1] ? fast_exp2(z[gr][3] - ms1) : 0.f;
            l[0] += pw[0] + pw[2];
            l[1] += pw[1] + pw[3];
            if constexpr (Q8) {
              pw[0] *= vsc[gr][0]; pw[1] *= vsc[gr][0]; pw[2] *= vsc[gr][1]; pw[3] *= vsc[gr][1];
            }
            // P^T operand: two bf16 terms per weight, transposed per 8x8 block
            const uint32_t h01 = pack_bf16(pw[0], pw[1]), h23 = pack_bf16(pw[2], pw[3]);
            const uint32_t l01 = pack_bf16(pw[0] - bf16_lo(h01), pw[1] - bf16_hi(h01));
            const uint32_t l23 = pack_bf16(pw[2] - bf16_lo(h23), pw[3] - bf16_hi(h23));
            bh[gr][0] = movmatrix_t(h01);
            bh[gr][1] = movmatrix_t(h23);
            bl[gr][0] = movmatrix_t(l01);
            bl[gr][1] = movmatrix_t(l23);
          }

          // ---- O^T += V^T . P^T
          if constexpr (Q8) {
#pragma unroll
            for (int pr = 0; pr < NKS / 2; ++pr) {       // m-tiles 2pr, 2pr+1: dims 32pr + 4g .. +3
#pragma unroll
              for (int gr = 0; gr < 2; ++gr) {
                // keys 2t, 2t+1, 2t+8, 2t+9 of the group, 4 dims each
                const int chv = 2 * pr + (g >> 2), bo = 4 * (g & 3);
                const uint32_t w0 = *reinterpret_cast<const uint32_t *>(stg_v + swz<L::kBoxB, kTR>(16 * gr + 2 * t, chv) + bo);
                const uint32_t w1 = *reinterpret_cast<const uint32_t *>(stg_v + swz<L::kBoxB, kTR>(16 * gr + 2 * t + 1, chv) + bo);
                const uint32_t w2 = *reinterpret_cast<const uint32_t *>(stg_v + swz<L::kBoxB, kTR>(16 * gr + 2 * t + 8, chv) + bo);
                const uint32_t w3 = *reinterpret_cast<const uint32_t *>(stg_v + swz<L::kBoxB, kTR>(16 * gr + 2 * t + 9, chv) + bo);
                uint32_t a[4];
                a[0] = i8pair_bf16(w0, 0, w1, 0);   a[1] = i8pair_bf16(w0, 8, w1, 8);
                a[2] = i8pair_bf16(w2, 0, w3, 0);   a[3] = i8pair_bf16(w2, 8, w3, 8);
                mma_bf16(acc[2 * pr], a, bh[gr][0], bh[gr][1]);
                mma_bf16(acc[2 * pr], a, bl[gr][0], bl[gr][1]);
                a[0] = i8pair_bf16(w0, 16, w1, 16); a[1] = i8pair_bf16(w0, 24, w1, 24);
                a[2] = i8pair_bf16(w2, 16, w3, 16); a[3] = i8pair_bf16(w2, 24, w3, 24);
                mma_bf16(acc[2 * pr + 1], a, bh[gr][0], bh[gr][1]);
                mma_bf16(acc[2 * pr + 1], a, bl[gr][0], bl[gr][1]);
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < NKS; ++i) {
#pragma unroll
              for (int gr = 0; gr < 2; ++gr) {
                uint32_t a[4];
                // matrices: (keys 0-7, dims 0-7), (keys 0-7, dims 8-15), (keys 8-15, dims 0-7), (keys 8-15, dims 8-15)
                ldsm_x4_t(v_base + swz<128, kTR>(16 * gr + lr + (li >> 1) * 8, 2 * i + (li & 1)), a);
                mma_bf16(acc[i], a, bh[gr][0], bh[gr][1]);
                mma_bf16(acc[i], a, bl[gr][0], bl[gr][1]);
              }
            }
          }
          // the stage is free again (order the zeroing stores before the next TMA write)
          if (!Q8 && n < kTR) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      ++j;
      const int64_t seg_end = min(x_end, wk.base_b + (int64_t)(wk.h + 1) * wk.len);
      advance(n);
      if (wk.x >= seg_end) dump_unit();
    }
  } else {
    // ============================================================ merger
    // Walks the same tiles; at every unit end it merges the consumers' dumps
    // and writes the output, or a partial record when other CTAs share the
    // unit (the last CTA to finish the unit merges the records: atomic
    // ticket, no waiting).
    auto owner = [&](int64_t xx) {
      int64_t c = xx * NC / R;
      while (c + 1 < NC && (c + 1) * R / NC <= xx) ++c;
      while (c > 0 && c * R / NC > xx) --c;
      return c;
    };
    constexpr int REC = D + 4;
    int k = 0;
    while (wk.x < x_end) {
      const int n = tile_rows();
      const int b = wk.b, h = wk.h;
      const int64_t seg_u0 = wk.base_b + (int64_t)wk.h * wk.len;
      const int64_t seg_end = min(x_end, seg_u0 + wk.len);
      advance(n);
      if (wk.x < seg_end) continue;
      const int d = k & 1;
      bool ok = flag[0] == 0 && mbar_wait(&dump_full[d], (k >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && lane == 0) flag[0] = 1;
      const int u = b * p.n_kv + h;
      const int len = p.kv_len[b];
      const int64_t first = owner(seg_u0), last = owner(seg_u0 + len - 1);
      float *outp = p.out + ((size_t)b * p.n_h + (size_t)h * G) * D;
      float *pp = p.part + ((size_t)u * p.slots + (size_t)(cta - first)) * (size_t)(G * REC);
      const float *dmp = dump + (size_t)d * L::kDumpFloats;
      if (ok) {
        // every lane owns D / 32 consecutive dims of every head
        constexpr int DPL = D / 32;
#pragma unroll
        for (int hd = 0; hd < G; ++hd) {
          float M = kNegInf;
#pragma unroll
          for (int w2 = 0; w2 < kCons; ++w2) M = fmaxf(M, dmp[(w2 * 8 + hd) * L::kRec]);
          float Ls = 0.f, A[DPL];
#pragma unroll
          for (int i = 0; i < DPL; ++i) A[i] = 0.f;
          if (M != kNegInf) {
#pragma unroll
            for (int w2 = 0; w2 < kCons; ++w2) {
              const float *rw = dmp + (w2 * 8 + hd) * L::kRec;
              const float sc = rw[0] == kNegInf ? 0.f : fast_exp2(rw[0] - M);
              Ls += rw[1] * sc;
#pragma unroll
              for (int i = 0; i < DPL; ++i) A[i] = fmaf(rw[2 + lane * DPL + i], sc, A[i]);
            }
          }
          if (first == last) {
#pragma unroll
            for (int i = 0; i < DPL; ++i) outp[hd * D + lane * DPL + i] = A[i] / Ls;
          } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) pp[hd * REC + 4 + lane * DPL + i] = A[i];
            if (lane == 0) { pp[hd * REC] = M; pp[hd * REC + 1] = Ls; }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dump_empty[d]);    // the consumers may reuse the buffer
      ++k;
      if (ok && first != last) {
        __threadfence();
        __syncwarp();
        int last_in = 0;
        if (lane == 0) last_in = (atomicAdd(&p.tickets[u], 1) == (int)(last - first)) ? 1 : 0;
        last_in = __shfl_sync(0xffffffffu, last_in, 0);
        if (last_in) {
          // every lane owns D / 32 consecutive dims of every head and folds
          // the segments in with a running max; the loads of a segment are
          // independent of the running values, so they overlap
          __threadfence();
          constexpr int DPL = D / 32;
          const int n_seg = (int)(last - first + 1);
          const float *pu = p.part + (size_t)u * p.slots * (size_t)(G * REC);
          float M[G], Ls[G], A[G][DPL];
#pragma unroll
          for (int hd = 0; hd < G; ++hd) {
            M[hd] = kNegInf;
            Ls[hd] = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) A[hd][i] = 0.f;
          }
#pragma unroll 2
          for (int sgi = 0; sgi < n_seg; ++sgi) {
            float mj[G], lj[G], aj[G][DPL];
#pragma unroll
            for (int hd = 0; hd < G; ++hd) {
              const float *rec = pu + ((size_t)sgi * G + hd) * REC;
              mj[hd] = __ldcg(rec);
              lj[hd] = __ldcg(rec + 1);
              if constexpr (DPL == 4) {
                const float4 a4 = __ldcg(reinterpret_cast<const float4 *>(rec + 4) + lane);
                aj[hd][0] = a4.x; aj[hd][1] = a4.y; aj[hd][2] = a4.z; aj[hd][3] = a4.w;
              } else {
                const float2 a2 = __ldcg(reinterpret_cast<const float2 *>(rec + 4) + lane);
                aj[hd][0] = a2.x; aj[hd][1] = a2.y;
              }
            }
#pragma unroll
            for (int hd = 0; hd < G; ++hd) {
              const float mn = fmaxf(M[hd], mj[hd]);
              if (mn == kNegInf) continue;
              const float sa = M[hd] == kNegInf ? 0.f : fast_exp2(M[hd] - mn);
              const float sb = mj[hd] == kNegInf ? 0.f : fast_exp2(mj[hd] - mn);
              Ls[hd] = Ls[hd] * sa + lj[hd] * sb;
#pragma unroll
              for (int i = 0; i < DPL; ++i) A[hd][i] = A[hd][i] * sa + aj[hd][i] * sb;
              M[hd] = mn;
            }
          }
#pragma unroll
          for (int hd = 0; hd < G; ++hd)
#pragma unroll
            for (int i = 0; i < DPL; ++i) outp[hd * D + lane * DPL + i] = A[hd][i] / Ls[hd];
          if (lane == 0) p.tickets[u] = 0;           // leave the counter zeroed for the next call
        }
      }
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
