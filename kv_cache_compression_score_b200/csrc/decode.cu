// GQA decode attention over float32 compact caches: out[b, qh] = softmax(scale *
// q[b, qh] . Kc[o_b + t, h]) . Vc[o_b + t, h], h = qh / G.  Decode streams
// the whole retained cache every step, so the kernel is an HBM stream (FastKV
// section 1; "Variantes de l'attention et compression du cache KV",
// introduction).
//
// Work split (stream-K over warps): the rows of all (batch entry, KV head)
// units are laid end to end and every warp of the grid takes an equal
// contiguous slice, so the load is balanced to a row whatever the lengths.
// A slice covers one or a few unit segments; each segment yields a partial
// (m, l, acc) and the last warp to finish a unit (atomic ticket, no waiting)
// merges its partials into the output.
//
// Per warp: a row of d_h elements is split over LPR = d_h / 16 lanes (16
// elements each), RPW = 32 / LPR rows per step.  Each lane prefetches the K
// and V bytes it will read itself with 16-byte cp.async into a private ring
// (so no cross-lane synchronisation is needed), computes its G query-head
// partial dot products (fma.rn.f32x2), reduces them over the LPR lanes with
// xor-shuffles and keeps an online softmax whose reference max is only moved,
// by warp vote, when a logit exceeds it by more than kSlack (log2 units):
// p = 2^(s - m) <= 2^kSlack never overflows and the rare rescale is
// warp-uniform.
#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kWarps = 8;                 // warps per CTA
constexpr int kThreadsDec = kWarps * 32;
constexpr float kSlack = 8.f;             // log2 headroom before the reference max moves
constexpr int kMinRowsPerWarp = 32;

template <typename T>
struct DecRing {
  static constexpr int kNch = (int)sizeof(T);                 // 16-byte chunks per lane and row (16 elements)
  static constexpr int kLaneBytes = kNch * 16 * 2;             // K + V of one row slice
  static constexpr int kStepBytes = 32 * kLaneBytes;           // whole warp
  static constexpr int kDepth = sizeof(T) == 2 ? 8 : 4;       // steps per warp (power of two)
  static constexpr int kSmem = kWarps * kDepth * kStepBytes;   // 128 KB
};

// partial record of one segment and head: m, l, 2 pad words, acc[D]
template <int D> constexpr int rec_floats() { return D + 4; }

struct DecParams {
  const void *q, *kc, *vc;
  const int64_t *row_off;
  const int *kv_len;
  float *out;
  float *part;
  int *tickets;
  int batch, n_h, n_kv, slots;   // slots: partial slots per unit
  float c;                       // scale * log2(e)
};

// (a0, a1) += (x0, x1) * (y0, y1) as one packed fp32x2 FMA
KVC_DEVINL void ffma2(float &a0, float &a1, float x0, float x1, float y0, float y1) {
  asm("{\n\t.reg .b64 x, y, a;\n\t"
      "mov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %5};\n\tmov.b64 a, {%0, %1};\n\t"
      "fma.rn.f32x2 a, x, y, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(x0), "f"(x1), "f"(y0), "f"(y1));
}

template <typename T> KVC_DEVINL void unpack16(const uint4 &v, float *o);
template <> KVC_DEVINL void unpack16<__nv_bfloat16>(const uint4 &v, float *o) { Elem<__nv_bfloat16>::unpack(v, o); }
template <> KVC_DEVINL void unpack16<float>(const uint4 &v, float *o) { Elem<float>::unpack(v, o); }

// warp w's slice of the flattened row space is [start(w), start(w + 1))
KVC_DEVINL int64_t slice_start(int64_t w, int64_t R, int64_t NW) { return w * R / NW; }
// the warp whose slice contains global row x (0 <= x < R)
KVC_DEVINL int64_t owner(int64_t x, int64_t R, int64_t NW) {
  int64_t w = x * NW / R;
  while (w + 1 < NW && slice_start(w + 1, R, NW) <= x) ++w;
  while (w > 0 && slice_start(w, R, NW) > x) --w;
  return w;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreadsDec, 1) gqa_decode_streamk(DecParams p) {
  grid_dependency_wait();
  using RG = DecRing<T>;
  constexpr int LPR = D / 16;              // lanes per row
  constexpr int RPW = 32 / LPR;            // rows per warp step
  constexpr int EPC = 16 / (int)sizeof(T); // elements per 16-byte chunk
  constexpr int NCH = RG::kNch;
  constexpr int kRing = RG::kDepth;
  static_assert(NCH * EPC == 16, "16 elements per lane");
  extern __shared__ uint4 smem_v4[];
  uint8_t *smem_raw = reinterpret_cast<uint8_t *>(smem_v4);
  const int warp = warp_id(), lane = lane_id();
  // ring of kRing steps per warp; within a step, 16-byte chunk j of lane L sits
  // at (j * 32 + L) * 16 so a quarter warp touches 128 consecutive bytes
  uint8_t *ring = smem_raw + warp * kRing * RG::kStepBytes + lane * 16;
  const int rg = lane / LPR, sl = lane % LPR;
  const int n_units = p.batch * p.n_kv;

  // ---- the flattened row space and this warp's slice
  int64_t R = 0;
  for (int b = 0; b < p.batch; ++b) R += (int64_t)p.kv_len[b] * p.n_kv;
  const int64_t NW_all = (int64_t)gridDim.x * kWarps;
  const int64_t NW = R > 0 ? min(NW_all, max((int64_t)1, R / kMinRowsPerWarp)) : 0;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + warp;

  // units of empty caches produce zeros (first warp of the grid)
  if (gw == 0)
    for (int u = 0; u < n_units; ++u)
      if (p.kv_len[u / p.n_kv] == 0)
        for (int e = lane; e < G * D; e += 32)
          p.out[((size_t)(u / p.n_kv) * p.n_h + (size_t)(u % p.n_kv) * G) * D + e] = 0.f;
  if (gw >= NW) return;

  int64_t x = slice_start(gw, R, NW);
  const int64_t x_end = slice_start(gw + 1, R, NW);
  // locate the unit containing row x
  int b = 0;
  int64_t base_b = 0;
  while (base_b + (int64_t)p.kv_len[b] * p.n_kv <= x) { base_b += (int64_t)p.kv_len[b] * p.n_kv; ++b; }

  while (x < x_end) {
    const int len = p.kv_len[b];
    const int h = (int)((x - base_b) / len);
    const int64_t u0 = base_b + (int64_t)h * len;           // unit start in the row space
    const int r0 = (int)(x - u0);
    const int r1 = (int)(min(x_end, u0 + len) - u0);
    const int u = b * p.n_kv + h;

    // query slices of the G heads of h: element d = j * (LPR * EPC) + sl * EPC + i of chunk j.
    // Slot g holds head g ^ xq: with this lane-dependent order every stage of
    // the reduce-scatter below keeps the low half of the slots and sends the
    // high half, so it needs no selects.
    const int xq = (G <= LPR) ? (sl / (LPR / G)) & (G - 1) : 0;
    float qr[G][16];
    const T *qb = static_cast<const T *>(p.q) + ((size_t)b * p.n_h + (size_t)h * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        unpack16<T>(ld_nc16(qb + (size_t)(g ^ xq) * D + j * (LPR * EPC) + sl * EPC), &qr[g][j * EPC]);
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

    const int64_t o = p.row_off[b];
    const T *kb = static_cast<const T *>(p.kc) + ((size_t)o * p.n_kv + h) * D + sl * EPC;
    const T *vb = static_cast<const T *>(p.vc) + ((size_t)o * p.n_kv + h) * D + sl * EPC;
    const size_t rstride = (size_t)p.n_kv * D;
    const int n_steps = (r1 - r0 + RPW - 1) / RPW;
    const size_t step_stride = (size_t)RPW * rstride;
    const T *k_any = kb + (size_t)r0 * rstride, *v_any = vb + (size_t)r0 * rstride;   // a valid dummy source
    const T *kq = kb + (size_t)(r0 + rg) * rstride, *vq = vb + (size_t)(r0 + rg) * rstride;
    // ring pointers: the slot of the next prefetched step and of the next consumed one
    uint8_t *const ring_end = ring + kRing * RG::kStepBytes;
    uint8_t *pf_dst = ring;
    const uint8_t *src = ring;
    int pf_row = r0 + rg;        // this lane's row of the next prefetched step
    auto prefetch = [&]() {
      // zero-filled (no read) past the segment; one cp.async group per step
      const bool ok = pf_row < r1;
      const T *ks = ok ? kq : k_any, *vs = ok ? vq : v_any;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        cp_async16(pf_dst + j * 512, ks + j * (LPR * EPC), ok);
        cp_async16(pf_dst + (NCH + j) * 512, vs + j * (LPR * EPC), ok);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      kq += step_stride;
      vq += step_stride;
      pf_row += RPW;
      pf_dst += RG::kStepBytes;
      if (pf_dst == ring_end) pf_dst = ring;
    };
#pragma unroll 1
    for (int s = 0; s < kRing - 1; ++s) prefetch();
    int row = r0 + rg;
#pragma unroll 1
    for (int st = 0; st < n_steps; ++st) {
      prefetch();                               // step st + kRing - 1
      asm volatile("cp.async.wait_group %0;" :: "n"(kRing - 1) : "memory");
      const bool valid = row < r1;
      row += RPW;
      float kf[16];
#pragma unroll
      for (int j = 0; j < NCH; ++j) unpack16<T>(*reinterpret_cast<const uint4 *>(src + j * 512), &kf[j * EPC]);
      float sc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int e = 0; e < 16; e += 2) ffma2(a0, a1, qr[g][e], qr[g][e + 1], kf[e], kf[e + 1]);
        sc[g] = a0 + a1;
      }
      if constexpr (G <= LPR) {
        // reduce-scatter over the LPR lanes of the row: afterwards this lane
        // holds the full logit of one head, xq = sl / (LPR / G); slot j holds
        // head j ^ xq, so the partner across bit o needs exactly our high half
#pragma unroll
        for (int k = G, o = LPR / 2; k > 1; k >>= 1, o >>= 1)
#pragma unroll
          for (int j = 0; j < k / 2; ++j) sc[j] += __shfl_xor_sync(0xffffffffu, sc[k / 2 + j], o);
#pragma unroll
        for (int o = (LPR / G) / 2; o >= 1; o >>= 1) sc[0] += __shfl_xor_sync(0xffffffffu, sc[0], o);
        const float s_my = sc[0];
        const int src0 = rg * LPR;                     // lane of head g: src0 + g * (LPR / G)
        // move this lane's reference max only when its logit exceeds it by kSlack
        const bool need = valid && s_my > m[0] + kSlack;
        if (__any_sync(0xffffffffu, need)) {
          const float mn = valid ? fmaxf(m[0], s_my) : m[0];
          const float a = (mn == kNegInf) ? 1.f : fast_exp2(m[0] - mn);
          l[0] *= a;
          m[0] = mn;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float ag = __shfl_sync(0xffffffffu, a, src0 + g * (LPR / G));
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[g][e] *= ag;
          }
        }
        const float pr = valid ? fast_exp2(s_my - m[0]) : 0.f;
        l[0] += pr;
        float pg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pg[g] = __shfl_sync(0xffffffffu, pr, src0 + g * (LPR / G));
        if (valid) {
          float vf[16];
#pragma unroll
          for (int j = 0; j < NCH; ++j)
            unpack16<T>(*reinterpret_cast<const uint4 *>(src + (NCH + j) * 512), &vf[j * EPC]);
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 16; e += 2) ffma2(acc[g][e], acc[g][e + 1], pg[g], pg[g], vf[e], vf[e + 1]);
        }
      } else {
        // more heads than lanes per row: every lane reduces every head
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1)
#pragma unroll
          for (int g = 0; g < G; ++g) sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], off);
        bool need = false;
#pragma unroll
        for (int g = 0; g < G; ++g) need |= valid && sc[g] > m[g] + kSlack;
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float mn = valid ? fmaxf(m[g], sc[g]) : m[g];
            const float a = (mn == kNegInf) ? 1.f : fast_exp2(m[g] - mn);
            l[g] *= a;
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[g][e] *= a;
            m[g] = mn;
          }
        }
        if (valid) {
          float vf[16];
#pragma unroll
          for (int j = 0; j < NCH; ++j)
            unpack16<T>(*reinterpret_cast<const uint4 *>(src + (NCH + j) * 512), &vf[j * EPC]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pr = fast_exp2(sc[g] - m[g]);
            l[g] += pr;
#pragma unroll
            for (int e = 0; e < 16; e += 2) ffma2(acc[g][e], acc[g][e + 1], pr, pr, vf[e], vf[e + 1]);
          }
        }
      }
      src += RG::kStepBytes;
      if (src == ring_end) src = ring;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");

    if constexpr (G <= LPR) {
      // every lane of the row group takes the (m, l) of each head from its owner lane
      const float m_my = m[0], l_my = l[0];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = __shfl_sync(0xffffffffu, m_my, rg * LPR + g * (LPR / G));
        l[g] = __shfl_sync(0xffffffffu, l_my, rg * LPR + g * (LPR / G));
      }
    }
    // merge the row groups of the warp (lanes holding the same slice)
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m[g], off);
        const float l2 = __shfl_xor_sync(0xffffffffu, l[g], off);
        const float mn = fmaxf(m[g], m2);
        const float s1 = (mn == kNegInf) ? 0.f : fast_exp2(m[g] - mn);
        const float s2 = (mn == kNegInf) ? 0.f : fast_exp2(m2 - mn);
        l[g] = l[g] * s1 + l2 * s2;
        m[g] = mn;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a2 = __shfl_xor_sync(0xffffffffu, acc[g][e], off);
          acc[g][e] = acc[g][e] * s1 + a2 * s2;
        }
      }

    float *outp = p.out + ((size_t)b * p.n_h + (size_t)h * G) * D;
    const int64_t first = owner(u0, R, NW), last = owner(u0 + len - 1, R, NW);
    if (first == last) {
      // this warp owns the whole unit
      if (rg == 0)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int j = 0; j < NCH; ++j)
#pragma unroll
            for (int i = 0; i < EPC; ++i)
              outp[g * D + j * (LPR * EPC) + sl * EPC + i] = acc[g][j * EPC + i] / l[g];
    } else {
      constexpr int REC = rec_floats<D>();
      float *pp = p.part + ((size_t)u * p.slots + (size_t)(gw - first)) * (size_t)(G * REC);
      if (rg == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (sl == 0) { pp[g * REC] = m[g]; pp[g * REC + 1] = l[g]; }
#pragma unroll
          for (int j = 0; j < NCH; ++j)
#pragma unroll
            for (int i = 0; i < EPC; ++i) pp[g * REC + 4 + j * (LPR * EPC) + sl * EPC + i] = acc[g][j * EPC + i];
        }
      }
      __threadfence();
      __syncwarp();
      int last_in = 0;
      if (lane == 0) last_in = (atomicAdd(&p.tickets[u], 1) == (int)(last - first));
      last_in = __shfl_sync(0xffffffffu, last_in, 0);
      if (last_in) {
        __threadfence();
        const int n_seg = (int)(last - first + 1);
        const float *pu = p.part + (size_t)u * p.slots * (size_t)(G * REC);
        // segment weights: lane j holds segment j's (m, l) of every head
        float Mg[G], Lg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float mx = kNegInf;
          for (int j = lane; j < n_seg; j += 32) mx = fmaxf(mx, __ldcg(pu + ((size_t)j * G + g) * REC));
          Mg[g] = warp_max(mx);
          float ls = 0.f;
          for (int j = lane; j < n_seg; j += 32) {
            const float2 ml = __ldcg(reinterpret_cast<const float2 *>(pu + ((size_t)j * G + g) * REC));
            if (ml.x != kNegInf) ls += ml.y * fast_exp2(ml.x - Mg[g]);
          }
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o2);
          Lg[g] = ls;
        }
        // accumulators: lane covers D / 32 consecutive elements of every head
        constexpr int EPL = D / 32;
        float A[G][EPL];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int i = 0; i < EPL; ++i) A[g][i] = 0.f;
#pragma unroll 4
        for (int j = 0; j < n_seg; ++j) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float *rec = pu + ((size_t)j * G + g) * REC;
            const float mj = __ldcg(rec);
            const float wgt = (mj == kNegInf) ? 0.f : fast_exp2(mj - Mg[g]);
            if constexpr (EPL == 4) {
              const float4 a4 = __ldcg(reinterpret_cast<const float4 *>(rec + 4) + lane);
              A[g][0] = fmaf(a4.x, wgt, A[g][0]); A[g][1] = fmaf(a4.y, wgt, A[g][1]);
              A[g][2] = fmaf(a4.z, wgt, A[g][2]); A[g][3] = fmaf(a4.w, wgt, A[g][3]);
            } else {
              const float2 a2 = __ldcg(reinterpret_cast<const float2 *>(rec + 4) + lane);
              A[g][0] = fmaf(a2.x, wgt, A[g][0]); A[g][1] = fmaf(a2.y, wgt, A[g][1]);
            }
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int i = 0; i < EPL; ++i) outp[g * D + lane * EPL + i] = A[g][i] / Lg[g];
        if (lane == 0) p.tickets[u] = 0;   // leave the counter zeroed for the next call
      }
    }
    // next segment: the rest of this unit's rows belong to later warps, or
    // the next unit starts here
    x = u0 + r1;
    if (r1 == len && h == p.n_kv - 1 && x < x_end) {
      base_b += (int64_t)len * p.n_kv;
      ++b;
      while (p.kv_len[b] == 0) ++b;   // x < x_end <= R: a non-empty entry follows
    }
  }
}

template <typename T, int D, int G>
cudaError_t launch(const DecodeArgs &a, cudaStream_t st) {
  const int smem = DecRing<T>::kSmem;
  cudaError_t e = ensure_smem_limit((const void *)gqa_decode_streamk<T, D, G>, smem);
  if (e != cudaSuccess) return e;
  DecParams p;
  p.q = a.q; p.kc = a.k_c; p.vc = a.v_c; p.row_off = a.row_off; p.kv_len = a.kv_len; p.out = a.out;
  p.part = a.part; p.tickets = a.tickets; p.batch = a.batch; p.n_h = a.n_h; p.n_kv = a.n_kv;
  p.slots = a.n_chunks; p.c = a.scale * kLog2e;
  count_launch();
  return launch_pdl(gqa_decode_streamk<T, D, G>, dim3(kNumSMs), dim3(kThreadsDec), (size_t)smem, st, p);
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

// Partial slots a unit can need: every warp slice holds at least
// kMinRowsPerWarp rows, so a unit of len rows meets at most
// len / kMinRowsPerWarp + 2 slices.
int decode_slots(int max_kv_len) { return max_kv_len / kMinRowsPerWarp + 2; }

// float32 caches run on the CUDA cores (full fp32 products); bf16 and int8
// caches go to the tensor-core kernel (decode_mma.cu)
cudaError_t gqa_decode(const DecodeArgs &a, cudaStream_t st) {
  if (a.dt == KVC_F32) return a.d_h == 64 ? by_group<float, 64>(a, st) : by_group<float, 128>(a, st);
  return gqa_decode_tc(a, st);
}

}  // namespace kvc
