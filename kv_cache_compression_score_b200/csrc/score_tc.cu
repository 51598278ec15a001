// Observation-window saliency scores on the 5th-generation tensor cores
// (bf16 inputs, float32 accumulation in tensor memory).
//
// Same exact two-pass softmax as the CUDA-core kernels (SnapKV observation
// window, "Variantes de l'attention et compression du cache KV", section
// "Compresser un cache existant"; causal window rows from section "Quand la
// reutilisation est-elle exacte ?"), with the window-block x key-tile
// contraction issued as tcgen05.mma:
//
//   stats pass:  D[row][key] = Q_win[row] . K[key]   (M = 128 rows, N = 128 keys)
//                one epilogue thread per TMEM lane = window row keeps the
//                running max / sum of 2^(y - m) in registers;
//   score pass:  D[key][row] = K[key] . Q_win[row]   (M = 128 keys, N = rows)
//                one epilogue thread per TMEM lane = key sums 2^(y - off_r)
//                over the rows, off_r = m_r + log2(l_r) merged from the
//                stats partials.
//
// Warp roles (192 threads): warp 0 streams K tiles with TMA into a 4-stage
// shared-memory ring (128-byte swizzle, no multicast), warp 1 owns tensor
// memory and issues the MMAs (one thread), warps 2-5 are the epilogue.  The
// accumulator is double-buffered in tensor memory (2 x 128 columns) so the
// MMA of tile t+1 overlaps the epilogue of tile t.  Every wait is bounded;
// a wait that gives up sets the device error word and the CTA drains.
#include <cuda.h>

#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kBN = 128;        // keys per tile (MMA N in the stats pass, M in the score pass)
constexpr int kRows = 128;      // window-block rows (padded)
constexpr int kStages = 4;
constexpr int kThreadsTC = 192;
constexpr int kEpiWarp0 = 2;

template <int D>
struct TcLayout {
  static constexpr int kAtoms = D / 64;                     // 128-byte swizzle atoms along d
  static constexpr int kQBytes = kRows * D * 2;              // window block
  static constexpr int kKBytes = kBN * D * 2;                // one K tile
  static constexpr int kAtomBytes = 128 * 128;               // 128 rows x 128 B
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffK + kStages * kKBytes;
  static constexpr int kBarCount = 2 * kStages + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + 128;           // 13 barriers need 104 bytes
  static constexpr int kOffOff = kOffMisc + 16;             // score pass: off_r[128], 16-byte aligned
  static constexpr int kBytes = kOffOff + kRows * 4;
  static constexpr int kAlloc = kBytes + 1024;              // room to align the base to 1 KB
  static_assert(kBarCount * 8 <= 128, "barrier area");
  static_assert(kOffOff % 16 == 0, "off[] is read as float4");
  static_assert(kOffK % 1024 == 0 && kKBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");
};

struct TcParams {
  const __nv_bfloat16 *q_win;
  const int *cu_seqlens;
  float2 *part;
  float *raw;
  int *err;
  int n_h, n_kv, G, w, R, n_chunks, keys_per_chunk, T_total;
  float c;   // scale * log2(e)
};

// Q_win rows r = g * w + i of (b, h) into the 128-byte-swizzled K-major tile;
// rows >= R are zero.  Generic-proxy writes, made visible to the tensor core
// by fence.proxy.async before the MMA thread is released.
template <int D>
KVC_DEVINL void stage_q(uint8_t *sq, const TcParams &p, int b, int h, int tid, int nthreads) {
  constexpr int kChunks = D / 8;   // 16-byte chunks per row
  for (int e = tid; e < kRows * kChunks; e += nthreads) {
    const int r = e / kChunks, ch = e % kChunks;
    const int atom = ch >> 3, c16 = ch & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < p.R) {
      const int g = r / p.w, i = r % p.w;
      v = *reinterpret_cast<const uint4 *>(p.q_win + ((size_t)(b * p.w + i) * p.n_h + (size_t)h * p.G + g) * D + ch * 8);
    }
    *reinterpret_cast<uint4 *>(sq + atom * TcLayout<D>::kAtomBytes + r * 128 + ((c16 ^ (r & 7)) << 4)) = v;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

KVC_DEVINL void set_err(int *err, int code) { atomicCAS(err, 0, code); }

// Stats-pass reduction of 32 logits of one window row (keys k0..k0+31):
// online max / sum of 2^(c*z - m), masked keys (beyond the chunk end or the
// row's causal limit) contribute nothing.
KVC_DEVINL void epi_stats_chunk(float *v, int k0, int key_end, int P, int row_pos, float c, float &m, float &l) {
  if (!(k0 + 31 <= P && k0 + 32 <= key_end)) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int key = k0 + j;
      if (!(key < key_end && key <= row_pos)) v[j] = kNegInf;
    }
  }
  float t[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) t[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
  for (int j = 0; j < 8; ++j) t[j] = fmaxf(t[j], t[j + 8]);
#pragma unroll
  for (int j = 0; j < 4; ++j) t[j] = fmaxf(t[j], t[j + 4]);
  const float cmax = fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3])) * c;   // c > 0
  const float mn = fmaxf(m, cmax);
  const float ms = (mn == kNegInf) ? 0.f : mn;
  float a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = fast_exp2(fmaf(v[j], c, -ms));
#pragma unroll
  for (int j = 8; j < 32; ++j) a[j & 7] += fast_exp2(fmaf(v[j], c, -ms));
  const float cs = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  l = fmaf(l, fast_exp2(m - ms), cs);
  m = mn;
}

// Score-pass accumulation for one key over window rows r0..r0+31:
// acc += 2^(c*z_r - off_r), rows above the key's causal limit skipped.
template <typename Params>
KVC_DEVINL void epi_score_chunk(const float *v, const float *off, int r0, int key, int P, const Params &p,
                                float *acc8) {
  if (key <= P) {     // prefix key (or the first window key): visible to every row
#pragma unroll
    for (int r = 0; r < 32; r += 4) {
      const float4 o4 = *reinterpret_cast<const float4 *>(off + r0 + r);
      acc8[(r >> 2) & 7] += fast_exp2(fmaf(v[r], p.c, -o4.x)) + fast_exp2(fmaf(v[r + 1], p.c, -o4.y)) +
                            (fast_exp2(fmaf(v[r + 2], p.c, -o4.z)) + fast_exp2(fmaf(v[r + 3], p.c, -o4.w)));
    }
  } else {            // window key: row r (window row r % w) sees it when key <= P + r % w
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int row = r0 + r;
      if (row < p.R && key <= P + row % p.w) acc8[r & 7] += fast_exp2(fmaf(v[r], p.c, -off[row]));
    }
  }
}

// --------------------------------------------------------------------------
// shared body: producer + MMA roles are identical for both passes, only the
// operand order of the MMA and the epilogue differ.
// --------------------------------------------------------------------------
template <int D, bool kScorePass>
__global__ void __launch_bounds__(kThreadsTC, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, TcParams p) {
  using L = TcLayout<D>;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = p.cu_seqlens[b], len = p.cu_seqlens[b + 1] - t0;
  const int key_begin = c * p.keys_per_chunk;
  if (key_begin >= len) return;
  const int key_end = min(len, key_begin + p.keys_per_chunk);
  const int n_tiles = (key_end - key_begin + kBN - 1) / kBN;
  const int P = len - p.w;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sq = smem + L::kOffQ;
  uint8_t *sk = smem + L::kOffK;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *full = bars, *empty = bars + kStages;
  uint64_t *acc_full = bars + 2 * kStages, *acc_empty = acc_full + 2, *q_full = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  int *cta_err = reinterpret_cast<int *>(smem + L::kOffMisc + 4);
  float *off = reinterpret_cast<float *>(smem + L::kOffOff);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], 4 * 32); }
    mbar_init(q_full, 4 * 32);
    *cta_err = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_k);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % kStages;
        if (!mbar_wait(&empty[s], ((t / kStages) & 1) ^ 1)) { *cta_err = 1; break; }
        mbar_expect_tx(&full[s], L::kKBytes);
        const int key0 = key_begin + t * kBN;
#pragma unroll
        for (int a = 0; a < L::kAtoms; ++a)
          tma_load_3d(sk + s * L::kKBytes + a * L::kAtomBytes, &tmap_k, &full[s], a * 64, h, t0 + key0);
        issued = t + 1;
      }
      // drain: every issued copy has landed before shared memory is released
      for (int t = max(0, issued - kStages); t < issued; ++t)
        if (!mbar_wait(&full[t % kStages], (t / kStages) & 1)) { *cta_err = 1; break; }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
      bool ok = mbar_wait(q_full, 0);
      int issued = 0;
      const uint32_t q_addr = smem_u32(sq), k_addr = smem_u32(sk);
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int s = t % kStages, buf = t & 1;
        if (!mbar_wait(&full[s], (t / kStages) & 1)) { ok = false; break; }
        if (!mbar_wait(&acc_empty[buf], ((t >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * 128;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * L::kAtomBytes + (ks & 3) * 32;
          const uint64_t dq = smem_desc_sw128(q_addr + koff);
          const uint64_t dk = smem_desc_sw128(k_addr + s * L::kKBytes + koff);
          if (kScorePass) umma_bf16(d_tmem, dk, dq, idesc, ks > 0);
          else umma_bf16(d_tmem, dq, dk, idesc, ks > 0);
        }
        umma_commit(&empty[s]);
        umma_commit(&acc_full[buf]);
        issued = t + 1;
      }
      if (!ok) *cta_err = 1;
      // drain: the last commit tracks every MMA issued by this thread
      if (issued > 0 && !mbar_wait(&acc_full[(issued - 1) & 1], ((issued - 1) >> 1) & 1)) *cta_err = 1;
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int et = threadIdx.x - kEpiWarp0 * 32;        // 0..127
    const int lane_base = 32 * (warp & 3);               // TMEM lanes this warp may access
    const int my_lane = lane_base + lane;                // row (stats) or key (score)
    if (kScorePass) {
      // merge the stats partials of every row into off_r = M + log2(L)
      const float2 *pp = p.part + (size_t)(b * p.n_kv + h) * p.n_chunks * kRows;
      const int nc = (len + p.keys_per_chunk - 1) / p.keys_per_chunk;
      for (int r = et; r < kRows; r += 128) {
        float o = kPosInf;
        if (r < p.R) {
          float M = kNegInf;
          for (int cc = 0; cc < nc; ++cc) M = fmaxf(M, pp[(size_t)cc * kRows + r].x);
          float Ls = 0.f;
          for (int cc = 0; cc < nc; ++cc) {
            const float2 v = pp[(size_t)cc * kRows + r];
            if (v.x != kNegInf) Ls += v.y * fast_exp2(v.x - M);
          }
          o = M + __log2f(Ls);
        }
        off[r] = o;
      }
    }
    stage_q<D>(sq, p, b, h, et, 128);
    mbar_arrive(q_full);
    if (kScorePass) asm volatile("bar.sync 1, 128;" ::: "memory");   // off[] visible to all epilogue warps

    float m = kNegInf, l = 0.f;
    const int row_pos = P + (my_lane % max(p.w, 1));     // stats pass: this thread's row position
    for (int t = 0; t < n_tiles; ++t) {
      const int buf = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (t >> 1) & 1))) { *cta_err = 1; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)lane_base << 16) + buf * 128;
      const int key0 = key_begin + t * kBN;
      // 32-column chunks, double-buffered: the load of chunk q+1 is in flight
      // while chunk q is reduced
      float va[32], vb[32];
      float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      tmem_ld32(taddr, va);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float *cur = (q & 1) ? vb : va;
        float *nxt = (q & 1) ? va : vb;
        if (q < 3) tmem_ld32(taddr + 32 * (q + 1), nxt);
        if (q == 3) {              // every column of this buffer has been read
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
        }
        if (!kScorePass) {
          epi_stats_chunk(cur, key0 + 32 * q, key_end, P, row_pos, p.c, m, l);
        } else {
          epi_score_chunk(cur, off, 32 * q, key0 + my_lane, P, p, acc8);
        }
        if (q < 3) tmem_wait_ld();
      }
      if (kScorePass) {
        const int key = key0 + my_lane;
        const float sum = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
        if (key < key_end) p.raw[(size_t)h * p.T_total + t0 + key] = sum;
      }
    }
    if (!kScorePass && my_lane < p.R)
      p.part[((size_t)(b * p.n_kv + h) * p.n_chunks + c) * kRows + my_lane] = make_float2(m, l);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem_base, 256); }
  if (threadIdx.x == 0 && *cta_err) set_err(p.err, 1);
}

// ---------------------------------------------------------- tensor maps
typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                     const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                     CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                     CUtensorMapFloatOOBfill);

PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

// K [T, n_kv, D] bf16 -> boxes of 64 d-elements x 1 head x 128 keys, 128-byte swizzle
bool make_k_map(CUtensorMap *map, const void *k, int T, int n_kv, int D) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)n_kv, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)n_kv * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kBN};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(k), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_tc(const ScoreArgs &a, cudaStream_t st) {
  CUtensorMap map;
  if (!make_k_map(&map, a.k, a.T_total, a.n_kv, D)) return cudaErrorInvalidValue;
  TcParams p;
  p.q_win = static_cast<const __nv_bfloat16 *>(a.q_win);
  p.cu_seqlens = a.cu_seqlens;
  p.part = a.part;
  p.raw = a.raw;
  p.err = a.err;
  p.n_h = a.n_h; p.n_kv = a.n_kv; p.G = a.n_h / a.n_kv; p.w = a.w; p.R = p.G * a.w;
  p.n_chunks = a.n_chunks; p.keys_per_chunk = a.keys_per_chunk; p.T_total = a.T_total;
  p.c = a.scale * kLog2e;
  const int smem = TcLayout<D>::kAlloc;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(score_tc_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
    return e;
  if ((e = cudaFuncSetAttribute(score_tc_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
    return e;
  dim3 grid(a.n_chunks, a.n_kv, a.n_seqs);
  score_tc_kernel<D, false><<<grid, kThreadsTC, smem, st>>>(map, p);
  if ((e = cudaGetLastError())) return e;
  score_tc_kernel<D, true><<<grid, kThreadsTC, smem, st>>>(map, p);
  return cudaGetLastError();
}

}  // namespace

int tc_keys_per_tile() { return kBN; }

cudaError_t score_window_tc(const ScoreArgs &a, cudaStream_t st) {
  if (a.d_h == 64) return launch_tc<64>(a, st);
  return launch_tc<128>(a, st);
}

}  // namespace kvc
