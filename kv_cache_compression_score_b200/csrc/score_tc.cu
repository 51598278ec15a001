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
//   score pass:  D[key][row] = K[key] . Q_win[row]   (M = 128 keys, N = 128 rows)
//                one epilogue thread per TMEM lane = key sums 2^(y - off_r)
//                over the rows, off_r = m_r + log2(l_r) merged from the
//                stats partials.
//
// Warp roles (416 threads, one CTA per SM):
//   warps 0-3   load K tiles (128 keys x d_h) with 16-byte cp.async straight
//               into the 128-byte-swizzled K-major layout the MMA reads, a
//               5-stage ring; 16-byte cp.async streams these strided head rows
//               faster than tensor-map copies with 128-byte boxes.  Rows past
//               the sequence are zero-filled (no read);
//   warp 4      owns tensor memory (512 columns: four 128-column accumulators)
//               and issues the MMAs from one thread;
//   warps 5-12  epilogue: two warps per TMEM lane quarter, each reading half
//               of the accumulator columns.
// Every wait is bounded; a wait that gives up sets the device error word and
// the CTA stops waiting (results are then flagged invalid, never a hang).
#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kBN = 128;          // keys per tile
constexpr int kRows = 128;        // window-block rows (padded)
constexpr int kStages = 5;        // K ring depth
constexpr int kLag = kStages - 1; // tiles in flight per loader thread
constexpr int kAccBufs = 4;       // TMEM accumulators
constexpr int kLoadWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kEpiWarp0 = 5;
constexpr int kEpiWarps = 8;
constexpr int kThreadsTC = (kLoadWarps + 1 + kEpiWarps) * 32;
constexpr int kXch = 8;           // half-column exchange slots (score pass)

template <int D>
struct TcLayout {
  static constexpr int kQBytes = kRows * D * 2;              // window block
  static constexpr int kKBytes = kBN * D * 2;                // one K tile
  static constexpr int kAtomBytes = 128 * 128;               // 128 rows x 128 B
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffK + kStages * kKBytes;
  static constexpr int kBarCount = 2 * kStages + 2 * kAccBufs + 1 + kXch;
  static constexpr int kOffMisc = kOffBar + 256;
  static constexpr int kOffOff = kOffMisc + 16;              // off_r[128] (score pass)
  static constexpr int kOffXch = kOffOff + kRows * 4;        // [kXch][128] (score) / m,l halves (stats)
  static constexpr int kBytes = kOffXch + kXch * kBN * 4;
  static constexpr int kAlloc = kBytes + 1024;               // room to align the base to 1 KB
  static_assert(kBarCount * 8 <= 256, "barrier area");
  static_assert(kOffOff % 16 == 0, "off[] is read as float4");
  static_assert(kOffK % 1024 == 0 && kKBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

struct TcParams {
  const __nv_bfloat16 *q_win;
  const __nv_bfloat16 *k;
  const int *cu_seqlens;
  float2 *part;
  float *raw;
  int *err;
  int n_h, n_kv, G, w, R, n_chunks, keys_per_chunk, T_total;
  float c;   // scale * log2(e)
};

// 16-byte cp.async, zero-filled (no global read) when !valid
KVC_DEVINL void cp_async16(void *dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               :: "r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0) : "memory");
}

// Q_win rows r = g * w + i of (b, h) into the 128-byte-swizzled K-major tile
// with cp.async (all chunks in flight at once); rows >= R are zero-filled.
// Completion, publication to the tensor core and the q_full arrive are done
// by the caller together with its first K tiles.
template <int D>
KVC_DEVINL void stage_q_async(uint8_t *sq, const TcParams &p, int b, int h, int tid, int nthreads) {
  constexpr int kChunks = D / 8;   // 16-byte chunks per row
#pragma unroll 4
  for (int e = tid; e < kRows * kChunks; e += nthreads) {
    const int r = e / kChunks, ch = e % kChunks;
    const int atom = ch >> 3, c16 = ch & 7;
    const bool valid = r < p.R;
    const int g = valid ? r / p.w : 0, i = valid ? r % p.w : 0;
    const __nv_bfloat16 *src = p.q_win + ((size_t)(b * p.w + i) * p.n_h + (size_t)h * p.G + g) * D + ch * 8;
    cp_async16(sq + atom * TcLayout<D>::kAtomBytes + r * 128 + ((c16 ^ (r & 7)) << 4), src, valid);
  }
}

// Stats-pass reduction of 32 logits of one window row (keys k0..k0+31):
// online max / sum of 2^(c*z - m); masked keys (beyond the chunk end or the
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
// acc += 2^(c*z_r - off_r); rows above the key's causal limit are skipped.
KVC_DEVINL void epi_score_chunk(const float *v, const float *off, int r0, int key, int P, const TcParams &p,
                                float *acc8) {
  if (key <= P) {     // prefix key (or the first window key): visible to every row
#pragma unroll
    for (int r = 0; r < 32; r += 4) {
      const float4 o4 = *reinterpret_cast<const float4 *>(off + r0 + r);
      acc8[(r >> 2) & 7] += (fast_exp2(fmaf(v[r], p.c, -o4.x)) + fast_exp2(fmaf(v[r + 1], p.c, -o4.y))) +
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

template <int D, bool kScorePass>
__global__ void __launch_bounds__(kThreadsTC, 1)
score_tc_kernel(TcParams p) {
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
  uint64_t *acc_full = bars + 2 * kStages, *acc_empty = acc_full + kAccBufs;
  uint64_t *q_full = acc_empty + kAccBufs;
  uint64_t *xch_full = q_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *cta_err = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
  float *off = reinterpret_cast<float *>(smem + L::kOffOff);
  float *xch = reinterpret_cast<float *>(smem + L::kOffXch);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], kLoadWarps * 32); mbar_init(&empty[s], 1); }
    for (int s = 0; s < kAccBufs; ++s) { mbar_init(&acc_full[s], 1); mbar_init(&acc_empty[s], kEpiWarps); }
    mbar_init(q_full, kLoadWarps * 32);
    for (int s = 0; s < kXch; ++s) mbar_init(&xch_full[s], 4);
    *cta_err = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kLoadWarps) {
    // ------------------------------------------------------------ K loaders
    const int lt = threadIdx.x;                      // 0..127
    stage_q_async<D>(sq, p, b, h, lt, kLoadWarps * 32);
    asm volatile("cp.async.commit_group;" ::: "memory");
    bool q_published = false;
    constexpr int kChunks = kBN * D / 8;             // 16-byte chunks per tile
    const uint8_t *kbase = reinterpret_cast<const uint8_t *>(p.k);
    for (int t = 0; t < n_tiles + kLag; ++t) {
      if (t < n_tiles) {
        const int s = t % kStages;
        if (!*cta_err && !mbar_wait(&empty[s], ((t / kStages) & 1) ^ 1)) *cta_err = 1;
        const int key0 = key_begin + t * kBN;
        uint8_t *dst = sk + s * L::kKBytes;
#pragma unroll 4
        for (int e = lt; e < kChunks; e += kLoadWarps * 32) {
          const int row = e / (D / 8), ch = e % (D / 8);
          const int atom = ch >> 3, c16 = ch & 7;
          const bool valid = key0 + row < key_end;
          const uint8_t *src = kbase + ((size_t)(t0 + (valid ? key0 + row : 0)) * p.n_kv + h) * (D * 2) + ch * 16;
          cp_async16(dst + atom * L::kAtomBytes + row * 128 + ((c16 ^ (row & 7)) << 4), src, valid);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      if (t >= kLag) {
        // the window block (group 0) and tile t - kLag have landed for this
        // thread: publish them to the tensor core
        asm volatile("cp.async.wait_group %0;" :: "n"(kLag) : "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (!q_published) { mbar_arrive(q_full); q_published = true; }
        mbar_arrive(&full[(t - kLag) % kStages]);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
      const uint32_t q_addr = smem_u32(sq), k_addr = smem_u32(sk);
      if (!mbar_wait(q_full, 0)) *cta_err = 1;
      int issued = 0;
      for (int t = 0; t < n_tiles && !*cta_err; ++t) {
        const int s = t % kStages, buf = t % kAccBufs;
        if (!mbar_wait(&full[s], (t / kStages) & 1)) { *cta_err = 1; break; }
        if (!mbar_wait(&acc_empty[buf], ((t / kAccBufs) & 1) ^ 1)) { *cta_err = 1; break; }
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
      // drain: the last commit tracks every MMA issued by this thread
      if (issued > 0 && !mbar_wait(&acc_full[(issued - 1) % kAccBufs], ((issued - 1) / kAccBufs) & 1)) *cta_err = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;                 // 0..7
    const int et = threadIdx.x - kEpiWarp0 * 32;     // 0..255
    const int quarter = warp & 3;                    // TMEM lanes this warp may access
    const int half = ew >> 2;                        // which 64 accumulator columns
    const int my_lane = 32 * quarter + lane;         // row (stats) or key (score)
    if (kScorePass) {
      // merge the stats partials of every row into off_r = M + log2(L)
      const float2 *pp = p.part + (size_t)(b * p.n_kv + h) * p.n_chunks * kRows;
      const int nc = (len + p.keys_per_chunk - 1) / p.keys_per_chunk;
      for (int r = et; r < kRows; r += kEpiWarps * 32) {
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
      asm volatile("bar.sync 1, %0;" :: "n"(kEpiWarps * 32) : "memory");
    }

    float m = kNegInf, l = 0.f;
    const int row_pos = P + (my_lane % max(p.w, 1));   // stats pass: this thread's row position
    for (int t = 0; t < n_tiles; ++t) {
      const int buf = t % kAccBufs;
      const bool got = *cta_err ? true : mbar_wait(&acc_full[buf], (t / kAccBufs) & 1);
      if (!__all_sync(0xffffffffu, got) && lane == 0) *cta_err = 1;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * quarter) << 16) + buf * 128 + half * 64;
      const int key0 = key_begin + t * kBN;
      float va[32], vb[32];
      float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      tmem_ld32(taddr, va);
      tmem_wait_ld();
      tmem_ld32(taddr + 32, vb);
      if (!kScorePass) epi_stats_chunk(va, key0 + half * 64, key_end, P, row_pos, p.c, m, l);
      else epi_score_chunk(va, off, half * 64, key0 + my_lane, P, p, acc8);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);    // this warp's columns are read
      if (!kScorePass) epi_stats_chunk(vb, key0 + half * 64 + 32, key_end, P, row_pos, p.c, m, l);
      else epi_score_chunk(vb, off, half * 64 + 32, key0 + my_lane, P, p, acc8);
      if (kScorePass) {
        const float sum = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
        const int slot = t % kXch;
        const int key = key0 + my_lane;
        if (half == 1) {
          xch[slot * kBN + my_lane] = sum;
          __syncwarp();
          if (lane == 0) mbar_arrive(&xch_full[slot]);
        } else {
          const bool ok = *cta_err ? true : mbar_wait(&xch_full[slot], (t / kXch) & 1);
          if (!__all_sync(0xffffffffu, ok) && lane == 0) *cta_err = 1;
          if (key < key_end) p.raw[(size_t)h * p.T_total + t0 + key] = sum + xch[slot * kBN + my_lane];
        }
      }
    }
    if (!kScorePass) {
      // merge the two column halves of every row, then publish the partial
      float *xm = xch, *xl = xch + kRows;
      if (half == 1) { xm[my_lane] = m; xl[my_lane] = l; }
      asm volatile("bar.sync 1, %0;" :: "n"(kEpiWarps * 32) : "memory");
      if (half == 0 && my_lane < p.R) {
        const float m2 = xm[my_lane], l2 = xl[my_lane];
        const float mn = fmaxf(m, m2);
        float ls = 0.f;
        if (mn != kNegInf) ls = l * fast_exp2(m - mn) + l2 * fast_exp2(m2 - mn);
        p.part[((size_t)(b * p.n_kv + h) * p.n_chunks + c) * kRows + my_lane] = make_float2(mn, ls);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) { tc_fence_after(); tmem_dealloc(tmem_base, 512); }
  if (threadIdx.x == 0 && *cta_err) atomicCAS(p.err, 0, 1);
}

template <int D>
cudaError_t launch_tc(const ScoreArgs &a, cudaStream_t st) {
  TcParams p;
  p.q_win = static_cast<const __nv_bfloat16 *>(a.q_win);
  p.k = static_cast<const __nv_bfloat16 *>(a.k);
  p.cu_seqlens = a.cu_seqlens;
  p.part = a.part;
  p.raw = a.raw;
  p.err = a.err;
  p.n_h = a.n_h; p.n_kv = a.n_kv; p.G = a.n_h / a.n_kv; p.w = a.w; p.R = p.G * a.w;
  p.n_chunks = a.n_chunks; p.keys_per_chunk = a.keys_per_chunk; p.T_total = a.T_total;
  p.c = a.scale * kLog2e;
  const int smem = TcLayout<D>::kAlloc;
  cudaError_t e;
  if ((e = ensure_smem_limit((const void *)score_tc_kernel<D, false>, smem)))
    return e;
  if ((e = ensure_smem_limit((const void *)score_tc_kernel<D, true>, smem)))
    return e;
  dim3 grid(a.n_chunks, a.n_kv, a.n_seqs);
  score_tc_kernel<D, false><<<grid, kThreadsTC, smem, st>>>(p);
  if ((e = cudaGetLastError())) return e;
  score_tc_kernel<D, true><<<grid, kThreadsTC, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

int tc_keys_per_tile() { return kBN; }

cudaError_t score_window_tc(const ScoreArgs &a, cudaStream_t st) {
  if (a.d_h == 64) return launch_tc<64>(a, st);
  return launch_tc<128>(a, st);
}

}  // namespace kvc
