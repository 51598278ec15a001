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
// Warp roles (672 threads, one CTA per SM):
//   warps 0-3   load K tiles (128 keys x d_h) with 16-byte cp.async straight
//               into the 128-byte-swizzled K-major layout the MMA reads, a
//               5-stage ring.  Each loader thread's copies arrive on the
//               stage's "full" barrier by themselves when they land
//               (cp.async.mbarrier.arrive.noinc), so a loader only ever waits
//               for a free stage.  Rows past the sequence are zero-filled
//               (no read).  On this head-sliced pattern (256 B of every 2 KB
//               key row) 16-byte cp.async streams as fast as tensor-map
//               copies and leaves the ring fuller;
//   warp 4      owns tensor memory (512 columns: four 128-column accumulators)
//               and issues the MMAs from one thread;
//   warps 5-20  epilogue: four warps per TMEM lane quarter, each reading 32
//               of the 128 accumulator columns, software-pipelined over
//               16-column halves.
// The grid runs the KV heads fastest, so the CTAs resident together read the
// head slices of the same 2 KB key rows.
//
// When the whole grid fits on the GPU at once (one CTA per SM), both passes
// and the max-pool run in ONE cooperative launch: a CTA publishes its stats
// partial and runs the score pass over its own chunk in reverse tile order --
// the last kStages tiles of the stats pass are still in its shared-memory
// ring and are not loaded again, the rest mostly come from L2.  Its loaders
// and MMA thread start at once (the products need no offsets) while its
// epilogue waits on a per-(sequence, head) arrival counter for the other key
// chunks of its head and merges the offsets.  After a second counter it pools
// its chunk (halo from the neighbours' raw scores).  This saves a launch, the window-block staging, the tensor-memory
// allocation and the separate pool kernel, and a third of the second K pass.
// Otherwise the two passes are separate launches and the pool kernel follows.
// Every wait is bounded; a wait that gives up sets the device error word and
// the CTA stops waiting (results are then flagged invalid, never a hang).
#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kBN = 128;          // keys per tile
constexpr int kRows = 128;        // window-block rows (padded)
constexpr int kStages = 5;        // K ring depth
constexpr int kAccBufs = 4;       // TMEM accumulators
constexpr int kLoadWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kEpiWarp0 = 5;
constexpr int kEpiWarps = 16;
constexpr int kColBlocks = kEpiWarps / 4;   // 32-column blocks per lane quarter
constexpr int kThreadsTC = (kLoadWarps + 1 + kEpiWarps) * 32;
constexpr int kXch = 8;           // column-block exchange slots (score pass)

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
  // score pass: [kXch][kColBlocks - 1][128] partial row sums; stats pass:
  // m and l of every row for column blocks 1..kColBlocks-1
  static constexpr int kOffXch = kOffOff + kRows * 4;
  static constexpr int kBytes = kOffXch + kXch * (kColBlocks - 1) * kBN * 4;
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
  float *scores;   // fused path: pooled output
  int *sync;       // fused path: kCtrPerUnit counters per (sequence, KV head), zero between calls
  int *err;
  // fused selection and gather (idx == nullptr: the launch stops after the pool)
  int32_t *idx;                 // [n_kv, total_budget]
  const int32_t *cu_budget;
  const uint8_t *v;             // V [T, n_kv, d_h]
  uint8_t *k_out, *v_out;       // compact caches [total_budget, n_kv, d_h]
  int *hist;                    // kHistInts per (sequence, KV head), zero between calls
  int *cnt;                     // 2 per (sequence, KV head, key chunk)
  int total_budget, budget;
  int n_h, n_kv, G, w, R, n_chunks, keys_per_chunk, T_total, pool_r;
  float c;   // scale * log2(e)
};

// fused selection: counters and per-(sequence, head) radix histograms
constexpr int kCtrPerUnit = 8;     // stats, raw, depart, radix levels 1-3, two spare
constexpr int kH1 = 4096, kH2 = 4096, kH3 = 256;
constexpr int kHistInts = kH1 + kH2 + kH3;
constexpr int kCntInts = 2 + kH3;  // per (sequence, head, chunk): keys above the 24-bit prefix, spare, level-3 bins
// keys of one chunk held in shared memory: the K ring (kStages tiles of kBN x d_h bf16) as uint32

// Shared-memory objects of one CTA.
struct TcSmem {
  uint8_t *sq, *sk;
  uint64_t *full, *empty, *acc_full, *acc_empty, *q_full, *xch_full;
  uint32_t *tmem_slot;
  volatile int *cta_err;
  float *off, *xch;
};

// The CTA's share of the work: key chunk c of KV head h of sequence b.
struct TcWork {
  int b, h, c, t0, len, P, key_begin, key_end, n_tiles;
};

// Q_win rows r = g * w + i of (b, h) into the 128-byte-swizzled K-major tile
// with cp.async (all chunks in flight at once); rows >= R are zero-filled.
// The caller makes their completion arrive on q_full.
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

constexpr float kSlack = 8.f;   // stats pass: log2 headroom before the running max moves

// Stats-pass reduction of 16 logits of one window row (keys k0..k0+15):
// running sum of 2^(c*z - m).  The reference m only moves, by warp vote, when
// a logit exceeds it by more than kSlack (so every term stays <= 2^kSlack and
// the rescale of l is rare and warp-uniform).  Masked keys (beyond the chunk
// end or the row's causal limit) contribute nothing.
KVC_DEVINL void epi_stats16(uint32_t (&r)[16], int k0, int key_end, int P, int row_pos, float c, float &m, float &l) {
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
  if (!(k0 + 15 <= P && k0 + 16 <= key_end)) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int key = k0 + j;
      if (!(key < key_end && key <= row_pos)) v[j] = kNegInf;
    }
  }
  float t[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) t[j] = fmaxf(v[j], v[j + 8]);
#pragma unroll
  for (int j = 0; j < 4; ++j) t[j] = fmaxf(t[j], t[j + 4]);
  const float cmax = fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3])) * c;   // c > 0
  const bool need = cmax > m + kSlack;
  if (__any_sync(0xffffffffu, need)) {
    const float mn = need ? cmax : m;
    if (need) l *= (m == kNegInf) ? 0.f : fast_exp2(m - mn);
    m = mn;
  }
  const float ms = (m == kNegInf) ? 0.f : m;
  float a[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) a[j] = fast_exp2(fmaf(v[j], c, -ms));
#pragma unroll
  for (int j = 4; j < 16; ++j) a[j & 3] += fast_exp2(fmaf(v[j], c, -ms));
  l += (a[0] + a[1]) + (a[2] + a[3]);
}

// Score-pass accumulation for one key over window rows r0..r0+15:
// returns the sum of 2^(c*z_r - off_r); rows above the key's causal limit are
// skipped.
KVC_DEVINL float epi_score16(uint32_t (&rr)[16], const float *off, int r0, int key, int P, const TcParams &p) {
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  if (key <= P) {     // prefix key (or the first window key): visible to every row
#pragma unroll
    for (int r = 0; r < 16; r += 4) {
      const float4 o4 = *reinterpret_cast<const float4 *>(off + r0 + r);
      a[(r >> 2) & 3] += (fast_exp2(fmaf(__uint_as_float(rr[r]), p.c, -o4.x)) +
                          fast_exp2(fmaf(__uint_as_float(rr[r + 1]), p.c, -o4.y))) +
                         (fast_exp2(fmaf(__uint_as_float(rr[r + 2]), p.c, -o4.z)) +
                          fast_exp2(fmaf(__uint_as_float(rr[r + 3]), p.c, -o4.w)));
    }
  } else {            // window key: row r (window row r % w) sees it when key <= P + r % w
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int row = r0 + r;
      if (row < p.R && key <= P + row % p.w) a[r & 3] += fast_exp2(fmaf(__uint_as_float(rr[r]), p.c, -off[row]));
    }
  }
  return (a[0] + a[1]) + (a[2] + a[3]);
}

template <int D>
KVC_DEVINL TcSmem carve_smem(uint8_t *smem_raw) {
  using L = TcLayout<D>;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TcSmem sm;
  sm.sq = smem + L::kOffQ;
  sm.sk = smem + L::kOffK;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  sm.full = bars;
  sm.empty = bars + kStages;
  sm.acc_full = bars + 2 * kStages;
  sm.acc_empty = sm.acc_full + kAccBufs;
  sm.q_full = sm.acc_empty + kAccBufs;
  sm.xch_full = sm.q_full + 1;
  sm.tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  sm.cta_err = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
  sm.off = reinterpret_cast<float *>(smem + L::kOffOff);
  sm.xch = reinterpret_cast<float *>(smem + L::kOffXch);
  return sm;
}

// (Re)initialise the pipeline barriers (one thread; the caller fences and syncs).
KVC_DEVINL void init_pass_barriers(const TcSmem &sm, bool reinit) {
  auto init = [&](uint64_t *bar, uint32_t count) {
    if (reinit) asm volatile("mbarrier.inval.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
    mbar_init(bar, count);
  };
  for (int s = 0; s < kStages; ++s) { init(&sm.full[s], kLoadWarps * 32); init(&sm.empty[s], 1); }
  for (int s = 0; s < kAccBufs; ++s) { init(&sm.acc_full[s], 1); init(&sm.acc_empty[s], kEpiWarps); }
  for (int s = 0; s < kXch; ++s) init(&sm.xch_full[s], 4 * (kColBlocks - 1));
}

KVC_DEVINL int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One thread: wait (bounded) until n CTAs have announced themselves on *ctr.
KVC_DEVINL bool wait_count(const int *ctr, int n) {
  const uint64_t t0 = global_ns();
  while (ld_acquire(ctr) < n) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(64);
  }
  return true;
}

// One thread: announce this CTA on *ctr (its earlier writes first).
KVC_DEVINL void arrive(int *ctr) {
  __threadfence();
  atomicAdd(ctr, 1);
}

// One thread: announce this CTA on *ctr, then wait (bounded) until n CTAs did.
KVC_DEVINL bool arrive_and_wait(int *ctr, int n) {
  arrive(ctr);
  return wait_count(ctr, n);
}

// One pass over the CTA's key chunk, all warp roles.
//   kScorePass = false: stats pass, writes the (m, l) partial of every row.
//   kScorePass = true:  score pass, writes the raw scores of the chunk; off[]
//                       must hold off_r.  With rev, tiles run last to first
//                       and the last min(kStages, n_tiles) tiles are taken as
//                       already resident in the ring (left by the stats pass).
template <int D, bool kScorePass>
KVC_DEVINL void tc_pass(const TcParams &p, const TcSmem &sm, const TcWork &wk, uint32_t tmem_base, bool rev) {
  using L = TcLayout<D>;
  const int warp = warp_id(), lane = lane_id();
  const int n = wk.n_tiles;
  const int resident = rev ? min(kStages, n) : 0;
  auto tile_of = [&](int j) { return rev ? n - 1 - j : j; };
  if (warp < kLoadWarps) {
    // ------------------------------------------------------------ K loaders
    const int lt = threadIdx.x;                      // 0..127
    constexpr int kChunks = kBN * D / 8;             // 16-byte chunks per tile
    const uint8_t *kbase = reinterpret_cast<const uint8_t *>(p.k);
    for (int j = resident; j < n; ++j) {
      const int t = tile_of(j), s = t % kStages;
      // use u of slot s in this pass (in rev mode use 0 is the resident
      // tile): wait until the MMA of use u - 1 released the slot, i.e. for
      // phase u - 1 of its "empty" barrier (u = 0: nothing to wait for)
      const int u = j / kStages;
      if (!*sm.cta_err && !mbar_wait(&sm.empty[s], (u - 1) & 1)) *sm.cta_err = 1;
      const int key0 = wk.key_begin + t * kBN;
      uint8_t *dst = sm.sk + s * L::kKBytes;
#pragma unroll 4
      for (int e = lt; e < kChunks; e += kLoadWarps * 32) {
        const int row = e / (D / 8), ch = e % (D / 8);
        const int atom = ch >> 3, c16 = ch & 7;
        const bool valid = key0 + row < wk.key_end;
        const uint8_t *src = kbase + ((size_t)(wk.t0 + (valid ? key0 + row : 0)) * p.n_kv + wk.h) * (D * 2) + ch * 16;
        cp_async16(dst + atom * L::kAtomBytes + row * 128 + ((c16 ^ (row & 7)) << 4), src, valid);
      }
      cp_async_arrive_noinc(&sm.full[s]);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
      const uint32_t q_addr = smem_u32(sm.sq), k_addr = smem_u32(sm.sk);
      int issued = 0;
      for (int j = 0; j < n && !*sm.cta_err; ++j) {
        const int t = tile_of(j), s = t % kStages, buf = j % kAccBufs;
        const int u = j / kStages;
        if (j >= resident) {
          const int load_no = rev ? u - 1 : u;
          if (!mbar_wait(&sm.full[s], load_no & 1)) { *sm.cta_err = 1; break; }
        }
        if (!mbar_wait(&sm.acc_empty[buf], ((j / kAccBufs) & 1) ^ 1)) { *sm.cta_err = 1; break; }
        // the stage was written through the generic proxy (cp.async); order
        // those writes, now visible to this thread, before the tensor core's reads
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
        // free the stage only if a later load of this pass waits for it
        if (j + kStages < n) umma_commit(&sm.empty[s]);
        umma_commit(&sm.acc_full[buf]);
        issued = j + 1;
      }
      // drain: the last commit tracks every MMA issued by this thread
      if (issued > 0 && !mbar_wait(&sm.acc_full[(issued - 1) % kAccBufs], ((issued - 1) / kAccBufs) & 1))
        *sm.cta_err = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;                 // 0..15
    const int quarter = warp & 3;                    // TMEM lanes this warp may access
    const int cb = ew >> 2;                          // which 32 accumulator columns
    const int my_lane = 32 * quarter + lane;         // row (stats) or key (score)
    float m = kNegInf, l = 0.f;
    const int row_pos = wk.P + (my_lane % max(p.w, 1));   // stats pass: this thread's row position
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quarter) << 16) + cb * 32;
    auto wait_full = [&](int j) {
      const bool got = *sm.cta_err ? true : mbar_wait(&sm.acc_full[j % kAccBufs], (j / kAccBufs) & 1);
      if (!__all_sync(0xffffffffu, got) && lane == 0) *sm.cta_err = 1;
      tc_fence_after();
    };
    // software pipeline over 16-column halves: the TMEM load of the next half
    // is in flight while the current one is reduced
    uint32_t ra[16], rb[16];
    if (n > 0) {
      wait_full(0);
      tmem_ld16(t_lane, ra);
      tmem_wait_ld16(ra);
    }
    for (int j = 0; j < n; ++j) {
      const int buf = j % kAccBufs;
      const int key0 = wk.key_begin + tile_of(j) * kBN;
      tmem_ld16(t_lane + buf * 128 + 16, rb);
      float sum = 0.f;
      if (!kScorePass) epi_stats16(ra, key0 + cb * 32, wk.key_end, wk.P, row_pos, p.c, m, l);
      else sum = epi_score16(ra, sm.off, cb * 32, key0 + my_lane, wk.P, p);
      tmem_wait_ld16(rb);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);   // this warp's columns of the tile are read
      if (j + 1 < n) {
        wait_full(j + 1);
        tmem_ld16(t_lane + ((j + 1) % kAccBufs) * 128, ra);
      }
      if (!kScorePass) epi_stats16(rb, key0 + cb * 32 + 16, wk.key_end, wk.P, row_pos, p.c, m, l);
      else sum += epi_score16(rb, sm.off, cb * 32 + 16, key0 + my_lane, wk.P, p);
      if (kScorePass) {
        const int slot = j % kXch;
        float *xs = sm.xch + (size_t)slot * (kColBlocks - 1) * kBN;
        const int key = key0 + my_lane;
        if (cb > 0) {
          xs[(cb - 1) * kBN + my_lane] = sum;
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.xch_full[slot]);
        } else {
          const bool ok = *sm.cta_err ? true : mbar_wait(&sm.xch_full[slot], (j / kXch) & 1);
          if (!__all_sync(0xffffffffu, ok) && lane == 0) *sm.cta_err = 1;
          float tot = sum;
#pragma unroll
          for (int q = 0; q < kColBlocks - 1; ++q) tot += xs[q * kBN + my_lane];
          if (key < wk.key_end) p.raw[(size_t)wk.h * p.T_total + wk.t0 + key] = tot;
        }
      }
      if (j + 1 < n) tmem_wait_ld16(ra);
    }
    if (!kScorePass) {
      // merge the column blocks of every row, then publish the partial
      float *xm = sm.xch, *xl = sm.xch + (kColBlocks - 1) * kRows;
      if (cb > 0) { xm[(cb - 1) * kRows + my_lane] = m; xl[(cb - 1) * kRows + my_lane] = l; }
      asm volatile("bar.sync 1, %0;" :: "n"(kEpiWarps * 32) : "memory");
      if (cb == 0 && my_lane < p.R) {
        float mn = m;
#pragma unroll
        for (int q = 0; q < kColBlocks - 1; ++q) mn = fmaxf(mn, xm[q * kRows + my_lane]);
        float ls = 0.f;
        if (mn != kNegInf) {
          ls = l * fast_exp2(m - mn);
#pragma unroll
          for (int q = 0; q < kColBlocks - 1; ++q) ls += xl[q * kRows + my_lane] * fast_exp2(xm[q * kRows + my_lane] - mn);
        }
        p.part[((size_t)(wk.b * p.n_kv + wk.h) * p.n_chunks + wk.c) * kRows + my_lane] = make_float2(mn, ls);
      }
    }
  }
}

// (M, L) <- merge of two running (max, sum of 2^(x - max)) pairs
KVC_DEVINL void merge_ml(float &M, float &L, float m, float l) {
  const float mn = fmaxf(M, m);
  if (mn == kNegInf) return;
  L = L * fast_exp2(M - mn) + l * fast_exp2(m - mn);
  M = mn;
}

// Epilogue threads: off_r = M + log2(L) of every row from the stats partials
// of all key chunks of the head (read through L2: other CTAs wrote them).
// Four threads per row fold every fourth chunk with independent loads in
// flight, then combine by shuffle, so the merge costs about one L2 round trip.
KVC_DEVINL void merge_offsets(const TcParams &p, const TcSmem &sm, const TcWork &wk) {
  static_assert(kEpiWarps * 32 == 4 * kRows, "four epilogue threads per row");
  const int et = threadIdx.x - kEpiWarp0 * 32;
  const int r = et >> 2, q = et & 3;
  const float2 *pp = p.part + (size_t)(wk.b * p.n_kv + wk.h) * p.n_chunks * kRows + r;
  const int nc = (wk.len + p.keys_per_chunk - 1) / p.keys_per_chunk;
  float M = kNegInf, Ls = 0.f;
  if (r < p.R) {
    for (int cc = q; cc < nc; cc += 16) {
      float2 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = cc + 4 * u < nc ? __ldcg(pp + (size_t)(cc + 4 * u) * kRows) : make_float2(kNegInf, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) merge_ml(M, Ls, v[u].x, v[u].y);
    }
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, M, o), l2 = __shfl_xor_sync(0xffffffffu, Ls, o);
    merge_ml(M, Ls, m2, l2);
  }
  if (q == 0) sm.off[r] = (r < p.R) ? M + __log2f(Ls) : kPosInf;
  asm volatile("bar.sync 1, %0;" :: "n"(kEpiWarps * 32) : "memory");
}

KVC_DEVINL bool setup_work(const TcParams &p, TcWork &wk) {
  wk.h = blockIdx.x; wk.c = blockIdx.y; wk.b = blockIdx.z;
  wk.t0 = p.cu_seqlens[wk.b];
  wk.len = p.cu_seqlens[wk.b + 1] - wk.t0;
  wk.key_begin = wk.c * p.keys_per_chunk;
  if (wk.key_begin >= wk.len) return false;
  wk.key_end = min(wk.len, wk.key_begin + p.keys_per_chunk);
  wk.n_tiles = (wk.key_end - wk.key_begin + kBN - 1) / kBN;
  wk.P = wk.len - p.w;
  return true;
}

// Barriers, tensor memory and the window block (loaders stage it with
// cp.async; the MMA thread waits for it before its first MMA).
template <int D>
KVC_DEVINL uint32_t cta_setup(const TcParams &p, const TcSmem &sm, const TcWork &wk) {
  const int warp = warp_id();
  if (threadIdx.x == 0) {
    init_pass_barriers(sm, false);
    mbar_init(sm.q_full, kLoadWarps * 32);
    *sm.cta_err = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) { tmem_alloc(sm.tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp < kLoadWarps) {
    stage_q_async<D>(sm.sq, p, wk.b, wk.h, threadIdx.x, kLoadWarps * 32);
    cp_async_arrive_noinc(sm.q_full);
  } else if (warp == kMmaWarp && lane_id() == 0) {
    if (!mbar_wait(sm.q_full, 0)) *sm.cta_err = 1;
  }
  return *sm.tmem_slot;
}

KVC_DEVINL void cta_teardown(const TcParams &p, const TcSmem &sm, uint32_t tmem_base) {
  tc_fence_before();
  __syncthreads();
  if (warp_id() == kMmaWarp) { tc_fence_after(); tmem_dealloc(tmem_base, 512); }
  if (threadIdx.x == 0 && *sm.cta_err) atomicCAS(p.err, 0, 1);
}

// ----------------------------------------------------------- fused selection
// Order-preserving 32-bit key of a float (larger float, larger key).
KVC_DEVINL uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of one int per thread (all kThreadsTC
// threads call it); returns this thread's exclusive prefix, *total the sum.
KVC_DEVINL int block_exclusive_scan(int v, int *scr, int *total) {
  constexpr int kWarps = kThreadsTC / 32;
  const int lane = lane_id(), warp = warp_id();
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scr[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < kWarps ? scr[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) scr[32 + lane] = s;      // inclusive warp totals
  }
  __syncthreads();
  const int base = warp > 0 ? scr[32 + warp - 1] : 0;
  *total = scr[32 + kWarps - 1];
  __syncthreads();
  return base + x - v;
}

// Scanning the bins of a global histogram from the top, the bin where the
// running count reaches `need` (1 <= need <= total count) and the count in
// the bins above it.  All threads call it and get the result.  Thread t holds
// the 8 bins [nbins - 8 (t + 1), nbins - 8 t) in registers (two 16-byte
// loads issued together), so the search costs one L2 round trip.
KVC_DEVINL void find_bucket_from_top(const int *hist, int nbins, int need, int *scr, int &bin, int &above) {
  const int t = threadIdx.x;
  const bool mine = t < nbins / 8;
  const int lo = nbins - 8 * (t + 1);
  int h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (mine) {
    const int4 a = __ldcg(reinterpret_cast<const int4 *>(hist + lo));
    const int4 b = __ldcg(reinterpret_cast<const int4 *>(hist + lo) + 1);
    h[0] = a.x; h[1] = a.y; h[2] = a.z; h[3] = a.w; h[4] = b.x; h[5] = b.y; h[6] = b.z; h[7] = b.w;
  }
  const int sum = ((h[0] + h[1]) + (h[2] + h[3])) + ((h[4] + h[5]) + (h[6] + h[7]));
  int total;
  const int before = block_exclusive_scan(sum, scr, &total);
  if (mine && before < need && before + sum >= need) {
    int run = before;
#pragma unroll
    for (int q = 7; q >= 0; --q) {
      if (run + h[q] >= need) { scr[64] = lo + q; scr[65] = run; break; }
      run += h[q];
    }
  }
  __syncthreads();
  bin = scr[64];
  above = scr[65];
  __syncthreads();
}

// After the pool, the CTAs of one (sequence, head) pick its budgeted top-k
// (pooled prefix scores, lowest position first among equal scores, window
// always kept, ascending positions) and gather the kept K/V rows.
//   A three-level radix select on the order keys (12, 12 and 8 bits) finds
//   the k-th largest key T and how many keys equal to T are taken: every CTA
//   adds its histogram of the candidates to a per-head histogram in the
//   workspace, waits on a counter, and reads the bucket holding the k-th key.
//   (A single log-scale bucket with a candidate exchange was tried: pooled
//   scores crowd into few buckets, so it was slower.)  With its level-3
//   histogram every CTA also publishes its own 256 level-3 bins and its count
//   of keys above the 24-bit prefix; once T is known, the keys > T and == T
//   of every earlier chunk follow from those records without another round.
//   A CTA writes its kept positions at (keys > T in earlier chunks) + (equal
//   keys taken in earlier chunks) + its own rank, which gives the ascending
//   order and the lowest-position tie rule across chunks.  The CTA gathers the
//   rows it placed; the CTA holding position P writes and gathers the window.
template <int D>
KVC_DEVINL void fused_select_gather(const TcParams &p, const TcSmem &sm, const TcWork &wk, int *ctr, int nc,
                                    const uint32_t *keys) {
  const int tid = threadIdx.x;
  const int P = wk.P, w = p.w;
  const int kept = min(p.budget, wk.len);
  const int k_sel = kept - w;                       // prefix tokens kept (the host checked budget >= w)
  const int j0 = wk.key_begin;
  const int n_my = max(0, min(wk.key_end, P) - j0);  // prefix keys of this chunk
  const bool all = k_sel >= P;                      // the whole prefix is kept
  int *scr = reinterpret_cast<int *>(sm.xch);        // scan scratch
  int *sh = reinterpret_cast<int *>(sm.sq);          // shared histogram (the window block is free)
  int *hist = p.hist + (size_t)(wk.b * p.n_kv + wk.h) * kHistInts;
  int *cnt = p.cnt + (size_t)(wk.b * p.n_kv + wk.h) * p.n_chunks * kCntInts;

  uint32_t T = 0;
  int need = 0;                                     // keys equal to T to take over the head
  int base_gt = 0, base_eq = 0;                     // keys > T and == T in the earlier chunks
  if (!all && k_sel > 0) {
    uint32_t fixed = 0;                              // key bits fixed by the earlier levels
    need = k_sel;
    int *above24 = scr + 96;                         // this chunk's keys above the 24-bit prefix (level 3)
    for (int lvl = 0; lvl < 3; ++lvl) {
      const int nbins = lvl < 2 ? 4096 : 256;
      const int shift = lvl == 0 ? 20 : (lvl == 1 ? 8 : 0);
      int *gh = hist + (lvl == 0 ? 0 : (lvl == 1 ? kH1 : kH1 + kH2));
      for (int b = tid; b < nbins; b += kThreadsTC) sh[b] = 0;
      if (tid == 0) *above24 = 0;
      __syncthreads();
      int my_above = 0;
      for (int i = tid; i < n_my; i += kThreadsTC) {
        const uint32_t kk = keys[i];
        const bool cand = lvl == 0 || (lvl == 1 ? (kk >> 20) == fixed : (kk >> 8) == fixed);
        if (cand) atomicAdd(&sh[(kk >> shift) & (nbins - 1)], 1);
        if (lvl == 2) my_above += (kk >> 8) > fixed;
      }
      if (lvl == 2 && my_above) atomicAdd(above24, my_above);
      __syncthreads();
      for (int b = tid; b < nbins; b += kThreadsTC)
        if (sh[b]) atomicAdd(&gh[b], sh[b]);
      if (lvl == 2) {
        // this chunk's level-3 record, read by the later chunks of the head
        // after the level-3 counter (so no separate round for the counts)
        int *rec = cnt + (size_t)wk.c * kCntInts;
        for (int b = tid; b < kH3; b += kThreadsTC) rec[2 + b] = sh[b];
        if (tid == 0) rec[0] = *above24;
      }
      __syncthreads();
      if (tid == 0 && !arrive_and_wait(&ctr[3 + lvl], nc)) *sm.cta_err = 1;
      __syncthreads();
      int bin, above;
      find_bucket_from_top(gh, nbins, need, scr, bin, above);
      need -= above;
      fixed = lvl == 0 ? (uint32_t)bin : (fixed << (lvl == 1 ? 12 : 8)) | (uint32_t)bin;
      if (lvl == 0) {
        // keys above the level-1 bucket are kept whatever T turns out to be:
        // bring their V rows (not read by the scoring) into L2 for the gather
        const size_t head_bytes = (size_t)D * 2;
        for (int i = tid; i < n_my; i += kThreadsTC)
          if ((keys[i] >> 20) > fixed) {
            const uint8_t *row = p.v + ((size_t)(wk.t0 + j0 + i) * p.n_kv + wk.h) * head_bytes;
#pragma unroll
            for (size_t o = 0; o < head_bytes; o += 128)
              asm volatile("prefetch.global.L2 [%0];" :: "l"(row + o));
          }
      }
    }
    T = fixed;
    // ---- keys > T and == T in the earlier chunks, from their level-3
    // records: keys above the 24-bit prefix plus the bins above / at T's bin
    const int tb = (int)(T & 255u);
    int gt = 0, eq = 0;
    for (int e = tid; e < wk.c * kCntInts; e += kThreadsTC) {
      const int f = e % kCntInts;
      if (f == 1) continue;
      const int v = __ldcg(cnt + e);
      if (f == 0) gt += v;
      else if (f - 2 > tb) gt += v;
      else if (f - 2 == tb) eq += v;
    }
    block_exclusive_scan(gt, scr, &base_gt);
    block_exclusive_scan(eq, scr, &base_eq);
  }

  // ---- this chunk's output offset and its share of the equal keys
  int off = 0, eq_take = 0;
  if (all) {
    off = j0;                                       // the kept prefix is the identity
  } else if (k_sel > 0) {
    off = base_gt + min(need, base_eq);
    eq_take = max(0, need - base_eq);
  }

  // ---- ordered compaction: thread t walks a contiguous run of the chunk
  const int total = p.total_budget;
  const int cb = p.cu_budget[wk.b];
  int32_t *idx = p.idx + (size_t)wk.h * total + cb;
  int n_sel = 0;
  if (all || k_sel > 0) {
    const int run = (n_my + kThreadsTC - 1) / kThreadsTC;
    const int i0 = min(n_my, tid * run), i1 = min(n_my, i0 + run);
    int my_gt = 0, my_eq = 0;
    if (!all)
      for (int i = i0; i < i1; ++i) { my_gt += keys[i] > T; my_eq += keys[i] == T; }
    int tot_gt, tot_eq;
    int gt_b = block_exclusive_scan(all ? i1 - i0 : my_gt, scr, &tot_gt);
    int eq_b = block_exclusive_scan(my_eq, scr, &tot_eq);
    // (slot checks only matter if a bounded wait gave up and the counts are inconsistent)
    auto put = [&](int slot, int pos) { if (slot >= 0 && slot < k_sel) idx[slot] = pos; };
    for (int i = i0; i < i1; ++i) {
      const uint32_t kk = keys[i];
      if (all || kk > T) {
        put(off + gt_b + min(eq_b, eq_take), j0 + i);
        ++gt_b;
      } else if (kk == T) {
        if (eq_b < eq_take) put(off + gt_b + eq_b, j0 + i);
        ++eq_b;
      }
    }
    n_sel = max(0, min(tot_gt + min(tot_eq, eq_take), k_sel - off));
  }
  // the window: positions P .. len-1 at slots k_sel .. kept-1, by the CTA holding P
  const bool win_owner = wk.key_begin <= P && P < wk.key_end;
  if (win_owner)
    for (int t = tid; t < w; t += kThreadsTC) idx[k_sel + t] = P + t;
  __syncthreads();

  // ---- gather the rows this CTA placed (their slots are contiguous)
  constexpr int kVec = D * 2 / 16;                  // 16-byte vectors per head row (bf16)
  const size_t head_bytes = (size_t)D * 2;
  auto gather_slots = [&](int s0, int n) {
    for (int e = tid; e < n * kVec; e += kThreadsTC) {
      const int slot = s0 + e / kVec, c = e % kVec;
      const int pos = __ldcg(idx + slot);
      const size_t dst = ((size_t)(cb + slot) * p.n_kv + wk.h) * head_bytes + (size_t)c * 16;
      uint4 kv_k = make_uint4(0, 0, 0, 0), kv_v = make_uint4(0, 0, 0, 0);
      if (pos >= 0 && pos < wk.len) {            // a position outside the sequence gives a zero row
        const size_t src = ((size_t)(wk.t0 + pos) * p.n_kv + wk.h) * head_bytes + (size_t)c * 16;
        kv_k = ld_stream16(reinterpret_cast<const uint8_t *>(p.k) + src);
        kv_v = ld_stream16(p.v + src);
      }
      st_stream16(p.k_out + dst, kv_k);
      st_stream16(p.v_out + dst, kv_v);
    }
  };
  if (off >= 0) gather_slots(off, n_sel);
  if (win_owner) gather_slots(k_sel, w);
}

// One pass per launch (the grid does not fit on the GPU at once).
template <int D, bool kScorePass>
__global__ void __launch_bounds__(kThreadsTC, 1)
score_tc_kernel(TcParams p) {
  TcWork wk;
  if (!setup_work(p, wk)) return;
  extern __shared__ uint8_t smem_raw[];
  const TcSmem sm = carve_smem<D>(smem_raw);
  const uint32_t tmem_base = cta_setup<D>(p, sm, wk);
  if (kScorePass && warp_id() >= kEpiWarp0) merge_offsets(p, sm, wk);
  tc_pass<D, kScorePass>(p, sm, wk, tmem_base, false);
  cta_teardown(p, sm, tmem_base);
}

// Both passes and the pool in one cooperative launch.
template <int D>
__global__ void __launch_bounds__(kThreadsTC, 1)
score_fused_kernel(TcParams p) {
  allow_dependents();
  TcWork wk;
  if (!setup_work(p, wk)) return;
  extern __shared__ uint8_t smem_raw[];
  const TcSmem sm = carve_smem<D>(smem_raw);
  const uint32_t tmem_base = cta_setup<D>(p, sm, wk);
  const int nc = (wk.len + p.keys_per_chunk - 1) / p.keys_per_chunk;
  int *ctr = p.sync + (size_t)(wk.b * p.n_kv + wk.h) * kCtrPerUnit;

  tc_pass<D, false>(p, sm, wk, tmem_base, false);

  // announce this chunk's stats partial; the loaders and the MMA thread start
  // the score pass on the resident tiles at once (its products do not depend
  // on the offsets), while the epilogue waits until every chunk of this head
  // has published its partial and merges the offsets
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    arrive(&ctr[0]);
    init_pass_barriers(sm, true);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  if (warp_id() >= kEpiWarp0) {
    if (threadIdx.x == kEpiWarp0 * 32 && !wait_count(&ctr[0], nc)) *sm.cta_err = 1;
    asm volatile("bar.sync 1, %0;" :: "n"(kEpiWarps * 32) : "memory");
    merge_offsets(p, sm, wk);
  }

  tc_pass<D, true>(p, sm, wk, tmem_base, true);

  // pool the chunk once every chunk of this head has written its raw scores
  __syncthreads();
  if (threadIdx.x == 0) arrive(&ctr[1]);
  {
    const float *src = p.raw + (size_t)wk.h * p.T_total + wk.t0;
    float *dst = p.scores + (size_t)wk.h * p.T_total + wk.t0;
    uint32_t *keys = reinterpret_cast<uint32_t *>(sm.sk);   // the K ring is no longer needed
    const int r = p.pool_r;
    // stage the chunk's raw scores and the halo in the (free) window-block
    // area with coalesced loads; neighbours outside the prefix read as -inf.
    // The chunk's own scores are staged while the other chunks finish; the
    // halo after the counter.
    float *stage = reinterpret_cast<float *>(sm.sq);
    const int own_end = min(wk.key_end, wk.P);
    const int s_lo = wk.key_begin - r, s_n = own_end + r - s_lo;
    const bool staged = s_n <= TcLayout<D>::kQBytes / 4;
    if (staged)
      for (int j = wk.key_begin + threadIdx.x; j < own_end; j += kThreadsTC) stage[j - s_lo] = __ldcg(src + j);
    __syncthreads();
    if (threadIdx.x == 0 && !wait_count(&ctr[1], nc)) *sm.cta_err = 1;
    __syncthreads();
    if (staged && own_end > wk.key_begin) {          // (a chunk inside the window pools nothing)
      for (int e = threadIdx.x; e < 2 * r; e += kThreadsTC) {
        const int j = e < r ? s_lo + e : own_end + (e - r);
        stage[j - s_lo] = (j >= 0 && j < wk.P) ? __ldcg(src + j) : kNegInf;
      }
      __syncthreads();
    }
    for (int j = wk.key_begin + threadIdx.x; j < wk.key_end; j += kThreadsTC) {
      float v = kPosInf;
      if (j < wk.P) {
        if (staged) {
          const float *c = stage + (j - s_lo);
          v = c[0];
          for (int q = 1; q <= r; ++q) v = fmaxf(v, fmaxf(c[-q], c[q]));
        } else {
          const int lo = max(0, j - r), hi = min(wk.P - 1, j + r);
          v = __ldcg(src + lo);
          for (int q = lo + 1; q <= hi; ++q) v = fmaxf(v, __ldcg(src + q));
        }
        if (p.idx) keys[j - wk.key_begin] = order_key(v);
      }
      dst[j] = v;
    }
  }
  if (p.idx) {
    __syncthreads();
    fused_select_gather<D>(p, sm, wk, ctr, nc, reinterpret_cast<const uint32_t *>(sm.sk));
  }

  // the last CTA of this head to leave resets the counters (and histograms)
  // for the next call
  __syncthreads();
  if (threadIdx.x == 0) sm.off[0] = __int_as_float(atomicAdd(&ctr[2], 1) == nc - 1 ? 1 : 0);
  __syncthreads();
  if (__float_as_int(sm.off[0])) {
    if (p.idx) {
      int *hist = p.hist + (size_t)(wk.b * p.n_kv + wk.h) * kHistInts;
      for (int e = threadIdx.x; e < kHistInts; e += kThreadsTC) hist[e] = 0;
    }
    if (threadIdx.x < kCtrPerUnit) ctr[threadIdx.x] = 0;
  }
  cta_teardown(p, sm, tmem_base);
}

template <int D>
cudaError_t launch_tc(const ScoreArgs &a, cudaStream_t st) {
  TcParams p;
  p.q_win = static_cast<const __nv_bfloat16 *>(a.q_win);
  p.k = static_cast<const __nv_bfloat16 *>(a.k);
  p.cu_seqlens = a.cu_seqlens;
  p.part = a.part;
  p.raw = a.raw;
  p.scores = a.scores;
  p.sync = a.sync;
  p.err = a.err;
  p.idx = a.fused ? a.idx : nullptr;
  p.cu_budget = a.cu_budget;
  p.v = static_cast<const uint8_t *>(a.v);
  p.k_out = static_cast<uint8_t *>(a.k_out);
  p.v_out = static_cast<uint8_t *>(a.v_out);
  p.hist = a.hist;
  p.cnt = a.cnt;
  p.total_budget = a.total_budget;
  p.budget = a.budget;
  p.n_h = a.n_h; p.n_kv = a.n_kv; p.G = a.n_h / a.n_kv; p.w = a.w; p.R = p.G * a.w;
  p.n_chunks = a.n_chunks; p.keys_per_chunk = a.keys_per_chunk; p.T_total = a.T_total;
  p.pool_r = a.pool_k / 2;
  p.c = a.scale * kLog2e;
  const int smem = TcLayout<D>::kAlloc;
  dim3 grid(a.n_kv, a.n_chunks, a.n_seqs);
  cudaError_t e;
  if (a.fused) {
    if ((e = ensure_smem_limit((const void *)score_fused_kernel<D>, smem))) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreadsTC);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, score_fused_kernel<D>, p);
  }
  if ((e = ensure_smem_limit((const void *)score_tc_kernel<D, false>, smem))) return e;
  if ((e = ensure_smem_limit((const void *)score_tc_kernel<D, true>, smem))) return e;
  score_tc_kernel<D, false><<<grid, kThreadsTC, smem, st>>>(p);
  count_launch();
  if ((e = cudaGetLastError())) return e;
  score_tc_kernel<D, true><<<grid, kThreadsTC, smem, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

int tc_keys_per_tile() { return kBN; }
int tc_counters_per_unit() { return kCtrPerUnit; }
int tc_hist_ints() { return kHistInts; }
int tc_count_ints() { return kCntInts; }
int tc_select_max_keys(int d_h) { return kStages * kBN * d_h * 2 / 4; }

cudaError_t score_window_tc(const ScoreArgs &a, cudaStream_t st) {
  if (a.d_h == 64) return launch_tc<64>(a, st);
  return launch_tc<128>(a, st);
}

}  // namespace kvc
