// xKV cross-layer factorisation and selective reconstruction ("xKV -
// Compression de Cache KV Inter-couche par Extraction de Vecteurs Singuliers
// Alignes", gist.science 2503.18893, technical summary section 2.2
// "Factorisation Inter-couche (CLF)" and section 2.3 "Reconstruction
// Selective (SR)").
//
// For every KV head h the keys of a window of W consecutive layers,
// concatenated along the feature axis, X_h = [K_1[:, h] | ... | K_W[:, h]]
// (S x F, F = W * d_h), get the rank-r factorisation X_h ~ A_h Vt_h with
// Vt_h = V^T spanning the top-r right singular subspace and the shared token
// basis A_h = X_h V; selective reconstruction rebuilds only chosen rows of one
// layer, K_l[idx] ~ A_h[idx] Vt_h[:, l d_h : (l + 1) d_h].
//
// The top-r right singular subspace of X_h is the top-r eigenspace of the Gram
// matrix G_h = X_h^T X_h.  It is found by subspace iteration from the caller's
// start basis: Y = G_h V, then V <- Y L^-T with C = Y^T Y = L L^T (Cholesky-QR;
// C, L and L^-1 in float64).
//
// Kernels (the iteration is a chain of three launches per step):
//   xkv_gram    G_h on the tensor cores (mma.sync m16n8k16, bf16 in, fp32
//               accumulate, both operands through ldmatrix.trans from
//               [token][feature] tiles); upper 64 x 64 tiles only, mirrored;
//               the token axis split over CTAs, reduced with atomics;
//   xkv_gv      32 rows of Y = G_h V per CTA (4 x CPT register blocks), and
//               those rows' share of C = Y^T Y (float64 atomics);
//   xkv_chol    one CTA per head: Cholesky of C and M = L^-T in float64;
//               leaves C zero for the next step;
//   xkv_apply   32 rows of V = Y M per CTA (float64 products); the last step
//               also writes Vt;
//   xkv_project_tc A_h = X_h V on the tensor cores (V split into two bf16
//               terms), a run of 128-token tiles per CTA;
//   xkv_rebuild_tc rows idx of layer l: A_h[idx] Vt_h[:, layer block] on the
//               tensor cores, rounded to bf16 (nearest even).
#include <algorithm>

#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kGramTile = 64;     // output tile of the Gram kernel
constexpr int kGramS = 64;        // tokens per pipeline stage
constexpr int kGramStages = 4;    // cp.async ring depth of the Gram kernel
constexpr int kGramPitch = 72;    // bf16 per padded smem row (144 bytes: the 8 rows of an ldmatrix hit distinct banks)
constexpr int kRowsPerCta = 32;   // xkv_gv / xkv_apply
constexpr int kGvK = 64;          // xkv_gv: rows k of G and V per pipeline step

struct XkArgs {
  const __nv_bfloat16 *k[kXkvMaxW];   // the W layers' key caches [S, n_kv, d_h]
  int S, n_kv, d, W, F, r;
  int tok_per_split;
  float *gram;                    // [n_kv, F, F]
  const float *v_in;              // [n_kv, F, r]: the basis this step multiplies
  float *y;                       // [n_kv, F, r]
  double *c;                      // [n_kv, r, r] (lower triangle used)
  double *m;                      // [n_kv, r, r] upper triangular L^-T
  float *v_out;                   // [n_kv, F, r]
  float *blocks;                  // Vt [n_kv, r, F] (written by the last apply)
  void *basis;                    // A [n_kv, S, r], float32 or bf16
  bool basis_bf16;
};

// X_h element (token s, feature f)
KVC_DEVINL const __nv_bfloat16 *xptr(const XkArgs &a, int h, int s, int f) {
  const int l = f / a.d, j = f - l * a.d;
  return a.k[l] + ((size_t)s * a.n_kv + h) * a.d + j;
}

// ------------------------------------------------------------------ Gram
constexpr int kGramSmem = 2 * kGramStages * kGramS * kGramPitch * 2;

__global__ void __launch_bounds__(128) xkv_gram(XkArgs a) {
  extern __shared__ __align__(16) uint8_t xk_gram_smem[];
  auto si = reinterpret_cast<__nv_bfloat16 (*)[kGramS][kGramPitch]>(xk_gram_smem);
  auto sj = reinterpret_cast<__nv_bfloat16 (*)[kGramS][kGramPitch]>(xk_gram_smem + kGramSmem / 2);
  // upper-triangular tile pair (ti <= tj) from blockIdx.x
  const int nt = a.F / kGramTile;
  int ti = 0, rem = blockIdx.x;
  while (rem >= nt - ti) { rem -= nt - ti; ++ti; }
  const int tj = ti + rem;
  const int h = blockIdx.y;
  const int s0 = blockIdx.z * a.tok_per_split, s1 = min(a.S, s0 + a.tok_per_split);
  if (s0 >= s1) return;
  const int fi0 = ti * kGramTile, fj0 = tj * kGramTile;
  const int warp = warp_id(), lane = lane_id();
  const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;      // this warp's 32 x 32 sub-tile
  const int g = lane >> 2, t = lane & 3, lr = lane & 7, li = lane >> 3;
  float acc[2][4][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
  // one step: kGramS tokens x 64 features of each operand, in 16-byte pieces
  // (8 features; d_h % 8 == 0 keeps a piece inside one layer)
  auto load = [&](int buf, int sb) {
    for (int e = threadIdx.x; e < 2 * kGramS * 8; e += 128) {
      const int which = e / (kGramS * 8), rr = e % (kGramS * 8), row = rr / 8, c8 = rr % 8;
      const int s = sb + row;
      const bool ok = s < s1;
      const int f = (which ? fj0 : fi0) + 8 * c8;
      __nv_bfloat16 *dst = which ? &sj[buf][row][8 * c8] : &si[buf][row][8 * c8];
      cp_async16(dst, xptr(a, h, ok ? s : s0, f), ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // ring of kGramStages stages: stage st is in buffer st % kGramStages; one
  // commit group per stage (empty past the end), so that waiting until at
  // most kGramStages - 1 groups are pending means stage st has landed
  const int n_steps = (s1 - s0 + kGramS - 1) / kGramS;
  for (int q = 0; q < kGramStages - 1; ++q) {
    if (q < n_steps) load(q, s0 + q * kGramS);
    else asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int st = 0; st < n_steps; ++st) {
    const int buf = st % kGramStages;
    const int nx = st + kGramStages - 1;
    if (nx < n_steps) load(nx % kGramStages, s0 + nx * kGramS);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group %0;" :: "n"(kGramStages - 1) : "memory");
    __syncthreads();
#pragma unroll
    for (int ks = 0; ks < kGramS / 16; ++ks) {
      // A = X^T (m = feature i, k = token): 8x8 pieces (i 0-7, s 0-7), (i 8-15, s 0-7), (i 0-7, s 8-15), (i 8-15, s 8-15)
      uint32_t af[2][4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
        ldsm_x4_t(smem_u32(&si[buf][16 * ks + lr + (li >> 1) * 8][wm + 16 * mi + (li & 1) * 8]), af[mi]);
      // B = X (k = token, n = feature j): pieces (s 0-7, j 0-7), (s 8-15, j 0-7), (s 0-7, j 8-15), (s 8-15, j 8-15)
      uint32_t bfr[2][4];
#pragma unroll
      for (int nj = 0; nj < 2; ++nj)
        ldsm_x4_t(smem_u32(&sj[buf][16 * ks + lr + (li & 1) * 8][wn + 16 * nj + (li >> 1) * 8]), bfr[nj]);
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int nj = 0; nj < 2; ++nj) {
          mma_bf16(acc[mi][2 * nj], af[mi], bfr[nj][0], bfr[nj][1]);
          mma_bf16(acc[mi][2 * nj + 1], af[mi], bfr[nj][2], bfr[nj][3]);
        }
    }
    __syncthreads();
  }
  float *G = a.gram + (size_t)h * a.F * a.F;
  const bool mirror = ti != tj;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int n8 = 0; n8 < 4; ++n8)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = fi0 + wm + 16 * mi + g + (q >> 1) * 8, j = fj0 + wn + 8 * n8 + 2 * t + (q & 1);
        atomicAdd(&G[(size_t)i * a.F + j], acc[mi][n8][q]);
        if (mirror) atomicAdd(&G[(size_t)j * a.F + i], acc[mi][n8][q]);
      }
}

// ------------------------------------------------------- Y = G V, C += Y^T Y
// 128 threads: rg = tid / 16 owns rows 4 rg .. 4 rg + 3 of the CTA's 32 rows,
// cg = tid % 16 owns columns cg * CPT ..; G is symmetric, so the CTA streams
// rows k of G (its own 32 columns) next to rows k of V.
template <int R>
__global__ void __launch_bounds__(128) xkv_gv(XkArgs a) {
  constexpr int CPT = R / 16;
  extern __shared__ __align__(16) float xk_gv_smem[];
  float *sg = xk_gv_smem;                               // [2][kGvK][32]
  float *sv = xk_gv_smem + 2 * kGvK * kRowsPerCta;      // [2][kGvK][R]
  const int h = blockIdx.y, i0 = blockIdx.x * kRowsPerCta, F = a.F;
  const float *G = a.gram + (size_t)h * F * F;
  const float *V = a.v_in + (size_t)h * F * R;
  const int tid = threadIdx.x, rg = tid / 16, cg = tid % 16;
  auto load = [&](int buf, int k0) {
    for (int e = tid; e < kGvK * (kRowsPerCta / 4); e += 128) {   // G rows k, 32 columns
      const int kk = e / (kRowsPerCta / 4), c4 = e % (kRowsPerCta / 4);
      cp_async16(sg + (buf * kGvK + kk) * kRowsPerCta + 4 * c4, G + (size_t)(k0 + kk) * F + i0 + 4 * c4, true);
    }
    for (int e = tid; e < kGvK * (R / 4); e += 128) {             // V rows k
      const int kk = e / (R / 4), c4 = e % (R / 4);
      cp_async16(sv + (buf * kGvK + kk) * R + 4 * c4, V + (size_t)(k0 + kk) * R + 4 * c4, true);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[4][CPT];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[q][c] = 0.f;
  const int n_steps = F / kGvK;
  load(0, 0);
  for (int st = 0; st < n_steps; ++st) {
    const int buf = st & 1;
    if (st + 1 < n_steps) {
      load(buf ^ 1, (st + 1) * kGvK);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const float *g_t = sg + buf * kGvK * kRowsPerCta + 4 * rg;
    const float *v_t = sv + buf * kGvK * R + cg * CPT;
#pragma unroll 8
    for (int kk = 0; kk < kGvK; ++kk) {
      const float4 g4 = *reinterpret_cast<const float4 *>(g_t + kk * kRowsPerCta);
      float vv[CPT];
      if constexpr (CPT == 4) {
        const float4 v4 = *reinterpret_cast<const float4 *>(v_t + kk * R);
        vv[0] = v4.x; vv[1] = v4.y; vv[2] = v4.z; vv[3] = v4.w;
      } else if constexpr (CPT == 2) {
        const float2 v2 = *reinterpret_cast<const float2 *>(v_t + kk * R);
        vv[0] = v2.x; vv[1] = v2.y;
      } else {
#pragma unroll
        for (int c = 0; c < CPT; ++c) vv[c] = v_t[kk * R + c];
      }
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        acc[0][c] = fmaf(g4.x, vv[c], acc[0][c]);
        acc[1][c] = fmaf(g4.y, vv[c], acc[1][c]);
        acc[2][c] = fmaf(g4.z, vv[c], acc[2][c]);
        acc[3][c] = fmaf(g4.w, vv[c], acc[3][c]);
      }
    }
    __syncthreads();
  }
  // Y rows to global and to shared memory (over the finished V stages)
  float *sy = sv;                                       // [32][R]
  float *Y = a.y + (size_t)h * F * R;
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int row = 4 * rg + q, col = cg * CPT + c;
      sy[row * R + col] = acc[q][c];
      Y[(size_t)(i0 + row) * R + col] = acc[q][c];
    }
  __syncthreads();
  double *C = a.c + (size_t)h * R * R;
  for (int e = tid; e < R * R; e += 128) {
    const int p = e / R, q = e % R;
    if (q > p) continue;
    double s = 0.0;
#pragma unroll 8
    for (int row = 0; row < kRowsPerCta; ++row) s = fma((double)sy[row * R + p], (double)sy[row * R + q], s);
    atomicAdd(&C[e], s);
  }
}

// ------------------------------------------------ Cholesky and M = L^-T
// 1 / sqrt(x) in float64: the float32 reciprocal square root as a seed (about
// 22 correct bits), then two Newton-Raphson steps y <- y (3 - x y^2) / 2, each
// doubling the correct bits (22 -> 44 -> past the 53 of a double).  Values
// outside the float32 range take the plain quotient.
KVC_DEVINL double rsqrt_newton(double x) {
  if (!(x > 1e-37 && x < 1e37)) return 1.0 / sqrt(x);
  double y = (double)rsqrtf((float)x);
  y = y * fma(-0.5 * x * y, y, 1.5);
  y = y * fma(-0.5 * x * y, y, 1.5);
  return y;
}

// One CTA per head, 512 threads, one barrier per column and one per four
// rows of the inverse.  Column c of L is written from the unscaled working
// copy in the same phase as the rank-1 update of the trailing block (thread
// (tp, tq) updates rows tp, tp + 16, .. and columns tq, tq + 32, ..), so no
// phase reads what it writes.  L^-1 is formed four rows at a time: 8 threads
// per column sum the terms of the rows above the block, and one of them
// finishes the 4 x 4 triangular block; it is stored transposed as M.  Pivots
// are inverted once (by the thread that finished them) and multiplied.
template <int R>
__global__ void __launch_bounds__(512) xkv_chol(XkArgs a) {
  constexpr int LP = R + 1;
  extern __shared__ __align__(16) double xk_chol_smem[];
  double *A = xk_chol_smem;          // [R][LP] working copy, updated in place
  double *L = A + R * LP;            // [R][LP] strictly lower part of the factor
  double *X = L + R * LP;            // [R][LP] L^-1
  double *dinv = X + R * LP;         // [R]: 1 / L[c][c]
  const int h = blockIdx.x, tid = threadIdx.x;
  double *C = a.c + (size_t)h * R * R;
  for (int e = tid; e < R * R; e += 512) {
    const int p = e / R, q = e % R;
    A[p * LP + q] = q <= p ? C[e] : 0.0;
    X[p * LP + q] = 0.0;
    C[e] = 0.0;                      // ready for the next step's atomics
  }
  __syncthreads();
  double tr = 0.0;
  for (int p = 0; p < R; ++p) tr += A[p * LP + p];
  // a pivot below this floor (a rank-deficient Y) is raised to it
  const double floor_piv = fmax(tr, 1e-300) * 1e-30;
  if (tid == 0) dinv[0] = rsqrt_newton(fmax(A[0], floor_piv));
  __syncthreads();
  const int tp = tid >> 5, tq = tid & 31;
  constexpr int NP = (R + 15) / 16, NQ = (R + 31) / 32;
  for (int c = 0; c < R; ++c) {
    const double inv = dinv[c];
    if (c + 1 + tid < R) L[(c + 1 + tid) * LP + c] = A[(c + 1 + tid) * LP + c] * inv;
    // the column-c values this thread needs, loaded before any update
    double lq[NQ], lp[NP];
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      const int q = c + 1 + tq + 32 * qi;
      lq[qi] = q < R ? A[q * LP + c] : 0.0;
    }
#pragma unroll
    for (int pi = 0; pi < NP; ++pi) {
      const int p = c + 1 + tp + 16 * pi;
      lp[pi] = p < R ? A[p * LP + c] * inv * inv : 0.0;
    }
#pragma unroll
    for (int pi = 0; pi < NP; ++pi) {
      const int p = c + 1 + tp + 16 * pi;
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        const int q = c + 1 + tq + 32 * qi;
        if (p < R && q <= p) A[p * LP + q] = fma(-lp[pi], lq[qi], A[p * LP + q]);
      }
    }
    // thread 0 owns (c + 1, c + 1): no other thread writes it in this phase
    if (tid == 0 && c + 1 < R) dinv[c + 1] = rsqrt_newton(fmax(A[(c + 1) * LP + c + 1], floor_piv));
    __syncthreads();
  }
  // X = L^-1 (lower), rows i0 .. i0 + 3 per step; thread group (j, part)
  const int j = tid >> 3, part = tid & 7;
  for (int i0 = 0; i0 < R; i0 += 4) {
    double s[4] = {0.0, 0.0, 0.0, 0.0};
    if (j < i0)
      for (int k = j + part; k < i0; k += 8) {
        const double xk = X[k * LP + j];
#pragma unroll
        for (int r = 0; r < 4; ++r) s[r] = fma(L[(i0 + r) * LP + k], xk, s[r]);
      }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      s[r] += __shfl_xor_sync(0xffffffffu, s[r], 1);
      s[r] += __shfl_xor_sync(0xffffffffu, s[r], 2);
      s[r] += __shfl_xor_sync(0xffffffffu, s[r], 4);
    }
    if (part == 0 && j < i0 + 4) {
      double xb[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = i0 + r;
        double v = 0.0;
        if (j == i) {
          v = dinv[i];
        } else if (j < i) {
          double sum = s[r];
          for (int k = max(j, i0); k < i; ++k) sum = fma(L[i * LP + k], xb[k - i0], sum);
          v = -sum * dinv[i];
        }
        xb[r] = v;
        X[i * LP + j] = v;
      }
    }
    __syncthreads();
  }
  double *M = a.m + (size_t)h * R * R;
  for (int e = tid; e < R * R; e += 512) {
    const int k = e / R, c = e % R;
    M[e] = X[c * LP + k];            // M[k][c] = (L^-1)[c][k], zero for k > c
  }
}

// ---------------------------------------------------------- V = Y M
template <int R>
__global__ void __launch_bounds__(128) xkv_apply(XkArgs a, int write_blocks) {
  extern __shared__ __align__(16) double xk_apply_smem[];
  double *sm = xk_apply_smem;                                   // [R][R]
  float *sy = reinterpret_cast<float *>(sm + R * R);            // [32][R + 1]
  const int h = blockIdx.y, i0 = blockIdx.x * kRowsPerCta, F = a.F, tid = threadIdx.x;
  const double *M = a.m + (size_t)h * R * R;
  const float *Y = a.y + (size_t)h * F * R;
  for (int e = tid; e < R * R; e += 128) sm[e] = M[e];
  for (int e = tid; e < kRowsPerCta * R; e += 128) sy[(e / R) * (R + 1) + e % R] = Y[(size_t)i0 * R + e];
  __syncthreads();
  const int row = tid / 4, c0 = tid % 4;
  float *Vo = a.v_out + (size_t)h * F * R;
  for (int c = c0; c < R; c += 4) {
    double s = 0.0;
    for (int k = 0; k <= c; ++k) s = fma((double)sy[row * (R + 1) + k], sm[k * R + c], s);
    const float v = (float)s;
    Vo[(size_t)(i0 + row) * R + c] = v;
    if (write_blocks) a.blocks[((size_t)h * R + c) * F + i0 + row] = v;
  }
}

// ------------------------------------------------------------ A = X V
// Tensor cores: A (tokens x r) = X (tokens x F, bf16, exact) times V (F x r)
// with V = Vt^T split into two bf16 terms (v = hi + lo, |v - hi - lo| <=
// 2^-17 |v|), mma.sync m16n8k16 with fp32 accumulation.  A CTA stages both
// terms of Vt ([r][F], F contiguous) once and walks a contiguous run of
// 128-token tiles; each tile's X streams in 64-feature chunks through two
// cp.async buffers.  Warp w owns tokens 16w .. 16w + 15 of a tile and all r
// columns.
constexpr int kPjTok = 128;       // tokens per tile
constexpr int kPjK = 64;          // features per chunk
constexpr int kPjXP = kPjK + 8;   // bf16 pitch of an X chunk row (144 B)

template <int R>
__global__ void __launch_bounds__(256) xkv_project_tc(XkArgs a, int tiles_per_cta) {
  extern __shared__ __align__(16) uint8_t xk_proj_smem[];
  const int F = a.F, VP = F + 8;                       // bf16 pitch of a Vt row
  __nv_bfloat16 *vhi = reinterpret_cast<__nv_bfloat16 *>(xk_proj_smem);   // [R][VP]
  __nv_bfloat16 *vlo = vhi + R * VP;
  __nv_bfloat16 *xs = vlo + R * VP;                                       // [2][kPjTok][kPjXP]
  const int h = blockIdx.y, warp = warp_id(), lane = lane_id();
  const int n_tiles = (a.S + kPjTok - 1) / kPjTok;
  const int tile0 = blockIdx.x * tiles_per_cta, tile1 = min(n_tiles, tile0 + tiles_per_cta);
  if (tile0 >= tile1) return;
  const int n_chunks = F / kPjK, n_items = (tile1 - tile0) * n_chunks;
  auto load = [&](int item, int buf) {
    const int tile = tile0 + item / n_chunks, f0 = (item % n_chunks) * kPjK;
    for (int e = threadIdx.x; e < kPjTok * (kPjK / 8); e += 256) {
      const int row = e / (kPjK / 8), c8 = e % (kPjK / 8), s = tile * kPjTok + row;
      const bool ok = s < a.S;
      cp_async16(xs + ((size_t)buf * kPjTok + row) * kPjXP + 8 * c8, xptr(a, h, ok ? s : 0, f0 + 8 * c8), ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  load(0, 0);
  // both terms of Vt (overlaps the first chunk's copies)
  const float *vt = a.blocks + (size_t)h * R * F;
  for (int e = threadIdx.x; e < R * F / 4; e += 256) {
    const int c = (4 * e) / F, f = (4 * e) % F;
    const float4 v = *reinterpret_cast<const float4 *>(vt + (size_t)c * F + f);
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(vv[q]);
      vhi[c * VP + f + q] = hi;
      vlo[c * VP + f + q] = __float2bfloat16_rn(vv[q] - __bfloat162float(hi));
    }
  }
  constexpr int NT = R / 8;                 // n8 tiles
  const int g = lane >> 2, t = lane & 3, lr = lane & 7, li = lane >> 3;
  float acc[NT][4];
  for (int item = 0; item < n_items; ++item) {
    const int buf = item & 1, chunk = item % n_chunks;
    if (item + 1 < n_items) {
      load(item + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    if (chunk == 0) {
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    }
    const __nv_bfloat16 *xb = xs + (size_t)buf * kPjTok * kPjXP;
#pragma unroll
    for (int ks = 0; ks < kPjK / 16; ++ks) {
      uint32_t af[4];
      ldsm_x4(smem_u32(xb + (16 * warp + lr + (li & 1) * 8) * kPjXP + 16 * ks + (li >> 1) * 8), af);
      const int fk = chunk * kPjK + 16 * ks;
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t bh[4], bl[4];
        const int off = (16 * np + lr + (li >> 1) * 8) * VP + fk + (li & 1) * 8;
        ldsm_x4(smem_u32(vhi + off), bh);
        ldsm_x4(smem_u32(vlo + off), bl);
        mma_bf16(acc[2 * np], af, bh[0], bh[1]);
        mma_bf16(acc[2 * np], af, bl[0], bl[1]);
        mma_bf16(acc[2 * np + 1], af, bh[2], bh[3]);
        mma_bf16(acc[2 * np + 1], af, bl[2], bl[3]);
      }
    }
    __syncthreads();
    if (chunk == n_chunks - 1) {
      const int tile = tile0 + item / n_chunks;
#pragma unroll
      for (int hi8 = 0; hi8 < 2; ++hi8) {
        const int s = tile * kPjTok + 16 * warp + g + 8 * hi8;
        if (s >= a.S) continue;
        const size_t o = ((size_t)h * a.S + s) * R + 2 * t;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const float x0 = acc[n][2 * hi8], x1 = acc[n][2 * hi8 + 1];
          if (a.basis_bf16)
            *reinterpret_cast<uint32_t *>(static_cast<__nv_bfloat16 *>(a.basis) + o + 8 * n) = pack_bf16(x0, x1);
          else
            *reinterpret_cast<float2 *>(static_cast<float *>(a.basis) + o + 8 * n) = make_float2(x0, x1);
        }
      }
    }
  }
}

// ------------------------------------------------- selective reconstruction
// CTA = (64 selected rows, head), 256 threads, on the tensor cores.  The
// layer's r x d_h block of Vt is split into two bf16 terms in shared memory
// ([c][j], j contiguous: the B operand through ldmatrix.trans); the 64 basis
// rows are gathered with cp.async (bf16 basis, exact) or loaded and split into
// two bf16 terms (float32 basis).  out = A . (Vt_hi + Vt_lo) [+ A_lo . Vt_hi]
// with mma.sync m16n8k16 and fp32 accumulation, rounded to bf16.  Warp w owns
// rows 16 (w & 3) .. + 15 and output dims (w >> 2) D/2 .. + D/2.
struct XrArgs {
  int S, n_kv, d, F, layer, n_sel;
  const void *basis;
  const float *blocks;
  const int32_t *idx;
  __nv_bfloat16 *out;
};

template <int R, int D>
struct RebuildLayout {
  static constexpr int BP = D + 8;            // bf16 pitch of a Vt block row
  static constexpr int AP = R + 8;            // bf16 pitch of a basis row
  static constexpr int kOffBl = R * BP * 2;
  static constexpr int kOffAh = 2 * R * BP * 2;
  static constexpr int kOffAl = kOffAh + 64 * AP * 2;
  static constexpr int kOffIdx = kOffAl + 64 * AP * 2;
  static constexpr int kBytes = kOffIdx + 64 * 4;
};

template <int R, int D, bool BF16>
__global__ void __launch_bounds__(256) xkv_rebuild_tc(XrArgs a) {
  using Ly = RebuildLayout<R, D>;
  constexpr int BP = Ly::BP, AP = Ly::AP;
  extern __shared__ __align__(16) uint8_t xk_rb_smem[];
  __nv_bfloat16 *bh = reinterpret_cast<__nv_bfloat16 *>(xk_rb_smem);
  __nv_bfloat16 *bl = reinterpret_cast<__nv_bfloat16 *>(xk_rb_smem + Ly::kOffBl);
  __nv_bfloat16 *ah = reinterpret_cast<__nv_bfloat16 *>(xk_rb_smem + Ly::kOffAh);
  __nv_bfloat16 *al = reinterpret_cast<__nv_bfloat16 *>(xk_rb_smem + Ly::kOffAl);
  int *sidx = reinterpret_cast<int *>(xk_rb_smem + Ly::kOffIdx);
  const int h = blockIdx.y, t0 = blockIdx.x * 64, tid = threadIdx.x;
  if (tid < 64) {
    const int t = t0 + tid;
    const int src = t < a.n_sel ? __ldg(a.idx + (size_t)h * a.n_sel + t) : -1;
    sidx[tid] = (src >= 0 && src < a.S) ? src : -1;
  }
  __syncthreads();
  // the 64 basis rows
  if constexpr (BF16) {
    const __nv_bfloat16 *base = static_cast<const __nv_bfloat16 *>(a.basis);
    for (int e = tid; e < 64 * (R / 8); e += 256) {
      const int row = e / (R / 8), p8 = e % (R / 8), src = sidx[row];
      cp_async16(ah + row * AP + 8 * p8, base + ((size_t)h * a.S + (src < 0 ? 0 : src)) * R + 8 * p8, src >= 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  } else {
    const float *base = static_cast<const float *>(a.basis);
    for (int e = tid; e < 64 * (R / 4); e += 256) {
      const int row = e / (R / 4), p4 = e % (R / 4), src = sidx[row];
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (src >= 0) v = __ldg(reinterpret_cast<const float4 *>(base + ((size_t)h * a.S + src) * R + 4 * p4));
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(vv[q]);
        ah[row * AP + 4 * p4 + q] = hi;
        al[row * AP + 4 * p4 + q] = __float2bfloat16_rn(vv[q] - __bfloat162float(hi));
      }
    }
  }
  // the layer's block of Vt, two terms
  const float *vt = a.blocks + (size_t)h * R * a.F + (size_t)a.layer * D;
  for (int e = tid; e < R * D / 4; e += 256) {
    const int c = e / (D / 4), j4 = e % (D / 4);
    const float4 v = __ldg(reinterpret_cast<const float4 *>(vt + (size_t)c * a.F + 4 * j4));
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(vv[q]);
      bh[c * BP + 4 * j4 + q] = hi;
      bl[c * BP + 4 * j4 + q] = __float2bfloat16_rn(vv[q] - __bfloat162float(hi));
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  constexpr int NTW = D / 16;                 // n8 tiles per warp
  const int warp = warp_id(), lane = lane_id();
  const int mt = warp & 3, n0 = (warp >> 2) * (D / 2);
  const int g = lane >> 2, t = lane & 3, lr = lane & 7, li = lane >> 3;
  float acc[NTW][4];
#pragma unroll
  for (int n = 0; n < NTW; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < R / 16; ++ks) {
    uint32_t af[4], afl[4];
    const int aoff = (16 * mt + lr + (li & 1) * 8) * AP + 16 * ks + (li >> 1) * 8;
    ldsm_x4(smem_u32(ah + aoff), af);
    if constexpr (!BF16) ldsm_x4(smem_u32(al + aoff), afl);
#pragma unroll
    for (int np = 0; np < NTW / 2; ++np) {
      uint32_t rh[4], rl[4];
      const int boff = (16 * ks + lr + (li & 1) * 8) * BP + n0 + 16 * np + (li >> 1) * 8;
      ldsm_x4_t(smem_u32(bh + boff), rh);
      ldsm_x4_t(smem_u32(bl + boff), rl);
      mma_bf16(acc[2 * np], af, rh[0], rh[1]);
      mma_bf16(acc[2 * np], af, rl[0], rl[1]);
      mma_bf16(acc[2 * np + 1], af, rh[2], rh[3]);
      mma_bf16(acc[2 * np + 1], af, rl[2], rl[3]);
      if constexpr (!BF16) {
        mma_bf16(acc[2 * np], afl, rh[0], rh[1]);
        mma_bf16(acc[2 * np + 1], afl, rh[2], rh[3]);
      }
    }
  }
#pragma unroll
  for (int hi8 = 0; hi8 < 2; ++hi8) {
    const int row = 16 * mt + g + 8 * hi8, tt = t0 + row;
    if (tt >= a.n_sel) continue;
    __nv_bfloat16 *o = a.out + ((size_t)tt * a.n_kv + h) * D + n0 + 2 * t;
#pragma unroll
    for (int n = 0; n < NTW; ++n)
      *reinterpret_cast<uint32_t *>(o + 8 * n) = pack_bf16(acc[n][2 * hi8], acc[n][2 * hi8 + 1]);
  }
}

template <int R>
cudaError_t factorize_r(XkArgs a, int iters, float *v_a, float *v_b, const float *v0, cudaStream_t st) {
  cudaError_t e;
  const int nt = a.F / kGramTile;
  const dim3 gg(nt * (nt + 1) / 2, a.n_kv, (a.S + a.tok_per_split - 1) / a.tok_per_split);
  if ((e = ensure_smem_limit((const void *)xkv_gram, kGramSmem))) return e;
  xkv_gram<<<gg, 128, kGramSmem, st>>>(a);
  count_launch();
  if ((e = cudaGetLastError())) return e;
  const int gv_smem = 2 * kGvK * (kRowsPerCta + R) * (int)sizeof(float);
  const int chol_smem = (3 * R * (R + 1) + R) * (int)sizeof(double);
  const int apply_smem = R * R * (int)sizeof(double) + kRowsPerCta * (R + 1) * (int)sizeof(float);
  const int proj_smem = (2 * R * (a.F + 8) + 2 * kPjTok * kPjXP) * (int)sizeof(__nv_bfloat16);
  if ((e = ensure_smem_limit((const void *)xkv_gv<R>, gv_smem))) return e;
  if ((e = ensure_smem_limit((const void *)xkv_chol<R>, chol_smem))) return e;
  if ((e = ensure_smem_limit((const void *)xkv_apply<R>, apply_smem))) return e;
  if ((e = ensure_smem_limit((const void *)xkv_project_tc<R>, proj_smem))) return e;
  const dim3 rows(a.F / kRowsPerCta, a.n_kv);
  const float *cur = v0;
  for (int it = 0; it < iters; ++it) {
    float *nxt = (it & 1) ? v_b : v_a;
    a.v_in = cur;
    a.v_out = nxt;
    xkv_gv<R><<<rows, 128, gv_smem, st>>>(a);
    count_launch();
    if ((e = cudaGetLastError())) return e;
    xkv_chol<R><<<a.n_kv, 512, chol_smem, st>>>(a);
    count_launch();
    if ((e = cudaGetLastError())) return e;
    xkv_apply<R><<<rows, 128, apply_smem, st>>>(a, it == iters - 1 ? 1 : 0);
    count_launch();
    if ((e = cudaGetLastError())) return e;
    cur = nxt;
  }
  // about one CTA per SM over (token runs, heads)
  const int n_tiles = (a.S + kPjTok - 1) / kPjTok;
  const int ctas_per_head = std::max(1, std::min(n_tiles, (kNumSMs + a.n_kv - 1) / a.n_kv));
  const int tiles_per_cta = (n_tiles + ctas_per_head - 1) / ctas_per_head;
  xkv_project_tc<R><<<dim3((n_tiles + tiles_per_cta - 1) / tiles_per_cta, a.n_kv), 256, proj_smem, st>>>(a, tiles_per_cta);
  count_launch();
  return cudaGetLastError();
}

template <int R, int D, bool BF16>
cudaError_t rebuild_launch(const XrArgs &a, cudaStream_t st) {
  constexpr int smem = RebuildLayout<R, D>::kBytes;
  cudaError_t e = ensure_smem_limit((const void *)xkv_rebuild_tc<R, D, BF16>, smem);
  if (e) return e;
  xkv_rebuild_tc<R, D, BF16><<<dim3((a.n_sel + 63) / 64, a.n_kv), 256, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <int R>
cudaError_t rebuild_r(const XrArgs &a, bool bf16, cudaStream_t st) {
  if (a.d == 128) return bf16 ? rebuild_launch<R, 128, true>(a, st) : rebuild_launch<R, 128, false>(a, st);
  return bf16 ? rebuild_launch<R, 64, true>(a, st) : rebuild_launch<R, 64, false>(a, st);
}

}  // namespace

int xkv_gram_split_tokens(int S, int n_kv, int F) {
  // about four CTAs per SM over (upper tiles, heads, token splits); each split
  // a whole number of pipeline steps
  const int nt = F / kGramTile;
  const int64_t tiles = (int64_t)nt * (nt + 1) / 2 * n_kv;
  int64_t splits = (4 * (int64_t)kNumSMs + tiles - 1) / tiles;
  splits = std::max<int64_t>(1, std::min<int64_t>(splits, (S + kGramS - 1) / kGramS));
  const int64_t per = (S + splits - 1) / splits;
  return (int)((per + kGramS - 1) / kGramS * kGramS);
}

cudaError_t xkv_factorize(const XkvArgs &x, cudaStream_t st) {
  XkArgs a = {};
  for (int l = 0; l < x.W; ++l) a.k[l] = static_cast<const __nv_bfloat16 *>(x.k_layers[l]);
  a.S = x.S; a.n_kv = x.n_kv; a.d = x.d_h; a.W = x.W; a.F = x.W * x.d_h; a.r = x.r;
  a.tok_per_split = xkv_gram_split_tokens(x.S, x.n_kv, a.F);
  a.gram = x.gram; a.y = x.y; a.c = x.c; a.m = x.m; a.blocks = x.blocks;
  a.basis = x.basis; a.basis_bf16 = x.basis_bf16;
  cudaError_t e = cudaMemsetAsync(x.gram, 0, (size_t)x.n_kv * a.F * a.F * sizeof(float), st);
  if (e) return e;
  e = cudaMemsetAsync(x.c, 0, (size_t)x.n_kv * x.r * x.r * sizeof(double), st);
  if (e) return e;
  switch (x.r) {
    case 16: return factorize_r<16>(a, x.iters, x.v_a, x.v_b, x.v0, st);
    case 32: return factorize_r<32>(a, x.iters, x.v_a, x.v_b, x.v0, st);
    default: return factorize_r<64>(a, x.iters, x.v_a, x.v_b, x.v0, st);
  }
}

cudaError_t xkv_reconstruct(const XkvArgs &x, cudaStream_t st) {
  XrArgs a = {};
  a.S = x.S; a.n_kv = x.n_kv; a.d = x.d_h; a.F = x.W * x.d_h; a.layer = x.layer; a.n_sel = x.n_sel;
  a.basis = x.basis; a.blocks = x.blocks; a.idx = x.idx; a.out = static_cast<__nv_bfloat16 *>(x.out);
  switch (x.r) {
    case 16: return rebuild_r<16>(a, x.basis_bf16, st);
    case 32: return rebuild_r<32>(a, x.basis_bf16, st);
    default: return rebuild_r<64>(a, x.basis_bf16, st);
  }
}

}  // namespace kvc
