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
//   xkv_project A_h = X_h V, 64 tokens per CTA, V in shared memory;
//   xkv_rebuild rows idx of layer l: A_h[idx] Vt_h[:, layer block], rounded to
//               bf16 (nearest even).
#include <algorithm>

#include "kvc_common.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr int kGramTile = 64;     // output tile of the Gram kernel
constexpr int kGramS = 32;        // tokens per pipeline step
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
  const float *v_final;           // [n_kv, F, r] for the projection
  void *basis;                    // A [n_kv, S, r], float32 or bf16
  bool basis_bf16;
};

// X_h element (token s, feature f)
KVC_DEVINL const __nv_bfloat16 *xptr(const XkArgs &a, int h, int s, int f) {
  const int l = f / a.d, j = f - l * a.d;
  return a.k[l] + ((size_t)s * a.n_kv + h) * a.d + j;
}

// ------------------------------------------------------------------ Gram
__global__ void __launch_bounds__(128) xkv_gram(XkArgs a) {
  __shared__ __align__(16) __nv_bfloat16 si[2][kGramS][kGramPitch];
  __shared__ __align__(16) __nv_bfloat16 sj[2][kGramS][kGramPitch];
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
  const int n_steps = (s1 - s0 + kGramS - 1) / kGramS;
  load(0, s0);
  for (int st = 0; st < n_steps; ++st) {
    const int buf = st & 1;
    if (st + 1 < n_steps) {
      load(buf ^ 1, s0 + (st + 1) * kGramS);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
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
#pragma unroll
      for (int c = 0; c < CPT; ++c) vv[c] = v_t[kk * R + c];
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
// One CTA per head, 256 threads.  Right-looking Cholesky of C with two
// barriers per column, then L^-1 row by row (4 threads per column, their
// partial sums combined by shuffles), stored transposed as M.
template <int R>
__global__ void __launch_bounds__(256) xkv_chol(XkArgs a) {
  constexpr int LP = R + 1;
  extern __shared__ __align__(16) double xk_chol_smem[];
  double *L = xk_chol_smem;          // [R][LP]
  double *X = L + R * LP;            // [R][LP]: L^-1
  double *diag = X + R * LP;         // [R]
  const int h = blockIdx.x, tid = threadIdx.x;
  double *C = a.c + (size_t)h * R * R;
  for (int e = tid; e < R * R; e += 256) {
    const int p = e / R, q = e % R;
    L[p * LP + q] = q <= p ? C[e] : 0.0;
    X[p * LP + q] = 0.0;
    C[e] = 0.0;                      // ready for the next step's atomics
  }
  __syncthreads();
  double tr = 0.0;
  for (int p = 0; p < R; ++p) tr += L[p * LP + p];
  // a pivot below this floor (a rank-deficient Y) is raised to it
  const double floor_piv = fmax(tr, 1e-300) * 1e-30;
  for (int c = 0; c < R; ++c) {
    const double dcc = sqrt(fmax(L[c * LP + c], floor_piv));
    if (tid == 0) diag[c] = dcc;
    for (int p = c + 1 + tid; p < R; p += 256) L[p * LP + c] /= dcc;
    __syncthreads();
    const int n = R - c - 1;
    for (int e = tid; e < n * n; e += 256) {
      const int p = c + 1 + e / n, q = c + 1 + e % n;
      if (q <= p) L[p * LP + q] -= L[p * LP + c] * L[q * LP + c];
    }
    __syncthreads();
  }
  // X = L^-1 (lower), row i from rows < i; thread group (j, part), j < R
  const int j = tid / 4, part = tid % 4;
  for (int i = 0; i < R; ++i) {
    double s = 0.0;
    if (j < i)
      for (int k = j + part; k < i; k += 4) s = fma(L[i * LP + k], X[k * LP + j], s);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (part == 0 && j <= i) X[i * LP + j] = j == i ? 1.0 / diag[i] : -s / diag[i];
    __syncthreads();
  }
  double *M = a.m + (size_t)h * R * R;
  for (int e = tid; e < R * R; e += 256) {
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
template <int R>
__global__ void __launch_bounds__(256) xkv_project(XkArgs a) {
  extern __shared__ __align__(16) float xk_proj_smem[];
  constexpr int CPT = R / 16;
  float *sv = xk_proj_smem;                       // [F][R]
  float *sx = xk_proj_smem + (size_t)a.F * R;     // [64][33]: 32 features of 64 tokens
  const int h = blockIdx.y, s0 = blockIdx.x * 64, F = a.F;
  const float *V = a.v_final + (size_t)h * F * R;
  for (int e = threadIdx.x; e < F * R / 4; e += blockDim.x)
    reinterpret_cast<float4 *>(sv)[e] = reinterpret_cast<const float4 *>(V)[e];
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;   // rows 4 ty .. 4 ty + 3, columns tx * CPT ..
  float acc[4][CPT];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[q][c] = 0.f;
  for (int f0 = 0; f0 < F; f0 += 32) {
    __syncthreads();
    {   // 64 tokens x 4 pieces of 8 features: one piece per thread
      const int row = threadIdx.x / 4, p8 = threadIdx.x % 4, s = s0 + row;
      float vals[8];
      if (s < a.S) {
        const uint4 u = *reinterpret_cast<const uint4 *>(xptr(a, h, s, f0 + 8 * p8));
        Elem<__nv_bfloat16>::unpack(u, vals);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) vals[q] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) sx[row * 33 + 8 * p8 + q] = vals[q];
    }
    __syncthreads();
#pragma unroll 4
    for (int ff = 0; ff < 32; ++ff) {
      float xv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) xv[q] = sx[(ty * 4 + q) * 33 + ff];
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const float vv = sv[(f0 + ff) * R + tx * CPT + c];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q][c] = fmaf(xv[q], vv, acc[q][c]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int s = s0 + ty * 4 + q;
    if (s >= a.S) continue;
    const size_t o = ((size_t)h * a.S + s) * R + tx * CPT;
    if (a.basis_bf16) {
      __nv_bfloat16 *b = static_cast<__nv_bfloat16 *>(a.basis) + o;
#pragma unroll
      for (int c = 0; c < CPT; ++c) b[c] = __float2bfloat16_rn(acc[q][c]);
    } else {
      float *b = static_cast<float *>(a.basis) + o;
#pragma unroll
      for (int c = 0; c < CPT; ++c) b[c] = acc[q][c];
    }
  }
}

// ------------------------------------------------- selective reconstruction
// CTA = (64 selected rows, head); the layer's r x d_h block of Vt in shared
// memory; one warp per row, each lane d_h / 32 output dims; the basis row is
// spread over the lanes and broadcast by shuffles.
struct XrArgs {
  int S, n_kv, d, F, layer, n_sel;
  const void *basis;
  const float *blocks;
  const int32_t *idx;
  __nv_bfloat16 *out;
};

template <int R, int D, bool BF16>
__global__ void __launch_bounds__(256) xkv_rebuild(XrArgs a) {
  constexpr int DPL = D / 32;
  constexpr int NU = (R + 31) / 32;
  __shared__ __align__(16) float sb[R * D];
  const int h = blockIdx.y, t0 = blockIdx.x * 64;
  const float *vt = a.blocks + (size_t)h * R * a.F + (size_t)a.layer * D;
  for (int e = threadIdx.x; e < R * D / 4; e += 256) {
    const int c = e / (D / 4), j4 = e % (D / 4);
    reinterpret_cast<float4 *>(sb)[e] = *reinterpret_cast<const float4 *>(vt + (size_t)c * a.F + 4 * j4);
  }
  __syncthreads();
  const int lane = lane_id();
  const int t_end = min(a.n_sel, t0 + 64);
  for (int t = t0 + warp_id(); t < t_end; t += 8) {
    const int src = __ldg(a.idx + (size_t)h * a.n_sel + t);
    const bool in = src >= 0 && src < a.S;
    float av[NU];
#pragma unroll
    for (int u = 0; u < NU; ++u) {
      const int c = lane + 32 * u;
      float x = 0.f;
      if (in && c < R) {
        const size_t o = ((size_t)h * a.S + src) * R + c;
        if constexpr (BF16) x = __bfloat162float(static_cast<const __nv_bfloat16 *>(a.basis)[o]);
        else x = static_cast<const float *>(a.basis)[o];
      }
      av[u] = x;
    }
    float acc[DPL];
#pragma unroll
    for (int q = 0; q < DPL; ++q) acc[q] = 0.f;
#pragma unroll 8
    for (int c = 0; c < R; ++c) {
      const float ac = __shfl_sync(0xffffffffu, av[c / 32], c % 32);
      const float *row = sb + c * D + lane * DPL;
      if constexpr (DPL == 4) {
        const float4 b4 = *reinterpret_cast<const float4 *>(row);
        acc[0] = fmaf(ac, b4.x, acc[0]);
        acc[1] = fmaf(ac, b4.y, acc[1]);
        acc[2] = fmaf(ac, b4.z, acc[2]);
        acc[3] = fmaf(ac, b4.w, acc[3]);
      } else {
        const float2 b2 = *reinterpret_cast<const float2 *>(row);
        acc[0] = fmaf(ac, b2.x, acc[0]);
        acc[1] = fmaf(ac, b2.y, acc[1]);
      }
    }
    __nv_bfloat16 *o = a.out + ((size_t)t * a.n_kv + h) * D + lane * DPL;
    if constexpr (DPL == 4) {
      uint2 u;
      u.x = pack_bf16(acc[0], acc[1]);
      u.y = pack_bf16(acc[2], acc[3]);
      *reinterpret_cast<uint2 *>(o) = u;
    } else {
      *reinterpret_cast<uint32_t *>(o) = pack_bf16(acc[0], acc[1]);
    }
  }
}

template <int R>
cudaError_t factorize_r(XkArgs a, int iters, float *v_a, float *v_b, const float *v0, cudaStream_t st) {
  cudaError_t e;
  const int nt = a.F / kGramTile;
  const dim3 gg(nt * (nt + 1) / 2, a.n_kv, (a.S + a.tok_per_split - 1) / a.tok_per_split);
  xkv_gram<<<gg, 128, 0, st>>>(a);
  count_launch();
  if ((e = cudaGetLastError())) return e;
  const int gv_smem = 2 * kGvK * (kRowsPerCta + R) * (int)sizeof(float);
  const int chol_smem = (2 * R * (R + 1) + R) * (int)sizeof(double);
  const int apply_smem = R * R * (int)sizeof(double) + kRowsPerCta * (R + 1) * (int)sizeof(float);
  const int proj_smem = (a.F * R + 64 * 33) * (int)sizeof(float);
  if ((e = ensure_smem_limit((const void *)xkv_gv<R>, gv_smem))) return e;
  if ((e = ensure_smem_limit((const void *)xkv_chol<R>, chol_smem))) return e;
  if ((e = ensure_smem_limit((const void *)xkv_apply<R>, apply_smem))) return e;
  if ((e = ensure_smem_limit((const void *)xkv_project<R>, proj_smem))) return e;
  const dim3 rows(a.F / kRowsPerCta, a.n_kv);
  const float *cur = v0;
  for (int it = 0; it < iters; ++it) {
    float *nxt = (it & 1) ? v_b : v_a;
    a.v_in = cur;
    a.v_out = nxt;
    xkv_gv<R><<<rows, 128, gv_smem, st>>>(a);
    count_launch();
    if ((e = cudaGetLastError())) return e;
    xkv_chol<R><<<a.n_kv, 256, chol_smem, st>>>(a);
    count_launch();
    if ((e = cudaGetLastError())) return e;
    xkv_apply<R><<<rows, 128, apply_smem, st>>>(a, it == iters - 1 ? 1 : 0);
    count_launch();
    if ((e = cudaGetLastError())) return e;
    cur = nxt;
  }
  a.v_final = cur;
  xkv_project<R><<<dim3((a.S + 63) / 64, a.n_kv), 256, proj_smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <int R>
cudaError_t rebuild_r(const XrArgs &a, bool bf16, cudaStream_t st) {
  const dim3 grid((a.n_sel + 63) / 64, a.n_kv);
  count_launch();
  if (a.d == 128) {
    if (bf16) xkv_rebuild<R, 128, true><<<grid, 256, 0, st>>>(a);
    else xkv_rebuild<R, 128, false><<<grid, 256, 0, st>>>(a);
  } else {
    if (bf16) xkv_rebuild<R, 64, true><<<grid, 256, 0, st>>>(a);
    else xkv_rebuild<R, 64, false><<<grid, 256, 0, st>>>(a);
  }
  return cudaGetLastError();
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
