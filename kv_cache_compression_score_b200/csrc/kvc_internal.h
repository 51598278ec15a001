// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kvc.h"

namespace kvc {

// B200: 148 SMs.  Work plans (and therefore workspace sizes) are computed for
// this count so that a size query needs no device call.
constexpr int kNumSMs = 148;

struct ScoreArgs {
  kvc_dtype dt;
  int n_seqs, n_h, n_kv, d_h, w;
  float scale;
  const int32_t *cu_seqlens;
  const void *q_win;
  const void *k;
  float2 *part;          // [n_seqs, n_kv, n_chunks, R_pad] (m, l) per window row
  float *raw;            // [n_kv, T_total]
  float *scores;         // [n_kv, T_total] pooled (written by the fused path)
  int *sync;             // fused path: counters per (sequence, KV head), zero between calls
  int *err;              // device error word (nonzero: a bounded wait gave up)
  int pool_k;
  bool fused;            // both passes and the pool in one cooperative launch
  // selection and gather inside the fused launch (idx == nullptr: not requested)
  int32_t *idx;
  const int32_t *cu_budget;
  const void *v;
  void *k_out, *v_out;
  int *hist, *cnt;
  int total_budget, budget;
  int T_total;
  int n_chunks;          // key chunks per (sequence, KV head) in the launch grid
  int keys_per_chunk;    // multiple of the kernel's key tile
  int R_pad;             // padded window-block rows used for the partials
};

cudaError_t score_window_simt(const ScoreArgs &a, cudaStream_t st);
cudaError_t score_window_tc(const ScoreArgs &a, cudaStream_t st);
int simt_keys_per_tile();
int tc_keys_per_tile();
int tc_counters_per_unit();   // fused launch: arrival counters per (sequence, KV head)
int tc_hist_ints();           // fused selection: histogram ints per (sequence, KV head)
int tc_count_ints();          // fused selection: count ints per (sequence, KV head, key chunk)
int tc_select_max_keys(int d_h);  // fused selection: largest key chunk it keeps on chip

cudaError_t pool_prefix(const float *raw, float *scores, const int32_t *cu_seqlens, int n_seqs, int n_kv,
                        int T_total, int max_len, int w, int pool_k, cudaStream_t st);

// mask (nullable): int32 [n_seqs * n_kv]; (sequence, head) pairs whose entry
// is 0 are left untouched
cudaError_t select_topk(const float *scores, int32_t *idx, const int32_t *cu_seqlens, const int32_t *cu_budget,
                        int n_seqs, int n_kv, int T_total, int total_budget, int w, int budget, int max_len,
                        cudaStream_t st, const int32_t *mask = nullptr);

cudaError_t gather_rows_kv(const void *k, const void *v, void *k_out, void *v_out, const int32_t *idx,
                           const int32_t *cu_seqlens, const int32_t *cu_budget, int n_seqs, int n_kv,
                           int row_bytes_per_head, int total_budget, int max_kept, cudaStream_t st,
                           const int32_t *mask = nullptr);

// FreeKV re-scoring of the drifted heads (freekv.cu)
struct FreeKvArgs {
  const __nv_bfloat16 *q_cur, *q_prev, *k;
  const int *cu_seqlens, *cu_budget;
  int *flags;            // [batch * n_kv] 1: scored and selected again this step
  int64_t *dec_off;      // [batch] decode row offsets of the compact caches
  int *dec_len;          // [batch] decode lengths
  float *z;              // [batch, n_kv, G, zpitch] logits (log2 units)
  float2 *part;          // [batch, n_kv, n_chunks, G] (max, sum of 2^(z - max)) per key chunk
  float *scores;         // [n_kv, T_total] pooled scores of the flagged heads
  int batch, n_h, n_kv, d_h, w, pool_r, n_chunks, T_total;
  int64_t zpitch;
  float c;               // scale * log2(e)
  float tau;
};
cudaError_t freekv_rescore(const FreeKvArgs &a, cudaStream_t st);
int freekv_chunk_keys();

cudaError_t gather_rows_kv_q8(const void *k, const void *v, int8_t *kq, int8_t *vq, float *ks, float *vs,
                              int64_t scale_pitch, const int32_t *idx, const int32_t *cu_seqlens,
                              const int32_t *cu_budget, int n_seqs, int n_kv, int d_h, int total_budget, int max_kept,
                              cudaStream_t st);

cudaError_t tsp_pool(const float *raw, int n_rows, int S, int w, int pool_k, float *pooled, cudaStream_t st);
cudaError_t tsp_select(const float *pooled, int S, int w, int k_tsp, int32_t *idx_out, cudaStream_t st);
cudaError_t gather_hidden(const void *hidden, void *out, const int32_t *idx, int n_rows, int row_bytes, int n_src,
                          cudaStream_t st);

struct DecodeArgs {
  kvc_dtype dt;
  int batch, n_h, n_kv, d_h;
  float scale;
  const void *q, *k_c, *v_c;
  const int64_t *row_off;
  const int32_t *kv_len;
  float *out;
  float *part;
  int *tickets;
  int *err;              // device error word
  int64_t cache_rows;    // rows of k_c / v_c
  int n_chunks;          // partial slots per (batch entry, KV head)
  int chunk_rows;        // unused by the stream-K kernel (kept 0)
  // int8 caches (k_c / v_c hold int8 codes): per-(row, head) scales [n_kv, scale_pitch]
  const float *k_scale = nullptr, *v_scale = nullptr;
  int64_t scale_pitch = 0;
};
cudaError_t gqa_decode(const DecodeArgs &a, cudaStream_t st);
cudaError_t gqa_decode_tc(const DecodeArgs &a, cudaStream_t st);   // bf16 / int8 caches, tensor cores
int decode_slots(int max_kv_len);

// xKV cross-layer factorisation (xkv.cu)
constexpr int kXkvMaxW = 8;
struct XkvArgs {
  int S, n_kv, d_h, W, r, iters;
  const void *k_layers[kXkvMaxW];   // bf16 key caches [S, n_kv, d_h] of the window's layers
  const float *v0;                  // [n_kv, W d_h, r] start basis
  float *gram, *y, *v_a, *v_b;      // workspace
  double *c, *m;                    // workspace
  float *blocks;                    // Vt [n_kv, r, W d_h]
  void *basis;                      // A [n_kv, S, r] float32 or bf16
  bool basis_bf16;
  // reconstruction
  int layer, n_sel;
  const int32_t *idx;               // [n_kv, n_sel]
  void *out;                        // bf16 [n_sel, n_kv, d_h]
};
cudaError_t xkv_factorize(const XkvArgs &a, cudaStream_t st);
cudaError_t xkv_reconstruct(const XkvArgs &a, cudaStream_t st);
int xkv_gram_split_tokens(int S, int n_kv, int F);

}  // namespace kvc

namespace kvc {
// Host-side count of kernels this library enqueued (or recorded into a graph
// under stream capture); every launch site calls it once per launch.
void count_launch();
// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel of the stream finishes; it calls grid_dependency_wait()
// before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}
// Raise a kernel's dynamic shared-memory limit once per device (a host call
// kept out of the per-launch path, so launches can be captured in graphs).
cudaError_t ensure_smem_limit(const void *fn, int bytes);
}  // namespace kvc
