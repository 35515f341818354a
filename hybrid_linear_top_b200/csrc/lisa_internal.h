// Internal launch parameters shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lisa.h"

namespace lisa {

constexpr int kMaxR = 8;        // indexer heads per KV head
constexpr int kMaxG = 16;       // query heads per KV head
constexpr int kAttnRows = 32;   // selected rows per attention CTA / tile
constexpr int kLinChunk = 64;   // chunk length of the chunked linear attention

// Raises the dynamic shared-memory limit of kernel `fn` to `dyn_smem` (once per
// device and size; host-side bookkeeping only).
cudaError_t prepare_kernel_ptr(const void *fn, int dyn_smem);

template <typename F>
cudaError_t prepare_kernel(F *fn, int dyn_smem = 0) {
  return prepare_kernel_ptr(reinterpret_cast<const void *>(fn), dyn_smem);
}

// 2-D tiled TMA tensor map over a row-major [rows][cols] array (elements of
// elem_bytes, rows row_stride_bytes apart), box [box_rows][box_cols], with the
// given shared-memory swizzle span (0, 32, 64 or 128 bytes).  Host only.
bool make_tmap_2d(CUtensorMap *map, const void *base, int elem_bytes, unsigned long long cols,
                  unsigned long long rows, unsigned long long row_stride_bytes, unsigned box_cols, unsigned box_rows,
                  int swizzle_bytes);
// Same for rank 1..5: dims[0] innermost; strides_bytes[i] is the stride of dims[i+1].
bool make_tmap(CUtensorMap *map, const void *base, int elem_bytes, int rank, const unsigned long long *dims,
               const unsigned long long *strides_bytes, const unsigned *box, int swizzle_bytes);

// ------------------------------------------------------------- decode
struct DecodeParams {
  int B, Hq, Hkv, G, HI, R, D, DI, M, L_max;
  int fuse_append;
  float scale;                          // 1 / sqrt(d)
  // layer buffers
  void *k_cache, *v_cache, *kidx_cache;
  float *state;
  const int *pos;
  int *err_word;
  // step inputs / outputs
  const void *q, *k, *v, *kidx, *qidx;
  const float *w, *gate;
  void *out;
  int *idx_out;
  // launch geometry (filled by the launcher)
  int split_req;                        // requested CTAs per (b, g): 0 (library's choice), 4, 8, 16, 32, 64
  int window;                           // 1: sliding-window variant (M = the window W; no indexer inputs)
  const int *sel_ext;                   // non-NULL: index lists given, [B, sel_groups, M] (no indexer inputs)
  int sel_groups;                       // selection groups of sel_ext: 1 (one set for every KV head) or Hkv
  const void *k_lin, *v_lin;            // non-NULL: linear-branch keys / values per query head [B, Hq, d]
  int nc;                               // CTAs per cluster
  int stages;                           // TMA ring stages
  int stage_keys;                       // keys per ring stage
  int kpc_max;                          // order keys per CTA, upper bound
  int independent;                      // 1: no wait on the previous launch of the stream (lisa_layer.independent)
  int debug_flags;                      // LISA_DEBUG_* bits
  // wide form (nw > 0): nw CTAs per (b, g) stream the keys and the state; the
  // last of their clusters to finish selects and attends.  Workspace per (b, g):
  int nw;                               // CTAs per (b, g), a multiple of 8, >= G; 0: the cluster form
  uint32_t *wkeys;                      // [B*Hkv][wkeys_stride] order keys of positions 0..t
  float *wpart;                         // [B*Hkv][nw][2][d] per-CTA partial o_lin of (up to) two heads
  unsigned *wcount;                     // [B*Hkv] arrival counters (zero between calls)
  int wkeys_stride;
};
// Workspace of the wide decode form (0 when it does not apply).
size_t decode_wide_workspace_bytes(int B, int Hkv, int G, int D, int L_max, int nw);
// CTAs per (b, g) the wide form would use for this layer (0: the cluster form).
int decode_wide_nw(int B, int Hkv, int G, int D, int DI, int dtype, int sms);
// Dynamic shared memory per CTA of the wide form.
int decode_wide_smem_bytes(int L_max, int M, int G, int D, int DI, int nw);

// Dynamic shared memory of the decode kernel for a cluster of nc CTAs.
int decode_smem_bytes(int L_max, int M, int G, int D, int DI, int esize, int nc, bool lin_kv = false);
cudaError_t launch_decode(const DecodeParams &p, int dtype, cudaStream_t st);

// ------------------------------------------------------------- row path
// (prefill and lisa_indexer_topk): T query tokens at positions pos[b] + tau.
struct RowsParams {
  int B, Hq, Hkv, G, HI, R, D, DI, M, L_max, T;
  float scale;
  void *k_cache, *v_cache, *kidx_cache;
  float *state;
  const int *pos;
  int *err_word;
  int require_pos0;                     // prefill: pos[b] must be 0
  const void *q, *k, *v, *kidx, *qidx;
  const float *w, *gate;
  void *out;
  int *idx;                             // [B, T, sel_heads, M] (caller's idx_out or workspace)
  int sel_heads;                        // index lists per token read by the attention: Hkv, or 1 (one set
                                        // shared by every KV head)
  // workspace
  uint32_t *keys;                       // [B, Hkv, row_chunk, L_keys]
  float *olin;                          // [B, T, Hq, d]
  float *dS;                            // [B, Hkv, n_lin_chunks, d, d]
  float *Ptot;                          // [B, Hkv, d, d]
  int row_chunk;                        // query rows scored per pass
  int L_keys;                           // key slots per row in `keys` (multiple of 4)
  int smem_keys_cap, cand_cap;
  size_t select_smem;
};

cudaError_t launch_append(const RowsParams &p, int dtype, cudaStream_t st);
// Indexer scores + row top-M.  With ph != NULL the scores are first computed
// per indexer head with ph (one head per group, into ph->keys) and then summed
// over the HI / (p.Hkv) heads of each of p's groups into p.keys.
cudaError_t launch_rows_topk(const RowsParams &p, int dtype, cudaStream_t st, int key_limit,
                             const RowsParams *ph = nullptr);
// bf16 indexer scores of rows [tau0, tau0 + rows) of the pass on the tensor cores.
cudaError_t launch_rows_score_tc(const RowsParams &p, cudaStream_t st, int tau0, int rows, int key_hi);
cudaError_t launch_prefill_linear(const RowsParams &p, int dtype, cudaStream_t st);
// bf16, d = 128: the chunked linear attention on the tensor cores (chunks of 128).
cudaError_t launch_prefill_linear_tc(const RowsParams &p, cudaStream_t st);
// Pieces shared by both chunked paths (d = 128): exclusive prefix of the chunk
// increments dS over chunks of `chunk` tokens, and S_T = S_0 + total.
cudaError_t launch_lin_prefix(const RowsParams &p, cudaStream_t st, int chunk);
cudaError_t launch_lin_state(const RowsParams &p, cudaStream_t st);
cudaError_t launch_prefill_attend(const RowsParams &p, int dtype, cudaStream_t st);
// Stage-2 objective (forward): per-head KL of teacher attention vs indexer, kl_out [B, T, Hq].
cudaError_t launch_indexer_kl(const RowsParams &p, float *kl_out, cudaStream_t st);
// Its tensor-core (tcgen05) form, for d = 128 and at most 4 indexer heads per KV head.
bool indexer_kl_tc_supported(const RowsParams &p);
cudaError_t launch_indexer_kl_tc(const RowsParams &p, float *kl_out, cudaStream_t st);
// Sliding-window variant: idx of every row = its M most recent positions.
cudaError_t launch_window_idx(const RowsParams &p, cudaStream_t st);

// ------------------------------------------------------------- projections
// Z[rows x N] = X[rows x K] W^T (bf16, W [N x K]); output column c belongs to
// the segment with c0 <= c < c0 + width and goes to ptr[row * width + c - c0].
struct ProjSeg {
  int c0, width;
  void *ptr;
  int f32;                              // 1: fp32 output, 0: bf16
};
struct ProjParams {
  int rows, N, K;
  int nseg;
  ProjSeg seg[8];
  int *err_word;
};
cudaError_t launch_proj(const ProjParams &p, const void *x, const void *W, cudaStream_t st);

}  // namespace lisa
