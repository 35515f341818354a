// Row path of LISA on sm_100a: cache append, indexer scores + top-M for a
// block of query rows (prefill and lisa_indexer_topk), and the per-row sparse
// attention with the gate epilogue (prefill).
//
// Method: arXiv 2607.19358 (LISA), abstract (indexer -> top-M -> sparse
// attention, gated with a linear branch) and the gptget.net digest's method
// section (ReLU dot-product indexer); exact formulas as stated in lisa.h.
#include "lisa_internal.h"
#include "lisa_common.cuh"
#include "lisa_select.cuh"

namespace lisa {

__device__ __forceinline__ bool rows_pos_ok(const RowsParams &p, int b) {
  const int p0 = p.pos[b];
  return p0 >= 0 && p0 + p.T <= p.L_max && (!p.require_pos0 || p0 == 0);
}

// ============================================================ append
// grid (T, B*Hkv); copies k, v, kidx row tau of (b, g) to cache row pos[b]+tau
// (k and v when p.k is non-NULL, kidx when p.kidx is non-NULL).
template <typename T>
__global__ void append_kernel(RowsParams p) {
  const int tau = blockIdx.x;
  const int bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (!rows_pos_ok(p, b)) {
    if (tau == 0 && g == 0 && threadIdx.x == 0) set_err(p.err_word, LISA_DEVERR_POS);
    return;
  }
  const size_t dst = ((size_t)bg * p.L_max + p.pos[b] + tau);
  const size_t src = ((size_t)b * p.T + tau) * p.Hkv + g;
  const int nd = p.D * (int)sizeof(T) / 16, ndi = p.DI * (int)sizeof(T) / 16;
  const uint4 *ks = reinterpret_cast<const uint4 *>(p.k) + src * nd;
  const uint4 *vs = reinterpret_cast<const uint4 *>(p.v) + src * nd;
  const uint4 *kis = reinterpret_cast<const uint4 *>(p.kidx) + src * ndi;
  uint4 *kd = reinterpret_cast<uint4 *>(p.k_cache) + dst * nd;
  uint4 *vd = reinterpret_cast<uint4 *>(p.v_cache) + dst * nd;
  uint4 *kid = reinterpret_cast<uint4 *>(p.kidx_cache) + dst * ndi;
  if (p.k)
    for (int i = threadIdx.x; i < nd; i += blockDim.x) {
      kd[i] = ks[i];
      vd[i] = vs[i];
    }
  if (p.kidx)
    for (int i = threadIdx.x; i < ndi; i += blockDim.x) kid[i] = kis[i];
}

// ============================================================ sliding window
// grid (T, B*Hkv): idx of row tau = the M most recent positions t-M+1 .. t of
// t = pos[b] + tau (the whole prefix, -1 padded, while t < M).
__global__ void window_idx_kernel(RowsParams p) {
  const int tau = blockIdx.x, bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (!rows_pos_ok(p, b)) return;
  const int t = p.pos[b] + tau, n = t + 1, M = p.M;
  int *out = p.idx + (((size_t)b * p.T + tau) * p.Hkv + g) * M;
  for (int j = threadIdx.x; j < M; j += blockDim.x) out[j] = n <= M ? (j < n ? j : -1) : t - M + 1 + j;
}

cudaError_t launch_window_idx(const RowsParams &p, cudaStream_t st) {
  cudaError_t e = prepare_kernel(window_idx_kernel);
  if (e != cudaSuccess) return e;
  window_idx_kernel<<<dim3(p.T, p.B * p.Hkv), 128, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_append(const RowsParams &p, int dtype, cudaStream_t st) {
  dim3 grid(p.T, p.B * p.Hkv);
  if (dtype == LISA_BF16) {
    cudaError_t e = prepare_kernel(append_kernel<__nv_bfloat16>);
    if (e != cudaSuccess) return e;
    append_kernel<__nv_bfloat16><<<grid, 64, 0, st>>>(p);
  } else {
    cudaError_t e = prepare_kernel(append_kernel<float>);
    if (e != cudaSuccess) return e;
    append_kernel<float><<<grid, 64, 0, st>>>(p);
  }
  return cudaGetLastError();
}

// ============================================================ scores (CUDA cores)
// grid (key tiles, row tiles of the pass, B*Hkv); 256 threads, 4x4 scores each.
// Row tau of the pass sits at position pos[b] + tau; key s is a candidate iff
// s <= pos[b] + tau.  Output: order keys, keys[(bg*row_chunk + tau - tau0)*L_keys + s].
template <typename T, int DI>
__global__ void __launch_bounds__(256) rows_score_kernel(RowsParams p, int tau0, int rows) {
  __shared__ float s_k[64][DI + 1];
  __shared__ float s_q[64][DI + 1];
  __shared__ float s_w[64];
  const int kt = blockIdx.x, rt = blockIdx.y, bg = blockIdx.z;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (!rows_pos_ok(p, b)) return;
  const int p0 = p.pos[b];
  const int r_lo = rt * 64;                      // within the pass
  if (r_lo >= rows) return;
  const int r_hi = min(r_lo + 64, rows);
  const int s_lo = kt * 64;
  const int last_pos = p0 + tau0 + r_hi - 1;
  if (s_lo > last_pos) return;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  // indexer keys of the tile
  for (int i = tid; i < 64 * DI; i += 256) {
    const int r = i / DI, c = i % DI;
    const int s = s_lo + r;
    float x = 0.f;
    if (s <= last_pos)
      x = Dt<T>::to_f(reinterpret_cast<const T *>(p.kidx_cache)[((size_t)bg * p.L_max + s) * DI + c]);
    s_k[r][c] = x;
  }
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int r = 0; r < p.R; ++r) {
    const int hi = g * p.R + r;
    __syncthreads();
    for (int i = tid; i < 64 * DI; i += 256) {
      const int rr = i / DI, c = i % DI;
      const int tau = tau0 + r_lo + rr;
      float x = 0.f;
      if (r_lo + rr < r_hi)
        x = Dt<T>::to_f(reinterpret_cast<const T *>(p.qidx)[(((size_t)b * p.T + tau) * p.HI + hi) * DI + c]);
      s_q[rr][c] = x;
    }
    if (tid < 64) {
      const int tau = tau0 + r_lo + tid;
      s_w[tid] = (r_lo + tid < r_hi) ? p.w[((size_t)b * p.T + tau) * p.HI + hi] : 0.f;
    }
    __syncthreads();
    float dot[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) dot[i][j] = 0.f;
#pragma unroll 8
    for (int c = 0; c < DI; ++c) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = s_q[ty * 4 + i][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = s_k[tx * 4 + j][c];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dot[i][j] = fmaf(a[i], bb[j], dot[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(s_w[ty * 4 + i], fmaxf(dot[i][j], 0.f), acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = r_lo + ty * 4 + i;
    if (rr >= r_hi) continue;
    const int tpos = p0 + tau0 + rr;
    uint32_t *krow = p.keys + ((size_t)bg * p.row_chunk + rr) * p.L_keys;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int s = s_lo + tx * 4 + j;
      if (s <= tpos) krow[s] = score_key(acc[i][j]);
    }
  }
}

// ============================================================ select
// grid (rows of the pass, B*Hkv)
template <int NT>
__global__ void __launch_bounds__(NT) rows_select_kernel(RowsParams p, int tau0, int rows) {
  extern __shared__ __align__(16) uint32_t s_dyn[];
  __shared__ TopmShared sm;
  const int rr = blockIdx.x, bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (rr >= rows || !rows_pos_ok(p, b)) return;
  const int tau = tau0 + rr;
  const int n = p.pos[b] + tau + 1;
  const uint32_t *gkeys = p.keys + ((size_t)bg * p.row_chunk + rr) * p.L_keys;
  const uint32_t *keys = gkeys;
  uint32_t *cand = s_dyn;
  if (n > p.smem_keys_cap && threadIdx.x < 32) {
    // a long row is read from global memory: all of it requested into L2 at
    // once (32 KB bulk prefetches; rows start 16-byte aligned and hold L_keys,
    // a multiple of 4, slots)
    const int bytes = ((n * 4) + 15) & ~15;
    for (int off = threadIdx.x * 32768; off < bytes; off += 32 * 32768)
      bulk_prefetch_l2(reinterpret_cast<const char *>(gkeys) + off, (uint32_t)min(32768, bytes - off));
  }
  if (n > p.M && n <= p.smem_keys_cap) {
    const int n4 = n & ~3;
    for (int i = threadIdx.x * 4; i < n4; i += NT * 4)
      *reinterpret_cast<uint4 *>(s_dyn + i) = __ldcg(reinterpret_cast<const uint4 *>(gkeys + i));
    for (int i = n4 + threadIdx.x; i < n; i += NT) s_dyn[i] = __ldcg(gkeys + i);
    __syncthreads();
    keys = s_dyn;
    cand = s_dyn + p.smem_keys_cap;
  }
  int *out = p.idx + (((size_t)b * p.T + tau) * p.Hkv + g) * p.M;
  if (n >= 8 * NT) {
    // long rows (read from global memory / L2, not staged, so that several
    // rows share an SM): a bound from a sample and one pass over the keys;
    // where that bound does not serve, a bound from every thread's 4 largest
    // keys, then an exact select among the few keys above it
    __shared__ BoundedShared bsm;
    int r = 0;
    if (keys == gkeys && n > p.M)
      r = block_topm_sampled<NT>(keys, n, p.M, out, bsm, cand, reinterpret_cast<int *>(cand + p.cand_cap),
                                 p.cand_cap);
    if (r == 0)
      r = block_topm_bounded<NT>(keys, n, p.M, out, bsm, cand, reinterpret_cast<int *>(cand + p.cand_cap),
                                 p.cand_cap);
    if (r == 1) return;
    if (r < 0) {
      if (threadIdx.x == 0) set_err(p.err_word, LISA_DEVERR_CHECK);
      return;
    }
  }
  if (!block_topm<NT>(keys, n, p.M, out, sm, cand, p.cand_cap) && threadIdx.x == 0)
    set_err(p.err_word, LISA_DEVERR_CHECK);
}

// grid (rows of the pass, B*Hkv of p); one indexer key per indexer head: the
// score of group g is the sum of the per-head scores of its Rc = ph.Hkv / p.Hkv
// heads (ph scored one head per group), each a weighted ReLU term already.
__global__ void combine_heads_kernel(RowsParams p, const uint32_t *__restrict__ keys_h, int Rc, int tau0, int rows) {
  const int rr = blockIdx.x, bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (rr >= rows || !rows_pos_ok(p, b)) return;
  const int n = p.pos[b] + tau0 + rr + 1;
  const uint32_t *src = keys_h + (((size_t)b * p.Hkv * Rc + (size_t)g * Rc) * p.row_chunk + rr) * p.L_keys;
  const size_t plane = (size_t)p.row_chunk * p.L_keys;
  uint32_t *dst = p.keys + ((size_t)bg * p.row_chunk + rr) * p.L_keys;
  for (int s = threadIdx.x; s < n; s += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < Rc; ++r) acc += key_score(__ldcg(src + r * plane + s));
    dst[s] = score_key(acc);
  }
}

template <typename T, int DI>
static cudaError_t rows_topk_t(const RowsParams &p, cudaStream_t st, int key_limit, const RowsParams *ph) {
  constexpr int NT = 256;
  cudaError_t e = prepare_kernel(rows_select_kernel<NT>, (int)p.select_smem);
  if (e != cudaSuccess) return e;
  e = prepare_kernel(rows_score_kernel<T, DI>);
  if (e != cudaSuccess) return e;
  const RowsParams &ps = ph ? *ph : p;                // the geometry the scores are computed in
  for (int tau0 = 0; tau0 < p.T; tau0 += p.row_chunk) {
    const int rows = min(p.row_chunk, p.T - tau0);
    // prefill (pos 0): keys up to tau0 + rows; general positions: up to key_limit
    const int key_hi = p.require_pos0 ? min(key_limit, tau0 + rows) : key_limit;
    if constexpr (sizeof(T) == 2) {
      e = launch_rows_score_tc(ps, st, tau0, rows, key_hi);     // tensor cores (tcgen05)
      if (e != cudaSuccess) return e;
    } else {
      dim3 g1((key_hi + 63) / 64, (rows + 63) / 64, ps.B * ps.Hkv);   // fp32: CUDA cores, exact products
      rows_score_kernel<T, DI><<<g1, 256, 0, st>>>(ps, tau0, rows);
    }
    if (ph) {
      dim3 gc(rows, p.B * p.Hkv);
      combine_heads_kernel<<<gc, 256, 0, st>>>(p, ph->keys, ph->Hkv / p.Hkv, tau0, rows);
    }
    dim3 g2(rows, p.B * p.Hkv);
    rows_select_kernel<NT><<<g2, NT, p.select_smem, st>>>(p, tau0, rows);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_rows_topk(const RowsParams &p, int dtype, cudaStream_t st, int key_limit, const RowsParams *ph) {
  if (dtype == LISA_BF16) {
    if (p.DI == 64) return rows_topk_t<__nv_bfloat16, 64>(p, st, key_limit, ph);
    if (p.DI == 32) return rows_topk_t<__nv_bfloat16, 32>(p, st, key_limit, ph);
  } else {
    if (p.DI == 64) return rows_topk_t<float, 64>(p, st, key_limit, ph);
    if (p.DI == 32) return rows_topk_t<float, 32>(p, st, key_limit, ph);
  }
  return cudaErrorInvalidValue;
}

// ============================================================ attention + gate
// grid (T, B*Hkv); 256 threads.  Online softmax over tiles of 32 selected rows.
template <typename T, int D>
__global__ void __launch_bounds__(256) prefill_attend_kernel(RowsParams p) {
  constexpr int kRows = kAttnRows;
  constexpr int kDPL = D / 32;
  constexpr int kSlots = kMaxG / 8;   // heads per warp
  __shared__ __align__(16) T s_k[kRows][D];
  __shared__ __align__(16) T s_v[kRows][D];
  __shared__ float s_q[kMaxG][D];
  __shared__ float s_logit[kMaxG][kRows];
  __shared__ int s_idx[kRows];
  const int tau = blockIdx.x, bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (!rows_pos_ok(p, b)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  for (int i = tid; i < G * D; i += 256) {
    const int hh = i / D, dd = i % D;
    s_q[hh][dd] = Dt<T>::to_f(reinterpret_cast<const T *>(p.q)[(((size_t)b * p.T + tau) * p.Hq + g * G + hh) * D + dd]);
  }
  float m[kSlots], l[kSlots], acc[kSlots][kDPL];
#pragma unroll
  for (int s = 0; s < kSlots; ++s) {
    m[s] = -INFINITY;
    l[s] = 0.f;
#pragma unroll
    for (int j = 0; j < kDPL; ++j) acc[s][j] = 0.f;
  }
  const int *idx = p.idx + (((size_t)b * p.T + tau) * p.sel_heads + (p.sel_heads == 1 ? 0 : g)) * p.M;
  const T *kc = reinterpret_cast<const T *>(p.k_cache) + (size_t)bg * p.L_max * D;
  const T *vc = reinterpret_cast<const T *>(p.v_cache) + (size_t)bg * p.L_max * D;
  constexpr int kSlices = D * (int)sizeof(T) / 16;
  for (int tile = 0; tile < p.M / kRows; ++tile) {
    __syncthreads();
    if (tid < kRows) {
      int s = idx[tile * kRows + tid];
      if (s < -1 || s > p.pos[b] + tau) {
        set_err(p.err_word, LISA_DEVERR_CHECK);
        s = -1;
      }
      s_idx[tid] = s;
    }
    __syncthreads();
    if (s_idx[0] < 0) break;
    for (int i = tid; i < kRows * kSlices; i += 256) {
      const int r = i / kSlices, sl = i % kSlices;
      const int s = s_idx[r];
      uint4 uk = make_uint4(0, 0, 0, 0), uv = make_uint4(0, 0, 0, 0);
      if (s >= 0) {
        uk = *reinterpret_cast<const uint4 *>(kc + (size_t)s * D + sl * (16 / sizeof(T)));
        uv = *reinterpret_cast<const uint4 *>(vc + (size_t)s * D + sl * (16 / sizeof(T)));
      }
      reinterpret_cast<uint4 *>(&s_k[r][0])[sl] = uk;
      reinterpret_cast<uint4 *>(&s_v[r][0])[sl] = uv;
    }
    __syncthreads();
    for (int r = warp; r < kRows; r += 8) {
      float kx[kDPL];
#pragma unroll
      for (int j = 0; j < kDPL; ++j) kx[j] = Dt<T>::to_f(s_k[r][lane * kDPL + j]);
      const bool valid = s_idx[r] >= 0;
      for (int hh = 0; hh < G; ++hh) {
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < kDPL; ++j) dot = fmaf(s_q[hh][lane * kDPL + j], kx[j], dot);
        dot = warp_sum(dot);
        if (lane == 0) s_logit[hh][r] = valid ? dot * p.scale : -INFINITY;
      }
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < kSlots; ++s) {
      const int hh = warp + 8 * s;
      if (hh >= G) continue;
      const float x = s_logit[hh][lane];
      const float mt = warp_max(x);
      const float mn = fmaxf(m[s], mt);
      const float f = (m[s] == -INFINITY) ? 0.f : expf(m[s] - mn);
      const float e = (x == -INFINITY) ? 0.f : expf(x - mn);
      l[s] = l[s] * f + warp_sum(e);
      m[s] = mn;
#pragma unroll
      for (int j = 0; j < kDPL; ++j) acc[s][j] *= f;
      for (int r = 0; r < kRows; ++r) {
        const float pr = __shfl_sync(0xffffffffu, e, r);
#pragma unroll
        for (int j = 0; j < kDPL; ++j) acc[s][j] = fmaf(pr, Dt<T>::to_f(s_v[r][lane * kDPL + j]), acc[s][j]);
      }
    }
  }
#pragma unroll
  for (int s = 0; s < kSlots; ++s) {
    const int hh = warp + 8 * s;
    if (hh >= G) continue;
    const int h = g * G + hh;
    const size_t row = ((size_t)b * p.T + tau) * p.Hq + h;
    const float gam = 1.f / (1.f + expf(-p.gate[row]));
#pragma unroll
    for (int j = 0; j < kDPL; ++j) {
      const int dd = lane * kDPL + j;
      const float o_sp = acc[s][j] / l[s];
      const float o_lin = p.olin[row * D + dd];
      reinterpret_cast<T *>(p.out)[row * D + dd] = Dt<T>::from_f(gam * o_sp + (1.f - gam) * o_lin);
    }
  }
}

// ------------------------------------------------------------ bf16 on warp MMAs
// grid (T, B*Hkv); kAttnWarps warps.  Warp w owns a contiguous 1/kAttnWarps of
// the (b, tau, g) list, in tiles of 16 rows staged by cp.async (two stages per
// warp), flash-attention style with the selected rows as the M dimension of
// the warp MMAs and the G query heads as the N dimension (NHT tiles of 8
// heads): S^T = K Q^T, online softmax per head in registers, O^T += V^T P^T
// with P^T moved from the accumulator layout into the B-operand layout by 8x8
// transposes (movmatrix), P in bf16.  The warps' (max, sum, O) are merged
// through shared memory, then the gate mixes in o_lin.
constexpr int kAttnWarps = 1;   // warps per (b, t, g); each owns M / kAttnWarps selected rows


template <int D>
constexpr int attn_mma_smem() {
  // per warp: 2 stages x (K, V) x 16 rows x (2D + 16) bytes; the merge reuses it
  return kAttnWarps * 2 * 2 * 16 * (2 * D + 16);
}

// An 8x8 b16 matrix held one row pair per lane (lane l: row l / 4, columns
// 2 (l % 4), +1) -> its transpose in the same layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <int D, int NHT>
__global__ void __launch_bounds__(kAttnWarps * 32) prefill_attend_mma_kernel(RowsParams p) {
  extern __shared__ __align__(16) unsigned char s_att[];
  constexpr int RS = 2 * D + 16;                 // padded row stride (bytes)
  constexpr int TILE = 16 * RS;                  // one 16-row K or V tile
  constexpr int MT = D / 16;                     // 16-row tiles of O^T (head dim)
  const int tau = blockIdx.x, bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (!rows_pos_ok(p, b)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int hl = lane >> 2, kq = (lane & 3) * 2;
  const int RW = p.M / kAttnWarps;               // rows of this warp (a multiple of 16)
  const int t_abs = p.pos[b] + tau;
  const float scale2 = p.scale * kLog2e;         // logits in log2 units: e^x = 2^(x log2 e)
  unsigned char *wbuf = s_att + warp * 4 * TILE; // [stage][K | V]
  const uint32_t wbuf_u32 = smem_u32(wbuf);
  const int *idx = p.idx + (((size_t)b * p.T + tau) * p.sel_heads + (p.sel_heads == 1 ? 0 : g)) * p.M + warp * RW;
  const __nv_bfloat16 *kc = reinterpret_cast<const __nv_bfloat16 *>(p.k_cache) + (size_t)bg * p.L_max * D;
  const __nv_bfloat16 *vc = reinterpret_cast<const __nv_bfloat16 *>(p.v_cache) + (size_t)bg * p.L_max * D;

  // the epilogue's o_lin rows (written by the linear branch, G * D floats)
  // requested into L2 now, so that its loads do not wait on DRAM at the end
  {
    const float *olr = p.olin + (((size_t)b * p.T + tau) * p.Hq + g * G) * D;
    for (int i = tid * 32; i < G * D; i += kAttnWarps * 32 * 32) prefetch_l2(olr + i);
  }
  // B fragments of Q^T (k = head dim, n = query head) for every 16-wide k-step
  uint32_t qb[NHT][D / 16][2];
  {
    const uint32_t *q32 = reinterpret_cast<const uint32_t *>(reinterpret_cast<const __nv_bfloat16 *>(p.q) +
                                                             (((size_t)b * p.T + tau) * p.Hq + g * G) * D);
#pragma unroll
    for (int nh = 0; nh < NHT; ++nh) {
      const int h = nh * 8 + hl;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        qb[nh][ks][0] = h < G ? q32[(h * D + ks * 16 + kq) >> 1] : 0u;
        qb[nh][ks][1] = h < G ? q32[(h * D + ks * 16 + kq + 8) >> 1] : 0u;
      }
    }
  }
  // rows of tile i: positions (or -1), lanes 0..15 hold one each
  auto tile_pos = [&](int i) {
    int s = -1;
    if (lane < 16) {
      s = idx[i * 16 + lane];
      if (s < -1 || s > t_abs) {
        set_err(p.err_word, LISA_DEVERR_CHECK);
        s = -1;
      }
    }
    return s;
  };
  // cp.async 16 rows of K and V into stage i & 1; each warp instruction
  // copies two whole rows (16 lanes x 16 bytes each), so it touches few
  // cache lines (zero-filled where the slot holds no position)
  auto stage_tile = [&](int i, int my_pos) {
    const uint32_t kdst = wbuf_u32 + (i & 1) * 2 * TILE, vdst = kdst + TILE;
    constexpr int CH = 2 * D / 16;               // 16-byte chunks per row
#pragma unroll
    for (int c = lane; c < 16 * CH; c += 32) {
      const int r = c / CH, ch = c % CH;
      const int s = __shfl_sync(0xffffffffu, my_pos, r);
      const size_t off = (size_t)(s < 0 ? 0 : s) * D + ch * 8;
      cp_async16(kdst + r * RS + ch * 16, kc + off, s >= 0);
      cp_async16(vdst + r * RS + ch * 16, vc + off, s >= 0);
    }
    cp_async_commit();
  };

  // this lane: heads nh * 8 + kq, + 1 of every n-tile; rows hl and hl + 8 of a tile
  float mh[NHT][2], lh[NHT][2];
  float o[NHT][MT][4];
#pragma unroll
  for (int nh = 0; nh < NHT; ++nh) {
    mh[nh][0] = mh[nh][1] = -INFINITY;
    lh[nh][0] = lh[nh][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) o[nh][mt][0] = o[nh][mt][1] = o[nh][mt][2] = o[nh][mt][3] = 0.f;
  }

  const int ntiles = RW / 16;
  int pos_cur = tile_pos(0);
  const bool any0 = __any_sync(0xffffffffu, lane < 16 && pos_cur >= 0);
  int nvalid = any0 ? ntiles : 0;
  if (nvalid) stage_tile(0, pos_cur);
  for (int i = 0; i < nvalid; ++i) {
    int pos_next = -1;
    bool more = false;
    if (i + 1 < ntiles) {
      pos_next = tile_pos(i + 1);
      more = __any_sync(0xffffffffu, lane < 16 && pos_next >= 0);
    }
    if (more) {
      stage_tile(i + 1, pos_next);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
      nvalid = i + 1;                              // the list is -1 padded at its end
    }
    __syncwarp();
    const uint32_t kt = wbuf_u32 + (i & 1) * 2 * TILE, vt = kt + TILE;
    // S^T = K Q^T: 16 rows x 8 heads per n-tile
    float sc[NHT][4];
#pragma unroll
    for (int nh = 0; nh < NHT; ++nh) sc[nh][0] = sc[nh][1] = sc[nh][2] = sc[nh][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      ldmatrix_x4(kt + (lane & 15) * RS + ks * 32 + (lane >> 4) * 16, a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int nh = 0; nh < NHT; ++nh) mma_16816_bf16(sc[nh], a, qb[nh][ks]);
    }
    const int pr0 = __shfl_sync(0xffffffffu, pos_cur, hl), pr1 = __shfl_sync(0xffffffffu, pos_cur, hl + 8);
    uint32_t pb[NHT][2];
#pragma unroll
    for (int nh = 0; nh < NHT; ++nh) {
      // scale (in log2 units), mask; c0, c1: row hl (heads kq, kq + 1); c2, c3: row hl + 8
      float x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = (j < 2 ? pr0 : pr1) >= 0 ? sc[nh][j] * scale2 : -INFINITY;
      // the heads' maxima over the tile's 16 rows (lanes with the same lane % 4)
      float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(mh[nh][0], mx0), mn1 = fmaxf(mh[nh][1], mx1);
      // the accumulators need rescaling only where a running maximum moved
      const bool moved = __any_sync(0xffffffffu, mn0 != mh[nh][0] || mn1 != mh[nh][1]);
      const float f0 = mh[nh][0] == -INFINITY ? 0.f : exp2_approx(mh[nh][0] - mn0);
      const float f1 = mh[nh][1] == -INFINITY ? 0.f : exp2_approx(mh[nh][1] - mn1);
      mh[nh][0] = mn0;
      mh[nh][1] = mn1;
      const float e0 = x[0] == -INFINITY ? 0.f : exp2_approx(x[0] - mn0);
      const float e1 = x[1] == -INFINITY ? 0.f : exp2_approx(x[1] - mn1);
      const float e2 = x[2] == -INFINITY ? 0.f : exp2_approx(x[2] - mn0);
      const float e3 = x[3] == -INFINITY ? 0.f : exp2_approx(x[3] - mn1);
      lh[nh][0] = lh[nh][0] * f0 + e0 + e2;
      lh[nh][1] = lh[nh][1] * f1 + e1 + e3;
      if (moved) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[nh][mt][0] *= f0;
          o[nh][mt][1] *= f1;
          o[nh][mt][2] *= f0;
          o[nh][mt][3] *= f1;
        }
      }
      // P^T (k = rows, n = heads) as the B operand: transposes of the two 8x8 blocks
      pb[nh][0] = movmatrix_trans(pack_bf16(e0, e1));
      pb[nh][1] = movmatrix_trans(pack_bf16(e2, e3));
    }
    // O^T += V^T P^T: A = V^T (head dim x rows) by transposing matrix loads
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(vt + ((lane & 7) + 8 * (lane >> 4)) * RS + (mt * 16 + 8 * ((lane >> 3) & 1)) * 2, a[0], a[1],
                        a[2], a[3]);
#pragma unroll
      for (int nh = 0; nh < NHT; ++nh) mma_16816_bf16(o[nh][mt], a, pb[nh]);
    }
    __syncwarp();                                  // this stage may be refilled next
    pos_cur = pos_next;
  }
#pragma unroll
  for (int nh = 0; nh < NHT; ++nh)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      lh[nh][0] += __shfl_xor_sync(0xffffffffu, lh[nh][0], off);
      lh[nh][1] += __shfl_xor_sync(0xffffffffu, lh[nh][1], off);
    }

  // merge the warps: [warp][16 heads] max and sum, [warp][16][D] O
  __syncthreads();
  float *s_ml = reinterpret_cast<float *>(s_att);                 // [kAttnWarps][16][2]
  float *s_o = s_ml + kAttnWarps * 32;                            // [kAttnWarps][16][D]
#pragma unroll
  for (int nh = 0; nh < NHT; ++nh) {
    const int h0 = nh * 8 + kq;
    if (lane < 4) {
      s_ml[(warp * 16 + h0) * 2] = mh[nh][0];
      s_ml[(warp * 16 + h0) * 2 + 1] = lh[nh][0];
      s_ml[(warp * 16 + h0 + 1) * 2] = mh[nh][1];
      s_ml[(warp * 16 + h0 + 1) * 2 + 1] = lh[nh][1];
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int d = mt * 16 + hl;
      s_o[(warp * 16 + h0) * D + d] = o[nh][mt][0];
      s_o[(warp * 16 + h0 + 1) * D + d] = o[nh][mt][1];
      s_o[(warp * 16 + h0) * D + d + 8] = o[nh][mt][2];
      s_o[(warp * 16 + h0 + 1) * D + d + 8] = o[nh][mt][3];
    }
  }
  // per head, once: the warps' weights gam * 2^(m_w - m) / sum and 1 - gam
  float *s_cf = s_o + kAttnWarps * 16 * D;                        // [G][kAttnWarps + 1]
  if (tid < G) {
    const int hh = tid;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) mx = fmaxf(mx, s_ml[(w * 16 + hh) * 2]);
    float f[kAttnWarps], den = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      const float mw = s_ml[(w * 16 + hh) * 2];          // log2 units
      f[w] = mw == -INFINITY ? 0.f : exp2_approx(mw - mx);
      den = fmaf(f[w], s_ml[(w * 16 + hh) * 2 + 1], den);
    }
    const size_t row = ((size_t)b * p.T + tau) * p.Hq + g * G + hh;
    const float gam = 1.f / (1.f + expf(-p.gate[row]));
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) s_cf[hh * (kAttnWarps + 1) + w] = gam * f[w] / den;
    s_cf[hh * (kAttnWarps + 1) + kAttnWarps] = 1.f - gam;
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kAttnWarps * 32) {
    const int hh = i / D, d = i % D;
    const float *cf = s_cf + hh * (kAttnWarps + 1);
    const size_t row = ((size_t)b * p.T + tau) * p.Hq + g * G + hh;
    float o = cf[kAttnWarps] * p.olin[row * D + d];
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) o = fmaf(cf[w], s_o[(w * 16 + hh) * D + d], o);
    reinterpret_cast<__nv_bfloat16 *>(p.out)[row * D + d] = __float2bfloat16_rn(o);
  }
}

cudaError_t launch_prefill_attend(const RowsParams &p, int dtype, cudaStream_t st) {
  dim3 grid(p.T, p.B * p.Hkv);
  cudaError_t e;
  if (dtype == LISA_BF16 && p.M % (16 * kAttnWarps) == 0) {
    // query heads of a group as the MMAs' N: one n-tile of 8 heads, or two
    auto go = [&](auto kern, int smem) -> cudaError_t {
      cudaError_t e2 = prepare_kernel(kern, smem);
      if (e2 != cudaSuccess) return e2;
      kern<<<grid, kAttnWarps * 32, smem, st>>>(p);
      return cudaGetLastError();
    };
    if (p.D == 128)
      return p.G <= 8 ? go(prefill_attend_mma_kernel<128, 1>, attn_mma_smem<128>())
                      : go(prefill_attend_mma_kernel<128, 2>, attn_mma_smem<128>());
    return p.G <= 8 ? go(prefill_attend_mma_kernel<64, 1>, attn_mma_smem<64>())
                    : go(prefill_attend_mma_kernel<64, 2>, attn_mma_smem<64>());
  }
  if (dtype == LISA_BF16) {
    if (p.D == 128) {
      if ((e = prepare_kernel(prefill_attend_kernel<__nv_bfloat16, 128>)) != cudaSuccess) return e;
      prefill_attend_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(p);
    } else {
      if ((e = prepare_kernel(prefill_attend_kernel<__nv_bfloat16, 64>)) != cudaSuccess) return e;
      prefill_attend_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(p);
    }
  } else {
    if (p.D == 128) {
      if ((e = prepare_kernel(prefill_attend_kernel<float, 128>)) != cudaSuccess) return e;
      prefill_attend_kernel<float, 128><<<grid, 256, 0, st>>>(p);
    } else {
      if ((e = prepare_kernel(prefill_attend_kernel<float, 64>)) != cudaSuccess) return e;
      prefill_attend_kernel<float, 64><<<grid, 256, 0, st>>>(p);
    }
  }
  return cudaGetLastError();
}

}  // namespace lisa
