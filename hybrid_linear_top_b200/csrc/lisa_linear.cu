// Chunked linear attention for the LISA prefill (phi = identity, state matrix
// S_t; gptget.net digest of arXiv 2607.19358, method section), on sm_100a.
//
// With chunks of C = 64 tokens, the per-token recurrence S_t = S_{t-1} + k_t^T v_t,
// o_t = q_t S_t is evaluated as
//   dS_c   = K_c^T V_c                          (per KV head, all chunks at once)
//   P_c    = sum_{c' < c} dS_c'                 (exclusive prefix over chunks)
//   O_c    = Q_c (S_0 + P_c) + tril(Q_c K_c^T) V_c
//   S_T    = S_0 + sum_c dS_c
// which is the same sum, regrouped.  fp32 throughout.
#include "lisa_internal.h"
#include "lisa_common.cuh"

namespace lisa {

// grid (n_chunks, B*Hkv); dynamic smem 2 * C * D floats
template <typename T, int D>
__global__ void __launch_bounds__(256) lin_dS_kernel(RowsParams p) {
  extern __shared__ __align__(16) float s_lin[];
  constexpr int C = kLinChunk;
  constexpr int kB = D / 16;            // outputs per thread along i and j
  float *sk = s_lin;                    // [C][D]
  float *sv = s_lin + C * D;            // [C][D]
  const int c = blockIdx.x, bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (p.pos[b] != 0) return;
  const int t0 = c * C;
  const int n = min(C, p.T - t0);
  const int tid = threadIdx.x;
  for (int i = tid; i < C * D; i += 256) {
    const int r = i / D, j = i % D;
    float kx = 0.f, vx = 0.f;
    if (r < n) {
      const size_t src = (((size_t)b * p.T + t0 + r) * p.Hkv + g) * D + j;
      kx = Dt<T>::to_f(reinterpret_cast<const T *>(p.k)[src]);
      vx = Dt<T>::to_f(reinterpret_cast<const T *>(p.v)[src]);
    }
    sk[i] = kx;
    sv[i] = vx;
  }
  __syncthreads();
  const int ti = tid / 16, tj = tid % 16;
  float acc[kB][kB];
#pragma unroll
  for (int a = 0; a < kB; ++a)
#pragma unroll
    for (int bb = 0; bb < kB; ++bb) acc[a][bb] = 0.f;
  for (int r = 0; r < n; ++r) {
    float ki[kB], vj[kB];
#pragma unroll
    for (int a = 0; a < kB; ++a) ki[a] = sk[r * D + ti * kB + a];
#pragma unroll
    for (int a = 0; a < kB; ++a) vj[a] = sv[r * D + tj * kB + a];
#pragma unroll
    for (int a = 0; a < kB; ++a)
#pragma unroll
      for (int bb = 0; bb < kB; ++bb) acc[a][bb] = fmaf(ki[a], vj[bb], acc[a][bb]);
  }
  const int nc = (p.T + C - 1) / C;
  float *dst = p.dS + ((size_t)bg * nc + c) * D * D;
#pragma unroll
  for (int a = 0; a < kB; ++a)
#pragma unroll
    for (int bb = 0; bb < kB; ++bb) dst[(ti * kB + a) * D + tj * kB + bb] = acc[a][bb];
}

// grid (D*D/256, B*Hkv): exclusive prefix over the chunks of `chunk` tokens,
// in place; total -> Ptot
template <int D>
__global__ void __launch_bounds__(256) lin_prefix_kernel(RowsParams p, int chunk) {
  const int e = blockIdx.x * 256 + threadIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv;
  if (p.pos[b] != 0) return;
  const int nc = (p.T + chunk - 1) / chunk;
  float *base = p.dS + (size_t)bg * nc * D * D + e;
  float run = 0.f;
  constexpr int kBatch = 16;
  for (int c0 = 0; c0 < nc; c0 += kBatch) {
    float x[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) x[i] = (c0 + i < nc) ? base[(size_t)(c0 + i) * D * D] : 0.f;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (c0 + i < nc) {
        base[(size_t)(c0 + i) * D * D] = run;
        run += x[i];
      }
    }
  }
  p.Ptot[(size_t)bg * D * D + e] = run;
}

// grid (n_chunks, Hq, B); dynamic smem: Q, K, V chunks [C][D], A [C][C+1], S tile [16][D]
template <typename T, int D>
__global__ void __launch_bounds__(256) lin_out_kernel(RowsParams p) {
  extern __shared__ __align__(16) float s_lin[];
  constexpr int C = kLinChunk;
  float *sq = s_lin;                       // [C][D]
  float *sk = sq + C * D;                  // [C][D]
  float *sv = sk + C * D;                  // [C][D]
  float *sa = sv + C * D;                  // [C][C+1]
  float *ss = sa + C * (C + 1);            // [16][D]
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (p.pos[b] != 0) return;
  const int g = h / p.G;
  const int bg = b * p.Hkv + g;
  const int t0 = c * C;
  const int n = min(C, p.T - t0);
  const int tid = threadIdx.x;
  for (int i = tid; i < C * D; i += 256) {
    const int r = i / D, j = i % D;
    float qx = 0.f, kx = 0.f, vx = 0.f;
    if (r < n) {
      const size_t t = (size_t)b * p.T + t0 + r;
      qx = Dt<T>::to_f(reinterpret_cast<const T *>(p.q)[(t * p.Hq + h) * D + j]);
      kx = Dt<T>::to_f(reinterpret_cast<const T *>(p.k)[(t * p.Hkv + g) * D + j]);
      vx = Dt<T>::to_f(reinterpret_cast<const T *>(p.v)[(t * p.Hkv + g) * D + j]);
    }
    sq[i] = qx;
    sk[i] = kx;
    sv[i] = vx;
  }
  __syncthreads();
  // A = tril(Q K^T): thread computes a 4x4 block
  {
    const int ai = (tid / 16) * 4, aj = (tid % 16) * 4;
    float a[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) a[x][y] = 0.f;
    for (int e = 0; e < D; ++e) {
      float qa[4], kb[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) qa[x] = sq[(ai + x) * D + e];
#pragma unroll
      for (int y = 0; y < 4; ++y) kb[y] = sk[(aj + y) * D + e];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) a[x][y] = fmaf(qa[x], kb[y], a[x][y]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) sa[(ai + x) * (C + 1) + aj + y] = (aj + y <= ai + x) ? a[x][y] : 0.f;
  }
  __syncthreads();
  // O = A V + Q (S0 + P_c): thread owns rows oi..oi+3, columns oj..oj+kJ-1
  constexpr int kJ = D / 32;
  const int oi = (tid / 32) * 8;          // 8 row groups of 8 rows
  const int oj = (tid % 32) * kJ;
  float o[8][kJ];
#pragma unroll
  for (int x = 0; x < 8; ++x)
#pragma unroll
    for (int y = 0; y < kJ; ++y) o[x][y] = 0.f;
  for (int r = 0; r < C; ++r) {
    float vv[kJ];
#pragma unroll
    for (int y = 0; y < kJ; ++y) vv[y] = sv[r * D + oj + y];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const float ax = sa[(oi + x) * (C + 1) + r];
#pragma unroll
      for (int y = 0; y < kJ; ++y) o[x][y] = fmaf(ax, vv[y], o[x][y]);
    }
  }
  const int nc = (p.T + C - 1) / C;
  const float *S0 = p.state + ((size_t)b * p.Hq + h) * D * D;
  const float *Pc = p.dS + ((size_t)bg * nc + c) * D * D;
  for (int i0 = 0; i0 < D; i0 += 16) {
    __syncthreads();
    for (int i = tid; i < 16 * D; i += 256) ss[i] = S0[(size_t)i0 * D + i] + Pc[(size_t)i0 * D + i];
    __syncthreads();
    for (int ii = 0; ii < 16; ++ii) {
      float sr[kJ];
#pragma unroll
      for (int y = 0; y < kJ; ++y) sr[y] = ss[ii * D + oj + y];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const float qx = sq[(oi + x) * D + i0 + ii];
#pragma unroll
        for (int y = 0; y < kJ; ++y) o[x][y] = fmaf(qx, sr[y], o[x][y]);
      }
    }
  }
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const int r = oi + x;
    if (r >= n) continue;
    float *dst = p.olin + (((size_t)b * p.T + t0 + r) * p.Hq + h) * D + oj;
#pragma unroll
    for (int y = 0; y < kJ; ++y) dst[y] = o[x][y];
  }
}

// grid (D*D/256, Hq, B): S_T = S_0 + Ptot
template <int D>
__global__ void __launch_bounds__(256) lin_state_kernel(RowsParams p) {
  const int e = blockIdx.x * 256 + threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  if (p.pos[b] != 0) return;
  const int g = h / p.G;
  float *S = p.state + ((size_t)b * p.Hq + h) * D * D;
  S[e] = S[e] + p.Ptot[((size_t)b * p.Hkv + g) * D * D + e];
}

template <typename T, int D>
static cudaError_t prefill_linear_t(const RowsParams &p, cudaStream_t st) {
  constexpr int C = kLinChunk;
  const int nc = (p.T + C - 1) / C;
  const size_t smem1 = 2 * C * D * sizeof(float);
  const size_t smem3 = (3 * C * D + C * (C + 1) + 16 * D) * sizeof(float);
  cudaError_t e = prepare_kernel(lin_dS_kernel<T, D>, (int)smem1);
  if (e != cudaSuccess) return e;
  if ((e = prepare_kernel(lin_out_kernel<T, D>, (int)smem3)) != cudaSuccess) return e;
  if ((e = prepare_kernel(lin_prefix_kernel<D>)) != cudaSuccess) return e;
  if ((e = prepare_kernel(lin_state_kernel<D>)) != cudaSuccess) return e;
  lin_dS_kernel<T, D><<<dim3(nc, p.B * p.Hkv), 256, smem1, st>>>(p);
  lin_prefix_kernel<D><<<dim3(D * D / 256, p.B * p.Hkv), 256, 0, st>>>(p, C);
  lin_out_kernel<T, D><<<dim3(nc, p.Hq, p.B), 256, smem3, st>>>(p);
  lin_state_kernel<D><<<dim3(D * D / 256, p.Hq, p.B), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_lin_prefix(const RowsParams &p, cudaStream_t st, int chunk) {
  if (p.D != 128) return cudaErrorInvalidValue;
  cudaError_t e = prepare_kernel(lin_prefix_kernel<128>);
  if (e != cudaSuccess) return e;
  lin_prefix_kernel<128><<<dim3(128 * 128 / 256, p.B * p.Hkv), 256, 0, st>>>(p, chunk);
  return cudaGetLastError();
}

cudaError_t launch_lin_state(const RowsParams &p, cudaStream_t st) {
  if (p.D != 128) return cudaErrorInvalidValue;
  cudaError_t e = prepare_kernel(lin_state_kernel<128>);
  if (e != cudaSuccess) return e;
  lin_state_kernel<128><<<dim3(128 * 128 / 256, p.Hq, p.B), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_prefill_linear(const RowsParams &p, int dtype, cudaStream_t st) {
  if (dtype == LISA_BF16) {
    if (p.D == 128) return launch_prefill_linear_tc(p, st);
    if (p.D == 64) return prefill_linear_t<__nv_bfloat16, 64>(p, st);
  } else {
    if (p.D == 128) return prefill_linear_t<float, 128>(p, st);
    if (p.D == 64) return prefill_linear_t<float, 64>(p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lisa
