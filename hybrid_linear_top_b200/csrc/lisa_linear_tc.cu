// Chunked linear attention of the LISA prefill on the sm_100a tensor cores
// (tcgen05, bf16 operands, fp32 accumulation in tensor memory), d = 128,
// chunks of 128 tokens.
//
// phi = identity with a state matrix S_t (gptget.net digest of arXiv
// 2607.19358, method section).  With chunks c of C tokens the per-token
// recurrence S_t = S_{t-1} + k_t^T v_t, o_t = q_t S_t is regrouped as
//   dS_c = K_c^T V_c,  P_c = sum_{c' < c} dS_c',
//   O_c  = Q_c (S_0 + P_c) + tril(Q_c K_c^T) V_c,   S_T = S_0 + sum_c dS_c.
// The state operand S_0 + P_c and the masked scores are fed to the tensor
// cores as bf16 hi + lo pairs (x = hi + lo, each product accumulated in fp32),
// which keeps them close to fp32 accuracy.
#include "lisa_internal.h"
#include "lisa_tc.cuh"

namespace lisa {

constexpr int kLC = 128;                  // chunk length of this path
constexpr int kHalf = kLC * 128;          // bytes of one 64-column half of a [128][128] bf16 tile

__device__ __forceinline__ uint32_t pack_bf16x2(float lo_elem, float hi_elem) {
  const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo_elem));
  const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi_elem));
  return a | (b << 16);
}
// x ~ hi + lo with hi = bf16(x), lo = bf16(x - hi); packs 8 consecutive values each.
__device__ __forceinline__ void split8(const float *x, uint4 &hi, uint4 &lo) {
  float h[8], l[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    h[j] = __bfloat162float(__float2bfloat16_rn(x[j]));
    l[j] = x[j] - h[j];
  }
  hi = make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
  lo = make_uint4(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]), pack_bf16x2(l[4], l[5]), pack_bf16x2(l[6], l[7]));
}

// ---------------------------------------------------------------- dS_c = K_c^T V_c
// grid (n_chunks, B*Hkv), 256 threads.  A = K_c^T and B = V_c are both MN-major
// views of the TMA-loaded [tokens][d] tiles.
__global__ void __launch_bounds__(256, 1)
    lin_dS_tc_kernel(const __grid_constant__ RowsParams p, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int c = blockIdx.x, bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  if (p.pos[b] != 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  unsigned char *ks = smem, *vs = smem + 2 * kHalf;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 4 * kHalf);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2);
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tc_alloc(tmem_slot, 128);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], 4 * kHalf);
    for (int h = 0; h < 2; ++h) {
      tma_load_4d(ks + h * kHalf, &kmap, h * 64, g, c * kLC, b, &bars[0]);
      tma_load_4d(vs + h * kHalf, &vmap, h * 64, g, c * kLC, b, &bars[0]);
    }
    if (!mbar_wait_bounded(&bars[0], 0)) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
    tc_fence_after();
    const uint32_t idesc = tc_idesc_bf16(128, 128, true, true);
#pragma unroll
    for (int kk = 0; kk < kLC / 16; ++kk)
      tc_mma_bf16(tmem, tc_sdesc_mnmajor(smem_u32(ks) + kk * 2048, kHalf),
                  tc_sdesc_mnmajor(smem_u32(vs) + kk * 2048, kHalf), idesc, kk > 0);
    tc_commit(&bars[1]);
  }
  if (!mbar_wait_bounded(&bars[1], 0) && lane == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
  __syncwarp();   // the TMEM loads below are warp-collective
  tc_fence_after();
  // row i of dS = TMEM lane i; warps w and w+4 share the lanes, split the columns
  const int i = (warp & 3) * 32 + lane;
  const int nc = (p.T + kLC - 1) / kLC;
  float *dst = p.dS + ((size_t)bg * nc + c) * 128 * 128 + (size_t)i * 128;
  for (int col = (warp >> 2) * 64; col < (warp >> 2) * 64 + 64; col += 16) {
    uint32_t v[16];
    tc_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + col, v);
    tc_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<float4 *>(dst + col + 4 * q) = make_float4(
          __uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
          __uint_as_float(v[4 * q + 3]));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------- O_c
// grid (n_chunks, Hq, B), 256 threads.
//   D1  = Q_c K_c^T                       (TMEM columns [0, 128))
//   OUT = Q_c (S_0 + P_c) + tril(D1) V_c  (TMEM columns [128, 256))
__global__ void __launch_bounds__(256, 1)
    lin_out_tc_kernel(const __grid_constant__ RowsParams p, const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (p.pos[b] != 0) return;
  const int g = h / p.G, bg = b * p.Hkv + g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  unsigned char *qs = smem;                    // Q_c          [tokens][d]  K-major
  unsigned char *kv = smem + 2 * kHalf;        // K_c, then the masked scores (hi) [tokens][tokens]
  unsigned char *vs = smem + 4 * kHalf;        // V_c          [tokens][d]  MN-major B
  unsigned char *shi = smem + 6 * kHalf;       // S_0 + P_c hi [i][j]       MN-major B
  unsigned char *slo = smem + 8 * kHalf;       // S_0 + P_c lo
  unsigned char *alo = smem + 10 * kHalf;      // masked scores (lo)
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 12 * kHalf);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3);
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tc_alloc(tmem_slot, 256);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], 6 * kHalf);
    for (int hh = 0; hh < 2; ++hh) {
      tma_load_4d(qs + hh * kHalf, &qmap, hh * 64, h, c * kLC, b, &bars[0]);
      tma_load_4d(kv + hh * kHalf, &kmap, hh * 64, g, c * kLC, b, &bars[0]);
      tma_load_4d(vs + hh * kHalf, &vmap, hh * 64, g, c * kLC, b, &bars[0]);
    }
  }
  // S_0 + P_c -> bf16 hi / lo in the MN-major swizzled layout (rows i, columns j)
  {
    const int nc = (p.T + kLC - 1) / kLC;
    const float *S0 = p.state + ((size_t)b * p.Hq + h) * 128 * 128;
    const float *Pc = p.dS + ((size_t)bg * nc + c) * 128 * 128;
    // 8 items of 8 columns per thread, in two batches of 4: the 16 loads of a
    // batch are all in flight before any of them is used
    constexpr int kBatch = 4;
    for (int base = tid; base < 128 * 16; base += 256 * kBatch) {
      float4 a[kBatch][2], bq[kBatch][2];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int item = base + k * 256, i = item >> 4, j0 = (item & 15) * 8;
        a[k][0] = *reinterpret_cast<const float4 *>(S0 + i * 128 + j0);
        a[k][1] = *reinterpret_cast<const float4 *>(S0 + i * 128 + j0 + 4);
        bq[k][0] = *reinterpret_cast<const float4 *>(Pc + i * 128 + j0);
        bq[k][1] = *reinterpret_cast<const float4 *>(Pc + i * 128 + j0 + 4);
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int item = base + k * 256, i = item >> 4, j0 = (item & 15) * 8;
        float x[8];
        x[0] = a[k][0].x + bq[k][0].x; x[1] = a[k][0].y + bq[k][0].y;
        x[2] = a[k][0].z + bq[k][0].z; x[3] = a[k][0].w + bq[k][0].w;
        x[4] = a[k][1].x + bq[k][1].x; x[5] = a[k][1].y + bq[k][1].y;
        x[6] = a[k][1].z + bq[k][1].z; x[7] = a[k][1].w + bq[k][1].w;
        uint4 hi, lo;
        split8(x, hi, lo);
        const uint32_t off = sw128_offset(i, j0, kHalf);
        *reinterpret_cast<uint4 *>(shi + off) = hi;
        *reinterpret_cast<uint4 *>(slo + off) = lo;
      }
    }
  }
  fence_async_shared();
  __syncthreads();
  if (tid == 0) {
    if (!mbar_wait_bounded(&bars[0], 0)) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
    tc_fence_after();
    const uint32_t id_kk = tc_idesc_bf16(128, 128, false, false);
    const uint32_t id_kmn = tc_idesc_bf16(128, 128, false, true);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {            // D1 = Q K^T, K = d
      const int hh = ks >> 2, kk = ks & 3;
      tc_mma_bf16(tmem, tc_sdesc_kmajor(smem_u32(qs + hh * kHalf), 128) + 2 * kk,
                  tc_sdesc_kmajor(smem_u32(kv + hh * kHalf), 128) + 2 * kk, id_kk, ks > 0);
    }
    tc_commit(&bars[1]);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {            // OUT = Q S_hi + Q S_lo, K = i
      const int hh = ks >> 2, kk = ks & 3;
      const uint64_t a = tc_sdesc_kmajor(smem_u32(qs + hh * kHalf), 128) + 2 * kk;
      tc_mma_bf16(tmem + 128, a, tc_sdesc_mnmajor(smem_u32(shi) + ks * 2048, kHalf), id_kmn, ks > 0);
      tc_mma_bf16(tmem + 128, a, tc_sdesc_mnmajor(smem_u32(slo) + ks * 2048, kHalf), id_kmn, 1);
    }
  }
  // masked scores: row tau keeps keys j <= tau; hi / lo into the K-major A layout
  if (!mbar_wait_bounded(&bars[1], 0) && lane == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
  __syncwarp();   // the TMEM loads below are warp-collective
  tc_fence_after();
  {
    const int tau = (warp & 3) * 32 + lane;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    for (int col = (warp >> 2) * 64; col < (warp >> 2) * 64 + 64; col += 16) {
      uint32_t v[16];
      tc_ld16(tmem + lane_base + col, v);
      tc_wait_ld();
#pragma unroll
      for (int half8 = 0; half8 < 2; ++half8) {
        float x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int key = col + half8 * 8 + j;
          x[j] = key <= tau ? __uint_as_float(v[half8 * 8 + j]) : 0.f;
        }
        uint4 hi, lo;
        split8(x, hi, lo);
        const uint32_t off = sw128_offset(tau, col + half8 * 8, kHalf);
        *reinterpret_cast<uint4 *>(kv + off) = hi;     // K_c is no longer read (D1 is complete)
        *reinterpret_cast<uint4 *>(alo + off) = lo;
      }
    }
  }
  fence_async_shared();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    const uint32_t id_kmn = tc_idesc_bf16(128, 128, false, true);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {            // OUT += A_hi V + A_lo V, K = key
      const int hh = ks >> 2, kk = ks & 3;
      const uint64_t bv = tc_sdesc_mnmajor(smem_u32(vs) + ks * 2048, kHalf);
      tc_mma_bf16(tmem + 128, tc_sdesc_kmajor(smem_u32(kv + hh * kHalf), 128) + 2 * kk, bv, id_kmn, 1);
      tc_mma_bf16(tmem + 128, tc_sdesc_kmajor(smem_u32(alo + hh * kHalf), 128) + 2 * kk, bv, id_kmn, 1);
    }
    tc_commit(&bars[2]);
  }
  if (!mbar_wait_bounded(&bars[2], 0) && lane == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
  __syncwarp();   // the TMEM loads below are warp-collective
  tc_fence_after();
  {
    const int tau = (warp & 3) * 32 + lane;
    const int t = c * kLC + tau;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float *dst = p.olin + (((size_t)b * p.T + (t < p.T ? t : 0)) * p.Hq + h) * 128;
    for (int col = (warp >> 2) * 64; col < (warp >> 2) * 64 + 64; col += 16) {
      uint32_t v[16];
      tc_ld16(tmem + lane_base + 128 + col, v);
      tc_wait_ld();
      if (t < p.T) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4 *>(dst + col + 4 * q) = make_float4(
              __uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
              __uint_as_float(v[4 * q + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(tmem, 256);
  }
}

// 4-D tensor map over x [B, T, H, 128] (bf16), box {64, 1, 128, 1}: 128 tokens x
// 64 features of one head, out-of-range tokens read as zero.
static bool map_tokens(CUtensorMap *m, const void *x, int B, int T, int H) {
  const unsigned long long dims[4] = {128, (unsigned long long)H, (unsigned long long)T, (unsigned long long)B};
  const unsigned long long str[3] = {256, (unsigned long long)H * 256, (unsigned long long)T * H * 256};
  const unsigned box[4] = {64, 1, (unsigned)kLC, 1};
  return make_tmap(m, x, 2, 4, dims, str, box, 128);
}

cudaError_t launch_prefill_linear_tc(const RowsParams &p, cudaStream_t st) {
  if (p.D != 128) return cudaErrorInvalidValue;
  CUtensorMap qm, km, vm;
  if (!map_tokens(&qm, p.q, p.B, p.T, p.Hq) || !map_tokens(&km, p.k, p.B, p.T, p.Hkv) ||
      !map_tokens(&vm, p.v, p.B, p.T, p.Hkv))
    return cudaErrorInvalidValue;
  const int nc = (p.T + kLC - 1) / kLC;
  const int smem1 = 1024 + 4 * kHalf + 64;
  const int smem3 = 1024 + 12 * kHalf + 64;
  cudaError_t e = prepare_kernel(lin_dS_tc_kernel, smem1);
  if (e != cudaSuccess) return e;
  if ((e = prepare_kernel(lin_out_tc_kernel, smem3)) != cudaSuccess) return e;
  lin_dS_tc_kernel<<<dim3(nc, p.B * p.Hkv), 256, smem1, st>>>(p, km, vm);
  if ((e = launch_lin_prefix(p, st, kLC)) != cudaSuccess) return e;
  lin_out_tc_kernel<<<dim3(nc, p.Hq, p.B), 256, smem3, st>>>(p, qm, km, vm);
  if ((e = launch_lin_state(p, st)) != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lisa
