// Projection GEMMs of the layer on the sm_100a tensor cores (tcgen05): the
// front-end that maps the hidden state to q, k, v, the indexer's queries, keys
// and head weights and the gate logits, and the output projection back to the
// hidden size.
//
// Method: arXiv 2607.19358 (LISA).  The abstract and the gptget.net digest's
// method section name these inputs as projections of the hidden state and
// give no fused form; the library reads the front-end as one linear map whose
// output columns are [q | k | v | qidx | kidx | w | lambda] (lisa.h).
//
// Z[rows x N] = X[rows x K] W^T with X and W (N x K, out-features x
// in-features) bf16 and K-major, fp32 accumulation in tensor memory.  Tiles
// of 128 rows x BN columns; one persistent CTA per SM walks its share of
// them: warp 0 lane 0 loads 64-wide K blocks of X and W through a TMA ring
// (128-byte swizzle), warp 1 lane 0 issues the MMAs (M = 128, N = BN, K = 16
// per instruction) into one of two TMEM accumulator buffers and owns the TMEM
// columns, and warps 4-7 (one TMEM lane quadrant each, one row per thread)
// write a finished tile to the column segments' own dense arrays (bf16 or
// fp32) while the MMAs of the next tile fill the other buffer.
// BN = 256 for many rows (the contraction is tensor-bound), BN = 32 up to 128.
// A decode step projects a few rows, which is bound by HBM (every weight read
// once), not by the tensor cores: 3 to 32 rows take the weights as the M
// operand with K split over a cluster (proj_swap_tc_kernel), 1 or 2 rows a
// CUDA-core weight stream (proj_gemv_kernel).
#include <cooperative_groups.h>

#include <algorithm>

#include "lisa_internal.h"
#include "lisa_tc.cuh"

namespace cg = cooperative_groups;

namespace lisa {

constexpr int kProjThreads = 256;
constexpr int kProjRows = 128;
constexpr int kProjKB = 64;     // K elements per block (128 bytes of bf16 = the swizzle span)

template <int BN>
struct ProjGeom {
  static constexpr int kStages = BN >= 256 ? 4 : 6;
  static constexpr int kABytes = kProjRows * kProjKB * 2;
  static constexpr int kBBytes = BN * kProjKB * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + 256;
};

__device__ __forceinline__ void proj_store(const ProjParams &p, int row, int col, float v) {
  for (int s = 0; s < p.nseg; ++s) {
    const ProjSeg &g = p.seg[s];
    if (col >= g.c0 && col < g.c0 + g.width) {
      const size_t off = (size_t)row * g.width + (col - g.c0);
      if (g.f32) reinterpret_cast<float *>(g.ptr)[off] = v;
      else reinterpret_cast<__nv_bfloat16 *>(g.ptr)[off] = __float2bfloat16_rn(v);
      return;
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_tc_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ CUtensorMap xmap,
                   const __grid_constant__ CUtensorMap wmap) {
  using PG = ProjGeom<BN>;
  constexpr int S = PG::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * PG::kStageBytes);
  uint64_t *full = bars, *empty = bars + S, *acc_full = bars + 2 * S, *acc_empty = bars + 2 * S + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntn = (p.N + BN - 1) / BN;
  const int ntiles = ntn * ((p.rows + kProjRows - 1) / kProjRows);
  const int nk = (p.K + kProjKB - 1) / kProjKB;
  constexpr uint32_t kCols = 2 * BN;               // two accumulator buffers

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4 * 32);            // every epilogue thread has read the buffer
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, kCols);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Persistent: CTA c takes tiles c, c + gridDim.x, ...; tile = (row block, column block).
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;                                   // K blocks issued so far (ring position)
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int row0 = (tile / ntn) * kProjRows, col0 = (tile % ntn) * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % S;
          if (it >= S && !mbar_wait_bounded(&empty[st], (uint32_t)(((it / S) - 1) & 1)))
            set_err(p.err_word, LISA_DEVERR_TIMEOUT);
          unsigned char *a = smem + st * PG::kStageBytes;
          mbar_arrive_expect_tx(&full[st], (uint32_t)PG::kStageBytes);   // whole boxes land, out of range zero
          tma_load_2d(a, &xmap, kb * kProjKB, row0, &full[st]);
          tma_load_2d(a + PG::kABytes, &wmap, kb * kProjKB, col0, &full[st]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc_idesc_bf16(kProjRows, BN);
      int it = 0, lt = 0;                           // K blocks consumed, tiles done by this CTA
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
        const int buf = lt & 1;
        if (lt >= 2 && !mbar_wait_bounded(&acc_empty[buf], (uint32_t)(((lt >> 1) - 1) & 1)))
          set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % S;
          if (!mbar_wait_bounded(&full[st], (uint32_t)((it / S) & 1))) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
          tc_fence_after();
          const uint32_t a = smem_u32(smem + st * PG::kStageBytes);
          const uint64_t adesc = tc_sdesc_kmajor(a, 128), bdesc = tc_sdesc_kmajor(a + PG::kABytes, 128);
#pragma unroll
          for (int ks = 0; ks < kProjKB / 16; ++ks)   // +32 bytes along K inside the swizzle atom
            tc_mma_bf16(tmem + (uint32_t)(buf * BN), adesc + 2 * ks, bdesc + 2 * ks, idesc, (kb | ks) != 0);
          tc_commit(&empty[st]);                    // the stage may be refilled once these MMAs are done
        }
        tc_commit(&acc_full[buf]);                  // this tile's accumulator is complete
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: thread = row
    // overlaps the MMAs of the next tile, which go to the other buffer
    const int quad = warp - 4;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    int lt = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
      const int buf = lt & 1;
      const int row = (tile / ntn) * kProjRows + quad * 32 + lane, col0 = (tile % ntn) * BN;
      if (!mbar_wait_bounded(&acc_full[buf], (uint32_t)((lt >> 1) & 1)) && lane == 0)
        set_err(p.err_word, LISA_DEVERR_TIMEOUT);
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN; c += 16) {
        uint32_t v[16];
        tc_ld16(tmem + lane_base + (uint32_t)(buf * BN + c), v);
        tc_wait_ld();
        const int gc = col0 + c;
        if (row >= p.rows || gc >= p.N) continue;
        // the 16 columns inside one bf16 segment, 16-column aligned in it: two 16-byte stores
        int s = 0;
        while (s < p.nseg && !(gc >= p.seg[s].c0 && gc < p.seg[s].c0 + p.seg[s].width)) ++s;
        const bool vec = s < p.nseg && !p.seg[s].f32 && gc + 16 <= p.seg[s].c0 + p.seg[s].width &&
                         ((gc - p.seg[s].c0) & 15) == 0 && (p.seg[s].width & 7) == 0;
        if (vec) {
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.seg[s].ptr) +
                                                 (size_t)row * p.seg[s].width + (gc - p.seg[s].c0));
          dst[0] = make_uint4(pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1])),
                              pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3])),
                              pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5])),
                              pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7])));
          dst[1] = make_uint4(pack_bf16(__uint_as_float(v[8]), __uint_as_float(v[9])),
                              pack_bf16(__uint_as_float(v[10]), __uint_as_float(v[11])),
                              pack_bf16(__uint_as_float(v[12]), __uint_as_float(v[13])),
                              pack_bf16(__uint_as_float(v[14]), __uint_as_float(v[15])));
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (gc + j < p.N) proj_store(p, row, gc + j, __uint_as_float(v[j]));
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);                 // the MMAs of tile lt + 2 may overwrite the buffer
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tc_dealloc(tmem, kCols);
  }
}

template <int BN>
static cudaError_t proj_t(const ProjParams &p, const void *x, const void *W, cudaStream_t st) {
  using PG = ProjGeom<BN>;
  cudaError_t e = prepare_kernel(proj_tc_kernel<BN>, PG::kSmem);
  if (e != cudaSuccess) return e;
  CUtensorMap xmap, wmap;
  if (!make_tmap_2d(&xmap, x, 2, (unsigned long long)p.K, (unsigned long long)p.rows, (unsigned long long)p.K * 2,
                    kProjKB, kProjRows, 128) ||
      !make_tmap_2d(&wmap, W, 2, (unsigned long long)p.K, (unsigned long long)p.N, (unsigned long long)p.K * 2,
                    kProjKB, BN, 128))
    return cudaErrorInvalidValue;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  const int ntiles = ((p.N + BN - 1) / BN) * ((p.rows + kProjRows - 1) / kProjRows);
  proj_tc_kernel<BN><<<std::min(ntiles, sms), kProjThreads, PG::kSmem, st>>>(p, xmap, wmap);   // persistent
  return cudaGetLastError();
}

// ============================================================ few rows: weight stream
// A decode step projects at most a few rows: Z = X W^T then reads every
// weight once and does 2 * rows flops per weight, so it is bound by HBM, not
// by the tensor cores.  A CTA owns CPC consecutive output columns, whose
// weight rows form one contiguous block: a producer warp streams it through a
// ring of kGemvStages shared-memory stages ([CPC rows][256 K] tiles, 2-D TMA,
// no swizzle), and 8 consumer warps (CPC / 8 columns each) take 16-byte
// chunks of the tile and of X (one bulk copy into shared memory, bf16) per
// lane.
// A warp reduction per (row, column) gives the result.
constexpr int kGemvWarps = 8;      // consumer warps; one more warp produces
constexpr int kGemvRowsMax = 2;    // rows handled by this path at most
constexpr int kGemvKB = 256;       // K elements per stage tile (512 bytes per weight row)

template <int CPC>
struct GemvGeom {
  static constexpr int F = CPC / kGemvWarps;             // columns per consumer warp
  static constexpr int kTile = CPC * kGemvKB * 2;        // bytes per stage
  static constexpr int kStages = 65536 / kTile;          // 64 KB of weights in flight per CTA
};

template <int CPC>
__host__ __device__ inline int gemv_smem_bytes(int rows, int K) {
  return 1024 + GemvGeom<CPC>::kStages * GemvGeom<CPC>::kTile + 256 + rows * K * 2;
}

template <int CPC>
__global__ void __launch_bounds__((kGemvWarps + 1) * 32)
    proj_gemv_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ CUtensorMap wmap,
                     const __nv_bfloat16 *__restrict__ x) {
  using GG = GemvGeom<CPC>;
  constexpr int F = GG::F, S = GG::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * GG::kTile);
  uint64_t *full = bars, *empty = bars + S, *x_full = bars + 2 * S;
  uint4 *xs = reinterpret_cast<uint4 *>(smem + S * GG::kTile + 256);   // [rows][K / 8]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nK = p.K / 8;
  const int nkb = (p.K + kGemvKB - 1) / kGemvKB;
  const int n0 = blockIdx.x * CPC;

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kGemvWarps);
    }
    mbar_init(x_full, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == kGemvWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // X in one bulk copy (rows * K * 2 bytes, a multiple of 16), then the weight tiles
      const uint32_t xbytes = (uint32_t)(p.rows * p.K * 2);
      mbar_arrive_expect_tx(x_full, xbytes);
      bulk_g2s(xs, x, xbytes, x_full);
      for (int kb = 0; kb < nkb; ++kb) {
        const int st = kb % S;
        if (kb >= S && !mbar_wait_bounded(&empty[st], (uint32_t)(((kb / S) - 1) & 1)))
          set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        mbar_arrive_expect_tx(&full[st], (uint32_t)GG::kTile);   // whole box, out of range zero
        tma_load_2d(smem + st * GG::kTile, &wmap, kb * kGemvKB, n0, &full[st]);
      }
    }
    return;
  }
  // ------------------------------------------------------------ consumers
  if (!mbar_wait_bounded(x_full, 0) && lane == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
  float acc[F][kGemvRowsMax];
#pragma unroll
  for (int f = 0; f < F; ++f)
#pragma unroll
    for (int r = 0; r < kGemvRowsMax; ++r) acc[f][r] = 0.f;
  for (int kb = 0; kb < nkb; ++kb) {
    const int st = kb % S;
    if (!mbar_wait_bounded(&full[st], (uint32_t)((kb / S) & 1)) && lane == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
    const int c = kb * (kGemvKB / 8) + lane;       // 16-byte chunk of K of this lane
    if (c < nK) {
      const unsigned char *tile = smem + st * GG::kTile;
      float wf[F][8];
#pragma unroll
      for (int f = 0; f < F; ++f)
        Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4 *>(tile + (warp * F + f) * (kGemvKB * 2) + lane * 16),
                                     wf[f]);
#pragma unroll
      for (int r = 0; r < kGemvRowsMax; ++r) {
        if (r >= p.rows) break;
        float xf[8];
        Vec16<__nv_bfloat16>::unpack(xs[r * nK + c], xf);
#pragma unroll
        for (int f = 0; f < F; ++f) {
          float a = acc[f][r];
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(wf[f][e], xf[e], a);
          acc[f][r] = a;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);        // this warp is done with the stage
  }
#pragma unroll
  for (int f = 0; f < F; ++f)
#pragma unroll
    for (int r = 0; r < kGemvRowsMax; ++r) {
      if (r >= p.rows) break;
      const float v = warp_sum(acc[f][r]);
      const int n = n0 + warp * F + f;
      if (lane == 0 && n < p.N) proj_store(p, r, n, v);
    }
}

template <int CPC>
static cudaError_t proj_gemv_t(const ProjParams &p, const void *x, const void *W, cudaStream_t st) {
  const int smem = gemv_smem_bytes<CPC>(p.rows, p.K);
  cudaError_t e = prepare_kernel(proj_gemv_kernel<CPC>, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap wmap;
  if (!make_tmap_2d(&wmap, W, 2, (unsigned long long)p.K, (unsigned long long)p.N, (unsigned long long)p.K * 2,
                    kGemvKB, CPC, 0))
    return cudaErrorInvalidValue;
  proj_gemv_kernel<CPC><<<(p.N + CPC - 1) / CPC, (kGemvWarps + 1) * 32, smem, st>>>(
      p, wmap, reinterpret_cast<const __nv_bfloat16 *>(x));
  return cudaGetLastError();
}

// ============================================================ few rows on the tensor cores
// Up to 32 rows with a wide K: the weights are the M = 128 operand and the
// rows of X the N = 16 or 32 operand (Z^T = W X^T), so nearly every byte a
// stage brings in is a weight byte the step needs.  A cluster of CS CTAs owns 128 output
// columns; CTA r streams the weight rows' K range r through a deep TMA ring.
// CS (up to 4) is chosen so that the clusters fill the SMs in one wave.  TMEM lane = output column, TMEM
// column = row of X.  Ranks 1.. store their partial sums into rank 0's shared
// memory (distributed shared memory); after one cluster barrier rank 0 adds
// them and writes each column for every row (32 lanes = 32 consecutive
// columns: coalesced per row).
constexpr int kSwapRowsMax = 32;   // rows handled by this path at most
constexpr int kSwapStages = 8;
constexpr int kSwapABytes = kProjRows * kProjKB * 2;      // 128 weight rows x 64 K
// per stage: the weight tile and SR rows of X (SR = MMA N: 16 or 32, rows padded)
__host__ __device__ constexpr int swap_stage_bytes(int SR) { return kSwapABytes + SR * kProjKB * 2; }
// shared memory: ring, barriers, and the partials of ranks 1..CS-1 ([CS-1][128][SR] fp32)
__host__ __device__ constexpr int swap_smem(int CS, int SR) {
  return 1024 + kSwapStages * swap_stage_bytes(SR) + 256 + (CS - 1) * kProjRows * SR * 4;
}

template <int CS, int SR>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_swap_tc_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ CUtensorMap wmap,
                        const __grid_constant__ CUtensorMap xmap) {
  constexpr int S = kSwapStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * swap_stage_bytes(SR));
  uint64_t *full = bars, *empty = bars + S, *acc_full = bars + 2 * S;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 1);
  float *red = reinterpret_cast<float *>(smem + S * swap_stage_bytes(SR) + 256);   // [CS-1][128][SR]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int col0 = (blockIdx.x / CS) * kProjRows;
  const int nk_all = (p.K + kProjKB - 1) / kProjKB;
  const int kb0 = rank * nk_all / CS, kb1 = (rank + 1) * nk_all / CS;
  const int nk = kb1 - kb0;                        // K blocks of this rank (may be 0)

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, SR < 32 ? 32 : SR);   // at least 32 columns
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % S;
        if (kb >= S && !mbar_wait_bounded(&empty[st], (uint32_t)(((kb / S) - 1) & 1)))
          set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        unsigned char *a = smem + st * swap_stage_bytes(SR);
        mbar_arrive_expect_tx(&full[st], (uint32_t)swap_stage_bytes(SR));   // whole boxes, out of range zero
        tma_load_2d(a, &wmap, (kb0 + kb) * kProjKB, col0, &full[st]);
        tma_load_2d(a + kSwapABytes, &xmap, (kb0 + kb) * kProjKB, 0, &full[st]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc_idesc_bf16(kProjRows, SR);
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % S;
        if (!mbar_wait_bounded(&full[st], (uint32_t)((kb / S) & 1))) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        tc_fence_after();
        const uint32_t a = smem_u32(smem + st * swap_stage_bytes(SR));
        const uint64_t adesc = tc_sdesc_kmajor(a, 128), bdesc = tc_sdesc_kmajor(a + kSwapABytes, 128);
#pragma unroll
        for (int ks = 0; ks < kProjKB / 16; ++ks)
          tc_mma_bf16(tmem, adesc + 2 * ks, bdesc + 2 * ks, idesc, (kb | ks) != 0);
        tc_commit(&empty[st]);
      }
      if (nk > 0) tc_commit(acc_full);
      else mbar_arrive(acc_full);                   // no K range for this rank: nothing was issued
    }
  }
  float part[SR];
#pragma unroll
  for (int r = 0; r < SR; ++r) part[r] = 0.f;
  const int quad = warp - 4, cl = quad * 32 + lane;   // epilogue: local output column of this thread
  if (warp >= 4) {
    if (!mbar_wait_bounded(acc_full, 0) && lane == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
    __syncwarp();
    tc_fence_after();
    if (nk > 0) {
#pragma unroll
      for (int c = 0; c < SR; c += 16) {
        uint32_t v[16];
        tc_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c, v);
        tc_wait_ld();
#pragma unroll
        for (int r = 0; r < 16; ++r) part[c + r] = __uint_as_float(v[r]);
      }
    }
    if (rank > 0) {                                 // partial sums into rank 0
      float4 *dst = reinterpret_cast<float4 *>(cluster.map_shared_rank(red, 0) +
                                               ((size_t)(rank - 1) * kProjRows + cl) * SR);
#pragma unroll
      for (int q4 = 0; q4 < SR / 4; ++q4)
        dst[q4] = make_float4(part[4 * q4], part[4 * q4 + 1], part[4 * q4 + 2], part[4 * q4 + 3]);
    }
  }
  cluster.sync();                                   // every partial has arrived in rank 0
  if (warp >= 4 && rank == 0) {
    const int n = col0 + cl;
    for (int j = 1; j < CS; ++j) {
      const float4 *src = reinterpret_cast<const float4 *>(red + ((size_t)(j - 1) * kProjRows + cl) * SR);
#pragma unroll
      for (int q4 = 0; q4 < SR / 4; ++q4) {
        const float4 a = src[q4];
        part[4 * q4] += a.x;
        part[4 * q4 + 1] += a.y;
        part[4 * q4 + 2] += a.z;
        part[4 * q4 + 3] += a.w;
      }
    }
    if (n < p.N)
#pragma unroll
      for (int r = 0; r < SR; ++r)
        if (r < p.rows) proj_store(p, r, n, part[r]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tc_dealloc(tmem, SR < 32 ? 32 : SR);
  }
}

template <int CS, int SR>
static cudaError_t proj_swap_t(const ProjParams &p, const void *x, const void *W, cudaStream_t st) {
  cudaError_t e = prepare_kernel(proj_swap_tc_kernel<CS, SR>, swap_smem(CS, SR));
  if (e != cudaSuccess) return e;
  CUtensorMap wmap, xmap;
  if (!make_tmap_2d(&wmap, W, 2, (unsigned long long)p.K, (unsigned long long)p.N, (unsigned long long)p.K * 2,
                    kProjKB, kProjRows, 128) ||
      !make_tmap_2d(&xmap, x, 2, (unsigned long long)p.K, (unsigned long long)p.rows, (unsigned long long)p.K * 2,
                    kProjKB, SR, 128))
    return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(((p.N + kProjRows - 1) / kProjRows) * CS);
  cfg.blockDim = dim3(kProjThreads);
  cfg.dynamicSmemBytes = swap_smem(CS, SR);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, proj_swap_tc_kernel<CS, SR>, p, wmap, xmap);
}

cudaError_t launch_proj(const ProjParams &p, const void *x, const void *W, cudaStream_t st) {
  if (p.rows <= 0 || p.N <= 0) return cudaSuccess;
  if (p.rows <= kGemvRowsMax && gemv_smem_bytes<32>(p.rows, p.K) <= 227 * 1024) {
    // enough CTAs to put every SM on the weight stream: 16 columns per CTA
    // while that gives at most ~2 waves, else 32 (X is re-read by fewer warps)
    if ((p.N + 15) / 16 <= 2 * 148) return proj_gemv_t<16>(p, x, W, st);
    return proj_gemv_t<32>(p, x, W, st);
  }
  if (p.rows <= kSwapRowsMax) {
    // K split over a cluster of CS CTAs: as many as still fit the SMs in one wave
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess) {
      cudaGetLastError();
      sms = 148;
    }
    const int tiles = (p.N + kProjRows - 1) / kProjRows;
    // (larger clusters measured slower: they fit the GPCs less evenly)
    const int cs = std::max(1, std::min(4, sms / tiles));
    if (p.rows <= 16) {
      switch (cs) {
        case 1: return proj_swap_t<1, 16>(p, x, W, st);
        case 2: return proj_swap_t<2, 16>(p, x, W, st);
        case 3: return proj_swap_t<3, 16>(p, x, W, st);
        default: return proj_swap_t<4, 16>(p, x, W, st);
      }
    }
    switch (cs) {
      case 1: return proj_swap_t<1, 32>(p, x, W, st);
      case 2: return proj_swap_t<2, 32>(p, x, W, st);
      case 3: return proj_swap_t<3, 32>(p, x, W, st);
      default: return proj_swap_t<4, 32>(p, x, W, st);
    }
  }
  // more rows: tensor cores; narrow column tiles while the rows fit one tile
  return p.rows <= kProjRows ? proj_t<32>(p, x, W, st) : proj_t<256>(p, x, W, st);
}

}  // namespace lisa
