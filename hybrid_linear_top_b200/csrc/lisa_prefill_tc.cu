// Lightning Indexer scores for a block of query rows on the sm_100a tensor
// cores (tcgen05), bf16 inputs, fp32 accumulation in tensor memory.
//
// Method: arXiv 2607.19358 (LISA), abstract and the gptget.net digest's method
// section (indexer = query / key projections and a ReLU dot product); the
// weighted sum over the R indexer heads of a KV head is as stated in lisa.h.
//
// For one (sequence b, KV head g), a CTA owns 128 query rows and a range of
// key tiles of N keys.  Per key tile the R head products Q_r K^T (128 x N,
// K = dI) are accumulated in tensor memory; the epilogue turns them into
// sum_r w_r * max(0, .), then into order keys, and stores the causal part
// (key position <= query position).  Warp roles: warps 0-3 and 8-11
// epilogue (one thread per query row = one TMEM lane; warps q and q + 8 take
// the two halves of a tile's keys), warp 4 TMA producer, warp 5 MMA issuer
// and TMEM owner.  Two accumulator buffers let the MMAs of one tile overlap
// the epilogue of the previous one.
#include "lisa_internal.h"
#include "lisa_tc.cuh"

namespace lisa {

constexpr int kTcThreads = 384;   // warps 0-3 and 8-11 epilogue, 4 TMA, 5 MMA, 6-7 idle
constexpr int kTcStages = 4;
constexpr int kTcKeyTilesPerCta = 8;
constexpr int kTcRows = 128;

// Keys per tile: 2 buffers x R accumulators x N columns fill the 512 TMEM columns.
__host__ __device__ inline int tc_tile_n(int R) { return R <= 1 ? 256 : R <= 2 ? 128 : R <= 4 ? 64 : 32; }

// Epilogue staging: per epilogue warp 32 rows x 32 keys, rows padded to 36
// words (16-byte aligned, conflict-free for the row-wise writes and the
// transposed reads).
constexpr int kStageRowWords = 36;
constexpr int kStageWarpWords = 32 * kStageRowWords;

__host__ __device__ inline int tc_smem_bytes(int R, int DI) {
  const int RB = DI * 2;
  return 1024 + R * kTcRows * RB + kTcStages * tc_tile_n(R) * RB + 256 + 8 * kStageWarpWords * 4;
}

template <int DI>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_score_tc_kernel(const __grid_constant__ RowsParams p, const __grid_constant__ CUtensorMap qmap,
                            const __grid_constant__ CUtensorMap kmap, int tau0, int rows) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  constexpr int RB = DI * 2;                       // bf16 row bytes (128 or 64)
  constexpr int KS = DI / 16;                      // MMA k-steps
  const int R = p.R;
  const int N = tc_tile_n(R);
  const int rb = blockIdx.x, kr = blockIdx.y, bg = blockIdx.z;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int p0 = p.pos[b];
  if (p0 < 0 || p0 + p.T > p.L_max || (p.require_pos0 && p0 != 0)) return;
  const int r_lo = rb * kTcRows;
  if (r_lo >= rows) return;
  const int r_hi = min(r_lo + kTcRows, rows);
  const int last_pos = p0 + tau0 + r_hi - 1;       // largest candidate position of this row block
  const int kt0 = kr * kTcKeyTilesPerCta;
  const int kt_end = min(kt0 + kTcKeyTilesPerCta, last_pos / N + 1);
  const int ntiles = kt_end - kt0;
  if (ntiles <= 0) return;                         // uniform for the CTA: nothing allocated yet

  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  unsigned char *q_tiles = smem;                                   // [R][128][DI], swizzled
  unsigned char *k_ring = smem + R * kTcRows * RB;                 // [stages][N][DI], swizzled
  uint64_t *bars = reinterpret_cast<uint64_t *>(k_ring + kTcStages * N * RB);
  uint64_t *q_full = bars;
  uint64_t *k_full = bars + 1;
  uint64_t *k_empty = bars + 1 + kTcStages;
  uint64_t *acc_full = bars + 1 + 2 * kTcStages;
  uint64_t *acc_empty = bars + 3 + 2 * kTcStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 5 + 2 * kTcStages);
  unsigned char *bars_end = reinterpret_cast<unsigned char *>(bars) + 256;   // staging of the epilogue warps
  constexpr uint32_t kTmemCols = 512;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 8 * 32);
    }
    fence_mbar_init();
  }
  if (warp == 5) {
    tc_alloc(tmem_slot, kTmemCols);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, (uint32_t)(R * kTcRows * RB));
      for (int r = 0; r < R; ++r)
        tma_load_3d(q_tiles + r * kTcRows * RB, &qmap, 0, g * R + r, b * p.T + tau0 + r_lo, q_full);
      for (int it = 0; it < ntiles; ++it) {
        const int st = it % kTcStages;
        if (it >= kTcStages && !mbar_wait_bounded(&k_empty[st], (uint32_t)(((it / kTcStages) - 1) & 1)))
          set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        mbar_arrive_expect_tx(&k_full[st], (uint32_t)(N * RB));
        tma_load_2d(k_ring + st * N * RB, &kmap, 0, bg * p.L_max + (kt0 + it) * N, &k_full[st]);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      if (!mbar_wait_bounded(q_full, 0)) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
      const uint32_t idesc = tc_idesc_bf16(kTcRows, N);
      for (int it = 0; it < ntiles; ++it) {
        const int st = it % kTcStages, buf = it & 1;
        if (!mbar_wait_bounded(&k_full[st], (uint32_t)((it / kTcStages) & 1))) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        if (it >= 2 && !mbar_wait_bounded(&acc_empty[buf], (uint32_t)(((it >> 1) - 1) & 1)))
          set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        tc_fence_after();
        const uint64_t bdesc0 = tc_sdesc_kmajor(smem_u32(k_ring + st * N * RB), RB);
        for (int r = 0; r < R; ++r) {
          const uint64_t adesc0 = tc_sdesc_kmajor(smem_u32(q_tiles + r * kTcRows * RB), RB);
#pragma unroll
          for (int ks = 0; ks < KS; ++ks)   // +32 bytes along K inside the swizzle atom
            tc_mma_bf16(tmem + (uint32_t)((buf * R + r) * N), adesc0 + 2 * ks, bdesc0 + 2 * ks, idesc, ks > 0);
        }
        tc_commit(&k_empty[st]);     // the key tile may be overwritten once these MMAs are done
        tc_commit(&acc_full[buf]);   // the accumulators of this tile are ready
      }
    }
  } else if (warp < 4 || warp >= 8) {
    // ------------------------------------------------------------ epilogue: thread = query row
    // Warps q and q + 8 share TMEM lanes 32q..32q+31 (one query row per
    // thread) and split the key columns of a tile.  Scores of 32 keys per row
    // are staged in shared memory, then written row-wise: 8 lanes cover 128
    // contiguous bytes of one row, so a warp store touches 4 rows, not 32.
    const int qd = warp & 3, hsel = warp >= 8 ? 1 : 0;
    const int cbeg = N >= 64 ? hsel * (N / 2) : 0;
    const int cend = N >= 64 ? cbeg + N / 2 : (hsel ? 0 : N);
    const int row = qd * 32 + lane;
    const int rr = r_lo + row;
    const bool row_ok = rr < r_hi;
    float wr[kMaxR];
#pragma unroll
    for (int r = 0; r < kMaxR; ++r)
      wr[r] = (row_ok && r < R) ? p.w[((size_t)b * p.T + tau0 + rr) * p.HI + g * R + r] : 0.f;
    uint32_t *stg = reinterpret_cast<uint32_t *>(bars_end) + (qd + 4 * hsel) * kStageWarpWords;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const int wrow = lane >> 3, wcol = (lane & 7) * 4;          // write-out: row within 4, key offset
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      if (!mbar_wait_bounded(&acc_full[buf], (uint32_t)((it >> 1) & 1)) && lane == 0)
        set_err(p.err_word, LISA_DEVERR_TIMEOUT);
      __syncwarp();
      tc_fence_after();
      const int s0 = (kt0 + it) * N;
      for (int c = cbeg; c < cend; c += 32) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float acc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = 0.f;
#pragma unroll
          for (int r = 0; r < kMaxR; ++r) {
            if (r >= R) break;
            uint32_t v[16];
            tc_ld16(tmem + lane_base + (uint32_t)((buf * R + r) * N + c + 16 * half), v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = fmaf(wr[r], fmaxf(__uint_as_float(v[j]), 0.f), acc[j]);
          }
          uint4 *sd = reinterpret_cast<uint4 *>(stg + lane * kStageRowWords + 16 * half);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            sd[q] = make_uint4(score_key(acc[4 * q]), score_key(acc[4 * q + 1]), score_key(acc[4 * q + 2]),
                               score_key(acc[4 * q + 3]));
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rloc = 4 * k + wrow;
          const int rr2 = r_lo + qd * 32 + rloc;
          const int sc = s0 + c + wcol;
          const int tpos2 = p0 + tau0 + rr2;
          if (rr2 < r_hi && sc <= tpos2) {
            const uint4 v = *reinterpret_cast<const uint4 *>(stg + rloc * kStageRowWords + wcol);
            uint32_t *gd = p.keys + ((size_t)bg * p.row_chunk + rr2) * p.L_keys + sc;
            if (sc + 3 <= tpos2) {
              *reinterpret_cast<uint4 *>(gd) = v;
            } else {
              gd[0] = v.x;
              if (sc + 1 <= tpos2) gd[1] = v.y;
              if (sc + 2 <= tpos2) gd[2] = v.z;
            }
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tc_dealloc(tmem, kTmemCols);
  }
}

template <int DI>
static cudaError_t score_tc_t(const RowsParams &p, cudaStream_t st, int tau0, int rows, int key_hi) {
  const int N = tc_tile_n(p.R);
  const int smem = tc_smem_bytes(p.R, DI) > 120 * 1024 ? tc_smem_bytes(p.R, DI) : 120 * 1024;   // one CTA per SM
  cudaError_t e = prepare_kernel(prefill_score_tc_kernel<DI>, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap qmap, kmap;
  // qidx [B, T, HI, DI] viewed as {DI, HI, B*T}; box = 128 rows of one head
  const unsigned long long qdims[3] = {(unsigned long long)DI, (unsigned long long)p.HI, (unsigned long long)p.B * p.T};
  const unsigned long long qstr[2] = {(unsigned long long)DI * 2, (unsigned long long)p.HI * DI * 2};
  const unsigned qbox[3] = {(unsigned)DI, 1u, (unsigned)kTcRows};
  if (!make_tmap(&qmap, p.qidx, 2, 3, qdims, qstr, qbox, DI * 2)) return cudaErrorInvalidValue;
  const unsigned long long kdims[2] = {(unsigned long long)DI, (unsigned long long)p.B * p.Hkv * p.L_max};
  const unsigned long long kstr[1] = {(unsigned long long)DI * 2};
  const unsigned kbox[2] = {(unsigned)DI, (unsigned)N};
  if (!make_tmap(&kmap, p.kidx_cache, 2, 2, kdims, kstr, kbox, DI * 2)) return cudaErrorInvalidValue;
  const int key_ranges = (key_hi + kTcKeyTilesPerCta * N - 1) / (kTcKeyTilesPerCta * N);
  dim3 grid((rows + kTcRows - 1) / kTcRows, key_ranges, p.B * p.Hkv);
  prefill_score_tc_kernel<DI><<<grid, kTcThreads, smem, st>>>(p, qmap, kmap, tau0, rows);
  return cudaGetLastError();
}

cudaError_t launch_rows_score_tc(const RowsParams &p, cudaStream_t st, int tau0, int rows, int key_hi) {
  if (p.DI == 64) return score_tc_t<64>(p, st, tau0, rows, key_hi);
  if (p.DI == 32) return score_tc_t<32>(p, st, tau0, rows, key_hi);
  return cudaErrorInvalidValue;
}

}  // namespace lisa
