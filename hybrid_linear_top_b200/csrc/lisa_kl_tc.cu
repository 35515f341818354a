// Stage-2 indexer objective of LISA (forward) on the sm_100a tensor cores
// (tcgen05): per-head KL divergence between the frozen model's attention and
// the indexer's distribution over the causal prefix, bf16 inputs, fp32
// accumulation in tensor memory.
//
// Method: arXiv 2607.19358, English abstract on arxivdaily.com (Stage 2 trains
// the Indexer with a per-head KL divergence that aligns its selection with the
// teacher's attention pattern).  Definition (lisa.h): for token t and query
// head h of KV head g,
//   p(s) = softmax_{s<=t}(q_h . k_s / sqrt(d)),  r(s) = softmax_{s<=t}(I_g(t, s)),
//   KL   = E_p[a - c] - logsumexp(a) + logsumexp(c)     (a, c: the two logits).
//
// A CTA owns 128 tokens of one (sequence, KV head) and up to kKlHeads query
// heads of its group.  It streams the causal prefix in tiles of 32 keys (K
// and indexer-key rows by TMA, 128-byte swizzle) and per tile issues, into one
// of two TMEM buffers, the head products Q_h K^T (M = 128 tokens, N = 32 keys,
// K = 128) and the indexer-head products Q^I_r K^I^T (K = dI).  The indexer
// logits of a tile are formed once for all heads of the CTA.  Warp roles:
// warp 0 lane 0 TMA producer, warp 1 lane 0 MMA issuer and TMEM owner, warps
// 4-11 epilogue: warps q + 4 and q + 8 share TMEM lane quadrant q (thread =
// token) and take the first and the second 16 keys of every tile.  Each keeps
// the online statistics of its token over its keys (running maximum, sum of
// exponentials, and the sum of exp(a - max) (a - c)), reading one buffer
// while the MMAs of the next tile fill the other; the two halves are merged
// at the end.
#include <type_traits>

#include "lisa_internal.h"
#include "lisa_tc.cuh"

namespace lisa {

constexpr int kKlRows = 128;       // tokens per CTA (MMA M = TMEM lanes)
constexpr int kKlKeys = 32;        // keys per tile (MMA N)
constexpr int kKlHeads = 3;        // query heads per CTA
constexpr int kKlMaxR = 4;         // indexer heads per KV head this kernel handles
constexpr int kKlStages = 4;
constexpr int kKlThreads = 384;    // warps 0-3: TMA, MMA, two idle; warps 4-11: epilogue
constexpr int kKlEpiThreads = 256;
constexpr int kKlBufCols = 256;    // per buffer: heads at j * 32, indexer heads at 96 + r * 32
constexpr float kLn2 = 0.6931471805599453f;     // ln(2)

template <int DI>
struct KlTcGeom {
  static constexpr int RBI = DI * 2;                        // indexer row bytes (128 or 64)
  static constexpr int kQHalf = kKlRows * 128;              // 64 dims of 128 tokens: 16 KB
  static constexpr int kQI = kKlRows * RBI;                 // one indexer head's queries
  static constexpr int kKHalf = kKlKeys * 128;              // 64 dims of 32 keys: 4 KB
  static constexpr int kStage = 2 * kKHalf + kKlKeys * RBI; // K tile + indexer-key tile
  // byte offsets (from a 1024-aligned base) for R indexer heads
  static __host__ __device__ int q_off() { return 0; }
  static __host__ __device__ int qi_off() { return kKlHeads * 2 * kQHalf; }
  static __host__ __device__ int ring_off(int R) { return qi_off() + R * kQI; }
  static __host__ __device__ int bar_off(int R) { return ring_off(R) + kKlStages * kStage; }
  static __host__ __device__ int smem(int R) { return 1024 + bar_off(R) + 256; }
};

// exp2_approx (lisa_common.cuh): the epilogue keeps its logits in log2 units
// so that no multiply precedes the exponential.

__device__ __forceinline__ float tree_max16(const float *x) {
  float s8[8], s4[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) s8[i] = fmaxf(x[i], x[i + 8]);
#pragma unroll
  for (int i = 0; i < 4; ++i) s4[i] = fmaxf(s8[i], s8[i + 4]);
  return fmaxf(fmaxf(s4[0], s4[2]), fmaxf(s4[1], s4[3]));
}

template <int DI>
__global__ void __launch_bounds__(kKlThreads, 1)
    indexer_kl_tc_kernel(const __grid_constant__ RowsParams p, const __grid_constant__ CUtensorMap qmap,
                         const __grid_constant__ CUtensorMap qimap, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap kimap, float *__restrict__ kl_out) {
  using KG = KlTcGeom<DI>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int R = p.R, G = p.G;
  const int nrb = (p.T + kKlRows - 1) / kKlRows;
  const int rb = nrb - 1 - (int)blockIdx.x;          // longest prefixes first
  const int bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int h0 = blockIdx.z * kKlHeads;               // first head of this CTA within the group
  const int hc = min(kKlHeads, G - h0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p0 = p.pos[b];
  if (p0 < 0 || p0 + p.T > p.L_max) return;           // uniform for the CTA: nothing allocated yet
  const int tau0 = rb * kKlRows;
  const int ntok = min(kKlRows, p.T - tau0);
  const int t_last = p0 + tau0 + ntok - 1;
  const int ntiles = t_last / kKlKeys + 1;

  unsigned char *qs = smem + KG::q_off();
  unsigned char *qis = smem + KG::qi_off();
  unsigned char *ring = smem + KG::ring_off(R);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + KG::bar_off(R));
  uint64_t *q_full = bars, *full = bars + 1, *empty = bars + 1 + kKlStages;
  uint64_t *acc_full = bars + 1 + 2 * kKlStages, *acc_empty = bars + 3 + 2 * kKlStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 5 + 2 * kKlStages);
  constexpr uint32_t kCols = 2 * kKlBufCols;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKlStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kKlEpiThreads);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, (uint32_t)(hc * 2 * KG::kQHalf + R * KG::kQI));
      for (int j = 0; j < hc; ++j)
        for (int half = 0; half < 2; ++half)
          tma_load_3d(qs + (j * 2 + half) * KG::kQHalf, &qmap, half * 64, g * G + h0 + j, b * p.T + tau0, q_full);
      for (int r = 0; r < R; ++r) tma_load_3d(qis + r * KG::kQI, &qimap, 0, g * R + r, b * p.T + tau0, q_full);
      for (int it = 0; it < ntiles; ++it) {
        const int st = it % kKlStages;
        if (it >= kKlStages && !mbar_wait_bounded(&empty[st], (uint32_t)(((it / kKlStages) - 1) & 1)))
          set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        unsigned char *s = ring + st * KG::kStage;
        const int row = bg * p.L_max + it * kKlKeys;
        mbar_arrive_expect_tx(&full[st], (uint32_t)KG::kStage);   // whole boxes land, out of range zero
        tma_load_2d(s, &kmap, 0, row, &full[st]);
        tma_load_2d(s + KG::kKHalf, &kmap, 64, row, &full[st]);
        tma_load_2d(s + 2 * KG::kKHalf, &kimap, 0, row, &full[st]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      if (!mbar_wait_bounded(q_full, 0)) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
      const uint32_t idesc = tc_idesc_bf16(kKlRows, kKlKeys);
      for (int it = 0; it < ntiles; ++it) {
        const int st = it % kKlStages, buf = it & 1;
        if (it >= 2 && !mbar_wait_bounded(&acc_empty[buf], (uint32_t)(((it >> 1) - 1) & 1)))
          set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        if (!mbar_wait_bounded(&full[st], (uint32_t)((it / kKlStages) & 1))) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
        tc_fence_after();
        const uint32_t s = smem_u32(ring + st * KG::kStage);
        const uint32_t dbuf = tmem + (uint32_t)(buf * kKlBufCols);
        for (int j = 0; j < hc; ++j)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint64_t ad = tc_sdesc_kmajor(smem_u32(qs + (j * 2 + half) * KG::kQHalf), 128);
            const uint64_t bd = tc_sdesc_kmajor(s + half * KG::kKHalf, 128);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)   // +32 bytes along K inside the swizzle atom
              tc_mma_bf16(dbuf + (uint32_t)(j * kKlKeys), ad + 2 * ks, bd + 2 * ks, idesc, (half | ks) != 0);
          }
        const uint64_t bdi = tc_sdesc_kmajor(s + 2 * KG::kKHalf, KG::RBI);
        for (int r = 0; r < R; ++r) {
          const uint64_t adi = tc_sdesc_kmajor(smem_u32(qis + r * KG::kQI), KG::RBI);
#pragma unroll
          for (int ks = 0; ks < DI / 16; ++ks)
            tc_mma_bf16(dbuf + (uint32_t)(kKlHeads * kKlKeys + r * kKlKeys), adi + 2 * ks, bdi + 2 * ks, idesc, ks > 0);
        }
        tc_commit(&empty[st]);       // the key tiles may be refilled once these MMAs are done
        tc_commit(&acc_full[buf]);   // the logits of this tile are ready
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue: thread = (token, half of the keys)
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const int row = quad * 32 + lane;
    const bool ok = row < ntok;
    const int t = p0 + tau0 + row;                    // this token's position
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    constexpr int HK = kKlKeys / 2;                   // keys of a tile per thread
    float wr[kKlMaxR];
#pragma unroll
    for (int r = 0; r < kKlMaxR; ++r)
      wr[r] = (ok && r < R) ? p.w[((size_t)b * p.T + tau0 + row) * p.HI + g * R + r] * kLog2e : 0.f;
    // Logits in log2 units: c2 = c log2(e) (folded into the weights), a2 =
    // a log2(e) (folded into the scale); every exponential is then 2^(x - m).
    const float scale2 = p.scale * kLog2e;
    float ma[kKlHeads], za[kKlHeads], ua[kKlHeads];
#pragma unroll
    for (int j = 0; j < kKlHeads; ++j) {
      ma[j] = -INFINITY;
      za[j] = 0.f;
      ua[j] = 0.f;
    }
    float mc = -INFINITY, zc = 0.f;
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      if (!mbar_wait_bounded(&acc_full[buf], (uint32_t)((it >> 1) & 1)) && lane == 0)
        set_err(p.err_word, LISA_DEVERR_TIMEOUT);
      __syncwarp();
      tc_fence_after();
      const uint32_t dbuf = tmem + lane_base + (uint32_t)(buf * kKlBufCols + half * HK);
      const int s0 = it * kKlKeys + half * HK;
      const int nvalid = ok ? max(0, min(HK, t - s0 + 1)) : 0;   // keys s0 .. t of this half tile
      // the indexer heads' TMEM loads in flight at once, then the query heads'
      uint32_t vi[kKlMaxR][HK];
#pragma unroll
      for (int r = 0; r < kKlMaxR; ++r)
        if (r < R) tc_ld16(dbuf + (uint32_t)(kKlHeads * kKlKeys + r * kKlKeys), vi[r]);
      tc_wait_ld();
      // indexer logits c = sum_r w_r relu(Q^I_r . K^I)
      float c[HK];
#pragma unroll
      for (int k = 0; k < HK; ++k) c[k] = 0.f;
#pragma unroll
      for (int r = 0; r < kKlMaxR; ++r) {
        if (r >= R) break;
#pragma unroll
        for (int k = 0; k < HK; ++k) c[k] = fmaf(wr[r], fmaxf(__uint_as_float(vi[r][k]), 0.f), c[k]);
      }
      uint32_t va[kKlHeads][HK];
#pragma unroll
      for (int j = 0; j < kKlHeads; ++j)
        if (j < hc) tc_ld16(dbuf + (uint32_t)(j * kKlKeys), va[j]);
      // Online statistics of this tile's keys.  All 16 keys valid for every
      // token of the warp (all tiles but those holding the tokens' own
      // positions): no masking.
      auto stats = [&](auto all_valid) {
        constexpr bool FULL = decltype(all_valid)::value;
        if (!FULL) {
#pragma unroll
          for (int k = 0; k < HK; ++k)
            if (k >= nvalid) c[k] = -INFINITY;
        }
        const float nmc = fmaxf(mc, tree_max16(c));
        if (nmc != -INFINITY) {                       // some key of the prefix seen (per lane: no sync inside)
          float z4[4] = {0.f, 0.f, 0.f, 0.f};         // four partial sums: short chains
#pragma unroll
          for (int k = 0; k < HK; ++k) z4[k & 3] += exp2_approx(c[k] - nmc);   // 0 for masked keys
          zc = (mc == -INFINITY ? 0.f : zc * exp2_approx(mc - nmc)) + ((z4[0] + z4[1]) + (z4[2] + z4[3]));
          mc = nmc;
        }
        tc_wait_ld();                                 // the query heads' logits
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);                 // registers hold the tile: the buffer may be refilled
        // teacher logits a = q_h . k / sqrt(d) of each head
#pragma unroll
        for (int j = 0; j < kKlHeads; ++j) {
          if (j >= hc) break;
          float a[HK];
#pragma unroll
          for (int k = 0; k < HK; ++k)
            a[k] = (FULL || k < nvalid) ? __uint_as_float(va[j][k]) * scale2 : -INFINITY;
          const float nm = fmaxf(ma[j], tree_max16(a));
          if (nm == -INFINITY) continue;              // no key of the prefix yet (this lane)
          const float f = ma[j] == -INFINITY ? 0.f : exp2_approx(ma[j] - nm);
          float z4[4] = {0.f, 0.f, 0.f, 0.f}, u4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k = 0; k < HK; ++k) {
            const float ek = exp2_approx(a[k] - nm);   // 0 for masked keys
            z4[k & 3] += ek;
            u4[k & 3] = fmaf(ek, (FULL || k < nvalid) ? a[k] - c[k] : 0.f, u4[k & 3]);
          }
          za[j] = za[j] * f + ((z4[0] + z4[1]) + (z4[2] + z4[3]));
          ua[j] = ua[j] * f + ((u4[0] + u4[1]) + (u4[2] + u4[3]));
          ma[j] = nm;
        }
      };
      // the branch must be uniform in the warp: stats() waits on the warp's
      // TMEM loads (a .sync.aligned instruction).  Keys past a token's
      // position (nvalid < HK, possibly 0) take the masked form.
      if (__all_sync(0xffffffffu, nvalid == HK)) stats(std::true_type{});
      else stats(std::false_type{});
    }
    // merge the two halves of each token (log-sum-exp merges) through shared
    // memory: the key ring is idle once the last tile's MMAs have completed
    float *mrg = reinterpret_cast<float *>(ring);     // [128 tokens][2 + 3 * kKlHeads]
    constexpr int MS = 2 + 3 * kKlHeads;
    if (half == 1) {
      mrg[row * MS + 0] = mc;
      mrg[row * MS + 1] = zc;
#pragma unroll
      for (int j = 0; j < kKlHeads; ++j) {
        mrg[row * MS + 2 + 3 * j] = ma[j];
        mrg[row * MS + 3 + 3 * j] = za[j];
        mrg[row * MS + 4 + 3 * j] = ua[j];
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kKlEpiThreads) : "memory");   // epilogue warps only
    if (half == 0 && ok) {
      auto merge = [](float &m, float &z, float &u, float m2, float z2, float u2) {
        const float nm = fmaxf(m, m2);
        const float f1 = m == -INFINITY ? 0.f : exp2_approx(m - nm), f2 = m2 == -INFINITY ? 0.f : exp2_approx(m2 - nm);
        z = z * f1 + z2 * f2;
        u = u * f1 + u2 * f2;
        m = nm;
      };
      float du = 0.f;
      merge(mc, zc, du, mrg[row * MS + 0], mrg[row * MS + 1], 0.f);
      const float lse_c = mc + log2f(zc);           // log2 units; KL = ln 2 x (...) below
#pragma unroll
      for (int j = 0; j < kKlHeads; ++j)
        if (j < hc) {
          merge(ma[j], za[j], ua[j], mrg[row * MS + 2 + 3 * j], mrg[row * MS + 3 + 3 * j], mrg[row * MS + 4 + 3 * j]);
          kl_out[((size_t)b * p.T + tau0 + row) * p.Hq + g * G + h0 + j] =
              kLn2 * (ua[j] / za[j] - (ma[j] + log2f(za[j])) + lse_c);
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tc_dealloc(tmem, kCols);
  }
}

template <int DI>
static cudaError_t kl_tc_t(const RowsParams &p, float *kl_out, cudaStream_t st) {
  using KG = KlTcGeom<DI>;
  const int smem = KG::smem(p.R);
  cudaError_t e = prepare_kernel(indexer_kl_tc_kernel<DI>, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap qmap, qimap, kmap, kimap;
  // q [B, T, Hq, 128] as {128, Hq, B*T}: box = 64 dims x 1 head x 128 tokens
  const unsigned long long qd[3] = {128ull, (unsigned long long)p.Hq, (unsigned long long)p.B * p.T};
  const unsigned long long qst[2] = {256ull, (unsigned long long)p.Hq * 256ull};
  const unsigned qb[3] = {64u, 1u, (unsigned)kKlRows};
  // qidx [B, T, HI, DI] as {DI, HI, B*T}
  const unsigned long long qid[3] = {(unsigned long long)DI, (unsigned long long)p.HI, (unsigned long long)p.B * p.T};
  const unsigned long long qist[2] = {(unsigned long long)DI * 2, (unsigned long long)p.HI * DI * 2};
  const unsigned qib[3] = {(unsigned)DI, 1u, (unsigned)kKlRows};
  if (!make_tmap(&qmap, p.q, 2, 3, qd, qst, qb, 128) || !make_tmap(&qimap, p.qidx, 2, 3, qid, qist, qib, DI * 2) ||
      !make_tmap_2d(&kmap, p.k_cache, 2, 128ull, (unsigned long long)p.B * p.Hkv * p.L_max, 256ull, 64, kKlKeys, 128) ||
      !make_tmap_2d(&kimap, p.kidx_cache, 2, (unsigned long long)DI, (unsigned long long)p.B * p.Hkv * p.L_max,
                    (unsigned long long)DI * 2, DI, kKlKeys, DI * 2))
    return cudaErrorInvalidValue;
  dim3 grid((p.T + kKlRows - 1) / kKlRows, p.B * p.Hkv, (p.G + kKlHeads - 1) / kKlHeads);
  indexer_kl_tc_kernel<DI><<<grid, kKlThreads, smem, st>>>(p, qmap, qimap, kmap, kimap, kl_out);
  return cudaGetLastError();
}

// d = 128, at most 4 indexer heads per KV head: the tensor-core kernel; else
// false (the caller uses the warp-MMA kernel).
bool indexer_kl_tc_supported(const RowsParams &p) { return p.D == 128 && p.R <= kKlMaxR; }

cudaError_t launch_indexer_kl_tc(const RowsParams &p, float *kl_out, cudaStream_t st) {
  if (p.DI == 64) return kl_tc_t<64>(p, kl_out, st);
  if (p.DI == 32) return kl_tc_t<32>(p, kl_out, st);
  return cudaErrorInvalidValue;
}

}  // namespace lisa
