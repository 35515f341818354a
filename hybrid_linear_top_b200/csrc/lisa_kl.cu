// Stage-2 indexer objective of LISA (forward): per-head KL divergence between
// the frozen model's attention and the indexer's distribution over the causal
// prefix, on warp tensor-core MMAs (bf16, fp32 accumulation).
//
// Method: arXiv 2607.19358, English abstract on arxivdaily.com (Stage 2 trains
// the Indexer with a per-head KL divergence that aligns its selection with the
// teacher's attention pattern).  Definition (see lisa.h): for token t and query
// head h of KV head g,
//   p(s) = softmax_{s<=t}(q_h . k_s / sqrt(d)),  r(s) = softmax_{s<=t}(I_g(t, s)),
//   KL   = sum_s p(s) (log p(s) - log r(s))
//        = E_p[a - c] - logsumexp(a) + logsumexp(c)   (a, c: the two logits),
// accumulated online over the prefix in one pass per head.
//
// Grid (ceil(T / 64), B * Hkv), 4 warps; warp w owns 16 consecutive tokens.
// For each query head of the group the warp streams the prefix in 16-key
// tiles (K rows and indexer-key rows staged with cp.async, two stages):
//   S   = Q K^T           (tokens x keys; A = the 16 tokens' q, B = K rows)
//   D_r = Q^I_r K^I^T     (per indexer head; A = the tokens' indexer queries)
//   c   = sum_r w_r relu(D_r)
// and keeps per-lane online statistics (max, sum of exponentials, and the sum
// of exp(a - max) (a - c)) that are merged across the lanes of a row at the end.
#include "lisa_internal.h"
#include "lisa_common.cuh"

namespace lisa {

constexpr int kKlWarps = 4;

template <int D, int DI>
struct KlGeom {
  static constexpr int RS = 2 * D + 16;                 // K row stride in shared memory (bytes)
  static constexpr int RSI = 2 * DI + 16;               // indexer-key row stride
  static constexpr int STG = 16 * RS + 16 * RSI;        // one stage: 16 K rows + 16 indexer-key rows
  static __host__ __device__ int qi_stride(int R) { return 2 * R * DI + 16; }   // staged indexer queries
  static __host__ __device__ int warp_bytes(int R) { return 2 * STG + 16 * qi_stride(R); }
};

template <int D, int DI>
__global__ void __launch_bounds__(kKlWarps * 32) indexer_kl_kernel(RowsParams p, float *kl_out) {
  extern __shared__ __align__(16) unsigned char s_kl[];
  using KG = KlGeom<D, DI>;
  const int bg = blockIdx.y;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int p0 = p.pos[b];
  if (p0 < 0 || p0 + p.T > p.L_max) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G, R = p.R;
  const int g4 = lane >> 2, t2 = (lane & 3) * 2;
  const int tau0 = blockIdx.x * (16 * kKlWarps) + warp * 16;   // first token of this warp
  if (tau0 >= p.T) return;                                       // warps never synchronise with each other
  const int ntok = min(16, p.T - tau0);
  const int t_last = p0 + tau0 + ntok - 1;                       // largest position among the warp's tokens
  const int trow0 = p0 + tau0 + g4, trow1 = trow0 + 8;           // positions of this lane's two rows
  const bool ok0 = g4 < ntok, ok1 = g4 + 8 < ntok;

  unsigned char *wb = s_kl + (size_t)warp * KG::warp_bytes(R);
  const uint32_t wb_u32 = smem_u32(wb);
  unsigned char *qis = wb + 2 * KG::STG;                          // [16 tokens][R * DI] indexer queries
  const int qstr = KG::qi_stride(R);
  const __nv_bfloat16 *kc = reinterpret_cast<const __nv_bfloat16 *>(p.k_cache) + (size_t)bg * p.L_max * D;
  const __nv_bfloat16 *kic = reinterpret_cast<const __nv_bfloat16 *>(p.kidx_cache) + (size_t)bg * p.L_max * DI;

  // indexer queries of the 16 tokens (heads gR .. gR+R-1) and this lane's weights
  {
    constexpr int CHI = 2 * DI / 16;                             // 16-byte chunks per head row
    for (int c = lane; c < 16 * R * CHI; c += 32) {
      const int tk = c / (R * CHI), rem = c % (R * CHI), r = rem / CHI, ch = rem % CHI;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (tk < ntok)
        v = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.qidx) +
                                            (((size_t)b * p.T + tau0 + tk) * p.HI + g * R + r) * DI)[ch];
      *reinterpret_cast<uint4 *>(qis + tk * qstr + r * 2 * DI + ch * 16) = v;
    }
  }
  float w0[kMaxR], w1[kMaxR];
#pragma unroll
  for (int r = 0; r < kMaxR; ++r) {
    w0[r] = (ok0 && r < R) ? p.w[((size_t)b * p.T + tau0 + g4) * p.HI + g * R + r] : 0.f;
    w1[r] = (ok1 && r < R) ? p.w[((size_t)b * p.T + tau0 + g4 + 8) * p.HI + g * R + r] : 0.f;
  }
  __syncwarp();

  auto stage_tile = [&](int i) {                                  // keys 16i .. 16i+15 -> stage i & 1
    const uint32_t kdst = wb_u32 + (i & 1) * KG::STG, idst = kdst + 16 * KG::RS;
    constexpr int CH = 2 * D / 16, CHI = 2 * DI / 16;
    for (int c = lane; c < 16 * CH; c += 32) {
      const int r = c / CH, ch = c % CH, s = i * 16 + r;
      cp_async16(kdst + r * KG::RS + ch * 16, kc + (size_t)(s < p.L_max ? s : 0) * D + ch * 8, s < p.L_max);
    }
    for (int c = lane; c < 16 * CHI; c += 32) {
      const int r = c / CHI, ch = c % CHI, s = i * 16 + r;
      cp_async16(idst + r * KG::RSI + ch * 16, kic + (size_t)(s < p.L_max ? s : 0) * DI + ch * 8, s < p.L_max);
    }
    cp_async_commit();
  };

  const int ntiles = t_last / 16 + 1;
  const float scale = p.scale;
  float mc0 = -INFINITY, zc0 = 0.f, mc1 = -INFINITY, zc1 = 0.f;  // indexer statistics (head pass 0)
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    // A fragments of the 16 tokens' q for this head
    uint32_t qa[D / 16][4];
    {
      const uint32_t *q32 = reinterpret_cast<const uint32_t *>(p.q);
      const size_t r0 = (((size_t)b * p.T + tau0 + g4) * p.Hq + h) * D;
      const size_t r1 = (((size_t)b * p.T + tau0 + g4 + 8) * p.Hq + h) * D;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int k0 = ks * 16 + t2;
        qa[ks][0] = ok0 ? q32[(r0 + k0) >> 1] : 0u;
        qa[ks][1] = ok1 ? q32[(r1 + k0) >> 1] : 0u;
        qa[ks][2] = ok0 ? q32[(r0 + k0 + 8) >> 1] : 0u;
        qa[ks][3] = ok1 ? q32[(r1 + k0 + 8) >> 1] : 0u;
      }
    }
    float ma0 = -INFINITY, za0 = 0.f, wa0 = 0.f, ma1 = -INFINITY, za1 = 0.f, wa1 = 0.f;
    stage_tile(0);
    for (int i = 0; i < ntiles; ++i) {
      if (i + 1 < ntiles) {
        stage_tile(i + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncwarp();
      const uint32_t kt = wb_u32 + (i & 1) * KG::STG, it = kt + 16 * KG::RS;
      // teacher logits: S = Q K^T (two 8-key n-tiles)
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int ks2 = 0; ks2 < D / 32; ++ks2) {
          uint32_t bk[4];
          ldmatrix_x4(kt + (nt * 8 + (lane & 7)) * KG::RS + ks2 * 64 + (lane >> 3) * 16, bk[0], bk[1], bk[2], bk[3]);
          mma_16816_bf16(sc[nt], qa[2 * ks2], bk);
          mma_16816_bf16(sc[nt], qa[2 * ks2 + 1], bk + 2);
        }
      }
      // indexer logits: c = sum_r w_r relu(Q^I_r K^I^T)
      float cs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 1
      for (int r = 0; r < R; ++r) {
        float dr[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < DI / 16; ++ks) {
          uint32_t a[4];
          const int m = lane >> 3;
          ldmatrix_x4(smem_u32(qis) + ((m & 1) * 8 + (lane & 7)) * qstr + r * 2 * DI + ks * 32 + (m >> 1) * 16,
                      a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            uint32_t bi[2];
            uint32_t dummy0, dummy1;
            ldmatrix_x4(it + (nt * 8 + (lane & 7)) * KG::RSI + ks * 32 + ((lane >> 3) & 1) * 16, bi[0], bi[1], dummy0,
                        dummy1);
            (void)dummy0;
            (void)dummy1;
            mma_16816_bf16(dr[nt], a, bi);
          }
        }
        float wr0 = 0.f, wr1 = 0.f;
#pragma unroll
        for (int rr = 0; rr < kMaxR; ++rr)
          if (rr == r) {
            wr0 = w0[rr];
            wr1 = w1[rr];
          }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          cs[nt][0] = fmaf(wr0, fmaxf(dr[nt][0], 0.f), cs[nt][0]);
          cs[nt][1] = fmaf(wr0, fmaxf(dr[nt][1], 0.f), cs[nt][1]);
          cs[nt][2] = fmaf(wr1, fmaxf(dr[nt][2], 0.f), cs[nt][2]);
          cs[nt][3] = fmaf(wr1, fmaxf(dr[nt][3], 0.f), cs[nt][3]);
        }
      }
      // online statistics over this lane's valid columns (rows trow0 / trow1)
      float a4[2][4];
      float tm0 = -INFINITY, tm1 = -INFINITY, cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int s = i * 16 + nt * 8 + t2 + (j & 1);
          const bool row1 = j >= 2;
          const bool valid = row1 ? (ok1 && s <= trow1) : (ok0 && s <= trow0);
          a4[nt][j] = valid ? sc[nt][j] * scale : -INFINITY;
          if (!valid) cs[nt][j] = -INFINITY;
          if (row1) {
            tm1 = fmaxf(tm1, a4[nt][j]);
            cm1 = fmaxf(cm1, cs[nt][j]);
          } else {
            tm0 = fmaxf(tm0, a4[nt][j]);
            cm0 = fmaxf(cm0, cs[nt][j]);
          }
        }
      const float n0 = fmaxf(ma0, tm0), n1 = fmaxf(ma1, tm1);
      const float f0 = n0 == -INFINITY ? 1.f : expf(ma0 - n0), f1 = n1 == -INFINITY ? 1.f : expf(ma1 - n1);
      za0 *= f0;
      wa0 *= f0;
      za1 *= f1;
      wa1 *= f1;
      ma0 = n0;
      ma1 = n1;
      const bool first = hh == 0;
      float c0n = mc0, c1n = mc1, cf0 = 1.f, cf1 = 1.f;
      if (first) {
        c0n = fmaxf(mc0, cm0);
        c1n = fmaxf(mc1, cm1);
        cf0 = c0n == -INFINITY ? 1.f : expf(mc0 - c0n);
        cf1 = c1n == -INFINITY ? 1.f : expf(mc1 - c1n);
        zc0 *= cf0;
        zc1 *= cf1;
        mc0 = c0n;
        mc1 = c1n;
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a = a4[nt][j];
          if (a == -INFINITY) continue;
          const bool row1 = j >= 2;
          const float e = expf(a - (row1 ? ma1 : ma0));
          const float dlt = a - cs[nt][j];
          if (row1) {
            za1 += e;
            wa1 = fmaf(e, dlt, wa1);
            if (first) zc1 += expf(cs[nt][j] - mc1);
          } else {
            za0 += e;
            wa0 = fmaf(e, dlt, wa0);
            if (first) zc0 += expf(cs[nt][j] - mc0);
          }
        }
      __syncwarp();                                  // this stage may be refilled next
    }
    // merge the four lanes of each row (log-sum-exp merges), then the KL
    auto merge = [&](float &m, float &z, float &wv, bool with_w) {
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float zo = __shfl_xor_sync(0xffffffffu, z, o);
        const float wo = __shfl_xor_sync(0xffffffffu, wv, o);
        const float mn = fmaxf(m, mo);
        const float fa = m == -INFINITY ? 0.f : expf(m - mn), fb = mo == -INFINITY ? 0.f : expf(mo - mn);
        z = z * fa + zo * fb;
        if (with_w) wv = wv * fa + wo * fb;
        m = mn;
      }
    };
    float ta0 = ma0, tz0 = za0, tw0 = wa0, ta1 = ma1, tz1 = za1, tw1 = wa1;
    merge(ta0, tz0, tw0, true);
    merge(ta1, tz1, tw1, true);
    float cm0m = mc0, cz0 = zc0, cm1m = mc1, cz1 = zc1, dummy = 0.f;
    merge(cm0m, cz0, dummy, false);
    merge(cm1m, cz1, dummy, false);
    if ((lane & 3) == 0) {
      if (ok0)
        kl_out[((size_t)b * p.T + tau0 + g4) * p.Hq + h] = tw0 / tz0 - (ta0 + logf(tz0)) + (cm0m + logf(cz0));
      if (ok1)
        kl_out[((size_t)b * p.T + tau0 + g4 + 8) * p.Hq + h] = tw1 / tz1 - (ta1 + logf(tz1)) + (cm1m + logf(cz1));
    }
  }
}

template <int D, int DI>
static cudaError_t kl_t(const RowsParams &p, float *kl_out, cudaStream_t st) {
  const int smem = kKlWarps * KlGeom<D, DI>::warp_bytes(p.R);
  cudaError_t e = prepare_kernel(indexer_kl_kernel<D, DI>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.T + 16 * kKlWarps - 1) / (16 * kKlWarps), p.B * p.Hkv);
  indexer_kl_kernel<D, DI><<<grid, kKlWarps * 32, smem, st>>>(p, kl_out);
  return cudaGetLastError();
}

cudaError_t launch_indexer_kl(const RowsParams &p, float *kl_out, cudaStream_t st) {
  if (indexer_kl_tc_supported(p)) return launch_indexer_kl_tc(p, kl_out, st);   // tcgen05 (lisa_kl_tc.cu)
  if (p.D == 128 && p.DI == 64) return kl_t<128, 64>(p, kl_out, st);
  if (p.D == 128 && p.DI == 32) return kl_t<128, 32>(p, kl_out, st);
  if (p.D == 64 && p.DI == 64) return kl_t<64, 64>(p, kl_out, st);
  if (p.D == 64 && p.DI == 32) return kl_t<64, 32>(p, kl_out, st);
  return cudaErrorInvalidValue;
}

}  // namespace lisa
