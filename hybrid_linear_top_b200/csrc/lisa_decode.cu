// LISA decode step on sm_100a: three kernels chained with programmatic
// dependent launch.
//
//   1. score_state: streams the indexer-key cache with 1-D TMA bulk copies into
//      shared memory and writes one order key per (b, g, s); in the same grid,
//      extra CTAs do the linear-state read-modify-write S <- S + k^T v and
//      o_lin = q S, and the CTA owning the new row appends it to the caches.
//   2. select: one CTA per (b, g) turns the order keys into the top-M set.
//   3. attend: split-M sparse attention over the gathered K/V rows, merged by
//      the last CTA of each (b, g), which also applies the gate.
//
// Method: arXiv 2607.19358 (LISA), abstract and the gptget.net digest's method
// section; exact formulas as stated in lisa.h.
#include "lisa_internal.h"
#include "lisa_select.cuh"

namespace lisa {

// ============================================================ kernel 1
template <typename T, int DI>
struct ScoreCfg {
  static constexpr int kRowBytes = DI * Dt<T>::kBytes;
  static constexpr int kLanesPerKey = kRowBytes / 16;          // 16-byte slices per key row
  static constexpr int kVec = 16 / Dt<T>::kBytes;              // elements per slice
  static constexpr int kThreads = 256;
  static constexpr int kKeysPerIter = kThreads / kLanesPerKey;
  static constexpr int kChunk = 128;                           // keys per CTA
};

template <typename T, int D, int DI>
__global__ void __launch_bounds__(256) decode_score_state_kernel(DecodeParams p) {
  using C = ScoreCfg<T, DI>;
  __shared__ __align__(128) unsigned char s_rows[C::kChunk * C::kRowBytes];
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ float s_red[256 / 8][33];

  // Let the select kernel get scheduled as soon as every CTA of this grid runs.
  grid_dep_launch();

  const int tid = threadIdx.x;
  if (blockIdx.x == 0)
    for (int i = tid; i < p.B * p.Hkv; i += blockDim.x) p.counters[i] = 0;

  if ((int)blockIdx.x < p.n_score_blocks) {
    // -------------------------------------------------- indexer score
    const int chunks = p.n_chunks;
    const int c = blockIdx.x % chunks;
    const int bg = blockIdx.x / chunks;
    const int g = bg % p.Hkv;
    const int b = bg / p.Hkv;
    const int t = p.pos[b];
    if (t < 0 || t >= p.L_max) {
      if (c == 0 && tid == 0) set_err(p.err_word, LISA_DEVERR_POS);
      return;
    }
    const int s0 = c * C::kChunk;
    if (s0 > t) return;
    const int s_end = min(s0 + C::kChunk, t + 1);  // exclusive
    const int n_cached = min(s_end, t) - s0;       // rows read from the cache

    // append the new token (row t) when this CTA owns it
    if (p.fuse_append && t >= s0 && t < s0 + C::kChunk) {
      const size_t row = ((size_t)b * p.Hkv + g) * p.L_max + t;
      const T *kin = reinterpret_cast<const T *>(p.k) + ((size_t)b * p.Hkv + g) * D;
      const T *vin = reinterpret_cast<const T *>(p.v) + ((size_t)b * p.Hkv + g) * D;
      const T *kiin = reinterpret_cast<const T *>(p.kidx) + ((size_t)b * p.Hkv + g) * DI;
      T *kc = reinterpret_cast<T *>(p.k_cache) + row * D;
      T *vc = reinterpret_cast<T *>(p.v_cache) + row * D;
      T *kic = reinterpret_cast<T *>(p.kidx_cache) + row * DI;
      for (int i = tid; i < D; i += blockDim.x) {
        kc[i] = kin[i];
        vc[i] = vin[i];
      }
      for (int i = tid; i < DI; i += blockDim.x) kic[i] = kiin[i];
    }

    const unsigned char *src = reinterpret_cast<const unsigned char *>(p.kidx_cache) +
                               (((size_t)b * p.Hkv + g) * p.L_max + s0) * C::kRowBytes;
    if (tid == 0) {
      mbar_init(&s_bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
      const uint32_t bytes = (uint32_t)n_cached * C::kRowBytes;
      if (bytes) {
        mbar_arrive_expect_tx(&s_bar, bytes);
        bulk_g2s(s_rows, src, bytes, &s_bar);
      } else {
        mbar_arrive(&s_bar);
      }
    }
    // the new token's indexer key comes from the argument
    if (t < s_end) {
      const unsigned char *kin =
          reinterpret_cast<const unsigned char *>(p.kidx) + ((size_t)b * p.Hkv + g) * C::kRowBytes;
      for (int i = tid; i < C::kRowBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(s_rows + (size_t)(t - s0) * C::kRowBytes)[i] =
            reinterpret_cast<const uint4 *>(kin)[i];
    }

    // indexer queries and weights of the R heads of this KV head -> registers
    const int part = tid % C::kLanesPerKey;
    float qv[kMaxR][C::kVec];
    float wv[kMaxR];
#pragma unroll
    for (int r = 0; r < kMaxR; ++r) {
      wv[r] = 0.f;
#pragma unroll
      for (int j = 0; j < C::kVec; ++j) qv[r][j] = 0.f;
      if (r < p.R) {
        const int hi = g * p.R + r;
        const T *qrow = reinterpret_cast<const T *>(p.qidx) + ((size_t)b * p.HI + hi) * DI;
        uint4 u = *reinterpret_cast<const uint4 *>(qrow + part * C::kVec);
        Vec16<T>::unpack(u, qv[r]);
        wv[r] = p.w[(size_t)b * p.HI + hi];
      }
    }
    __syncthreads();  // new-token row visible
    if (!mbar_wait_bounded(&s_bar, 0)) {
      if (tid == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
      return;
    }

    uint32_t *keys_out = p.keys + ((size_t)b * p.Hkv + g) * p.keys_stride;
    const int n = s_end - s0;
    for (int base = 0; base < n; base += C::kKeysPerIter) {
      const int kk = base + tid / C::kLanesPerKey;
      float x[C::kVec];
      if (kk < n) {
        uint4 u = *reinterpret_cast<const uint4 *>(s_rows + (size_t)kk * C::kRowBytes + part * 16);
        Vec16<T>::unpack(u, x);
      } else {
#pragma unroll
        for (int j = 0; j < C::kVec; ++j) x[j] = 0.f;
      }
      float score = 0.f;
#pragma unroll
      for (int r = 0; r < kMaxR; ++r) {
        if (r < p.R) {
          float dot = 0.f;
#pragma unroll
          for (int j = 0; j < C::kVec; ++j) dot = fmaf(qv[r][j], x[j], dot);
#pragma unroll
          for (int o = C::kLanesPerKey / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
          score = fmaf(wv[r], fmaxf(dot, 0.f), score);
        }
      }
      if (part == 0 && kk < n) keys_out[s0 + kk] = score_key(score);
    }
    return;
  }

  // -------------------------------------------------- linear state
  // CTA = (b, h, 32-column slab); thread = (row group, float4 column)
  const int sb = blockIdx.x - p.n_score_blocks;
  constexpr int kSlabs = D / 32;
  const int slab = sb % kSlabs;
  const int bh = sb / kSlabs;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int t = p.pos[b];
  if (t < 0 || t >= p.L_max) return;
  const int g = h / p.G;
  const int cg = tid & 7;           // float4 column within the slab
  const int rg = tid >> 3;          // 32 row groups
  const int j0 = slab * 32 + cg * 4;
  const T *kin = reinterpret_cast<const T *>(p.k) + ((size_t)b * p.Hkv + g) * D;
  const T *vin = reinterpret_cast<const T *>(p.v) + ((size_t)b * p.Hkv + g) * D;
  const T *qin = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + h) * D;
  float vj[4];
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) vj[c4] = Dt<T>::to_f(vin[j0 + c4]);
  float* S = p.state + ((size_t)b * p.Hq + h) * D * D;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float4 sv[D / 32];
#pragma unroll
  for (int it = 0; it < D / 32; ++it) {
    const int i = rg + 32 * it;
    sv[it] = *reinterpret_cast<const float4 *>(S + (size_t)i * D + j0);
  }
#pragma unroll
  for (int it = 0; it < D / 32; ++it) {
    const int i = rg + 32 * it;
    const float ki = Dt<T>::to_f(kin[i]);
    const float qi = Dt<T>::to_f(qin[i]);
    float4 s = sv[it];
    s.x = fmaf(ki, vj[0], s.x);
    s.y = fmaf(ki, vj[1], s.y);
    s.z = fmaf(ki, vj[2], s.z);
    s.w = fmaf(ki, vj[3], s.w);
    *reinterpret_cast<float4 *>(S + (size_t)i * D + j0) = s;
    acc[0] = fmaf(qi, s.x, acc[0]);
    acc[1] = fmaf(qi, s.y, acc[1]);
    acc[2] = fmaf(qi, s.z, acc[2]);
    acc[3] = fmaf(qi, s.w, acc[3]);
  }
  // reduce over the 32 row groups: s_red[rg][col]
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) s_red[rg][cg * 4 + c4] = acc[c4];
  __syncthreads();
  if (tid < 32) {
    float o = 0.f;
    for (int r = 0; r < 32; ++r) o += s_red[r][tid];
    p.olin[((size_t)b * p.Hq + h) * D + slab * 32 + tid] = o;
  }
}

// ============================================================ kernel 2
template <int NT>
__global__ void __launch_bounds__(NT) decode_select_kernel(DecodeParams p) {
  extern __shared__ __align__(16) uint32_t s_dyn[];
  __shared__ TopmShared sm;
  grid_dep_wait();
  grid_dep_launch();
  const int bg = blockIdx.x;
  const int b = bg / p.Hkv;
  const int t = p.pos[b];
  if (t < 0 || t >= p.L_max) return;
  const int n = t + 1;
  const uint32_t *gkeys = p.keys + (size_t)bg * p.keys_stride;
  const uint32_t *keys = gkeys;
  uint32_t *cand = s_dyn;
  if (n <= p.smem_keys_cap && n > p.M) {
    uint32_t *sk = s_dyn;
    const int n4 = n & ~3;
    for (int i = threadIdx.x * 4; i < n4; i += NT * 4)
      *reinterpret_cast<uint4 *>(sk + i) = __ldcg(reinterpret_cast<const uint4 *>(gkeys + i));
    for (int i = n4 + threadIdx.x; i < n; i += NT) sk[i] = __ldcg(gkeys + i);
    __syncthreads();
    keys = sk;
    cand = s_dyn + p.smem_keys_cap;
  }
  int *out = p.idx + (size_t)bg * p.M;
  if (!block_topm<NT>(keys, n, p.M, out, sm, cand, p.cand_cap) && threadIdx.x == 0)
    set_err(p.err_word, LISA_DEVERR_CHECK);
  if (p.idx_out) {
    __syncthreads();
    for (int i = threadIdx.x; i < p.M; i += NT) p.idx_out[(size_t)bg * p.M + i] = __ldcg(out + i);
  }
}

// ============================================================ kernel 3
// CTA = (b, g, split of kRows selected rows); 256 threads = 8 warps.
template <typename T, int D>
__global__ void __launch_bounds__(256) decode_attend_kernel(DecodeParams p) {
  constexpr int kRows = kAttnRows;     // selected rows per CTA
  constexpr int kDPL = D / 32;         // dims per lane
  __shared__ __align__(16) T s_k[kRows][D];
  __shared__ __align__(16) T s_v[kRows][D];
  __shared__ float s_q[kMaxG][D];
  __shared__ float s_logit[kMaxG][kRows];
  __shared__ int s_idx[kRows];
  __shared__ int s_last;

  grid_dep_wait();
  grid_dep_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nsplit = p.M / kRows;
  const int sp = blockIdx.x % nsplit;
  const int bg = blockIdx.x / nsplit;
  const int g = bg % p.Hkv;
  const int b = bg / p.Hkv;
  const int t = p.pos[b];
  if (t < 0 || t >= p.L_max) return;
  const int G = p.G;

  if (tid < kRows) {
    int s = __ldcg(p.idx + (size_t)bg * p.M + sp * kRows + tid);
    if (s < -1 || s > t) {
      set_err(p.err_word, LISA_DEVERR_CHECK);
      s = -1;
    }
    s_idx[tid] = s;
  }
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int hh = i / D, dd = i % D;
    s_q[hh][dd] = Dt<T>::to_f(reinterpret_cast<const T *>(p.q)[((size_t)b * p.Hq + g * G + hh) * D + dd]);
  }
  __syncthreads();

  // gather K and V rows (16-byte loads); the new token comes from the arguments
  constexpr int kSlices = D * (int)sizeof(T) / 16;
  const T *kc = reinterpret_cast<const T *>(p.k_cache) + ((size_t)b * p.Hkv + g) * p.L_max * D;
  const T *vc = reinterpret_cast<const T *>(p.v_cache) + ((size_t)b * p.Hkv + g) * p.L_max * D;
  const T *kn = reinterpret_cast<const T *>(p.k) + ((size_t)b * p.Hkv + g) * D;
  const T *vn = reinterpret_cast<const T *>(p.v) + ((size_t)b * p.Hkv + g) * D;
  for (int i = tid; i < kRows * kSlices; i += blockDim.x) {
    const int r = i / kSlices, sl = i % kSlices;
    const int s = s_idx[r];
    uint4 uk = make_uint4(0, 0, 0, 0), uv = make_uint4(0, 0, 0, 0);
    if (s >= 0) {
      const T *ks = (s == t) ? kn : kc + (size_t)s * D;
      const T *vs = (s == t) ? vn : vc + (size_t)s * D;
      uk = *reinterpret_cast<const uint4 *>(ks + sl * (16 / sizeof(T)));
      uv = *reinterpret_cast<const uint4 *>(vs + sl * (16 / sizeof(T)));
    }
    reinterpret_cast<uint4 *>(&s_k[r][0])[sl] = uk;
    reinterpret_cast<uint4 *>(&s_v[r][0])[sl] = uv;
  }
  __syncthreads();

  // logits: warp per row, lanes split d
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

  // per head: local max, exp, sum, and the weighted V sum -> partials
  float *part = p.partials + (((size_t)bg * nsplit + sp) * G) * (D + 2);
  for (int hh = warp; hh < G; hh += 8) {
    float m = s_logit[hh][lane];  // kRows == 32
    m = warp_max(m);
    const float e = (m == -INFINITY) ? 0.f : expf(s_logit[hh][lane] - m);
    const float l = warp_sum(e);
    s_logit[hh][lane] = e;
    __syncwarp();
    float acc[kDPL];
#pragma unroll
    for (int j = 0; j < kDPL; ++j) acc[j] = 0.f;
    for (int r = 0; r < kRows; ++r) {
      const float pr = s_logit[hh][r];
#pragma unroll
      for (int j = 0; j < kDPL; ++j) acc[j] = fmaf(pr, Dt<T>::to_f(s_v[r][lane * kDPL + j]), acc[j]);
    }
    float *ph = part + (size_t)hh * (D + 2);
#pragma unroll
    for (int j = 0; j < kDPL; ++j) ph[lane * kDPL + j] = acc[j];
    if (lane == 0) {
      ph[D] = m;
      ph[D + 1] = l;
    }
  }

  // last CTA of this (b, g) merges the splits and applies the gate
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(p.counters + bg, 1u) == (unsigned)(nsplit - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float *pb = p.partials + ((size_t)bg * nsplit) * G * (D + 2);
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int hh = i / D, dd = i % D;
    float mx = -INFINITY;
    for (int s2 = 0; s2 < nsplit; ++s2) mx = fmaxf(mx, __ldcg(pb + ((size_t)s2 * G + hh) * (D + 2) + D));
    float num = 0.f, den = 0.f;
    for (int s2 = 0; s2 < nsplit; ++s2) {
      const float *ph = pb + ((size_t)s2 * G + hh) * (D + 2);
      const float ms = __ldcg(ph + D);
      if (ms == -INFINITY) continue;
      const float f = expf(ms - mx);
      num = fmaf(f, __ldcg(ph + dd), num);
      den = fmaf(f, __ldcg(ph + D + 1), den);
    }
    const int h = g * G + hh;
    const float o_sp = num / den;
    const float o_lin = __ldcg(p.olin + ((size_t)b * p.Hq + h) * D + dd);
    const float gam = 1.f / (1.f + expf(-p.gate[(size_t)b * p.Hq + h]));
    const float o = gam * o_sp + (1.f - gam) * o_lin;
    reinterpret_cast<T *>(p.out)[((size_t)b * p.Hq + h) * D + dd] = Dt<T>::from_f(o);
  }
}

// ============================================================ launcher
template <typename T, int D, int DI>
static cudaError_t launch_decode_t(const DecodeParams &p, cudaStream_t st) {
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;

  {
    cudaError_t e = prepare_kernel(decode_score_state_kernel<T, D, DI>);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_score_blocks + p.n_state_blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    e = cudaLaunchKernelEx(&cfg, decode_score_state_kernel<T, D, DI>, p);
    if (e != cudaSuccess) return e;
  }
  {
    constexpr int NT = 1024;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.B * p.Hkv);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = p.select_smem;
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    cudaError_t e = prepare_kernel(decode_select_kernel<NT>, (int)p.select_smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_select_kernel<NT>, p);
    if (e != cudaSuccess) return e;
  }
  {
    cudaError_t e = prepare_kernel(decode_attend_kernel<T, D>);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.B * p.Hkv * (p.M / kAttnRows));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_attend_kernel<T, D>, p);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeParams &p, int dtype, cudaStream_t st) {
  if (dtype == LISA_BF16) {
    if (p.D == 128 && p.DI == 64) return launch_decode_t<__nv_bfloat16, 128, 64>(p, st);
    if (p.D == 128 && p.DI == 32) return launch_decode_t<__nv_bfloat16, 128, 32>(p, st);
    if (p.D == 64 && p.DI == 64) return launch_decode_t<__nv_bfloat16, 64, 64>(p, st);
    if (p.D == 64 && p.DI == 32) return launch_decode_t<__nv_bfloat16, 64, 32>(p, st);
  } else {
    if (p.D == 128 && p.DI == 64) return launch_decode_t<float, 128, 64>(p, st);
    if (p.D == 128 && p.DI == 32) return launch_decode_t<float, 128, 32>(p, st);
    if (p.D == 64 && p.DI == 64) return launch_decode_t<float, 64, 64>(p, st);
    if (p.D == 64 && p.DI == 32) return launch_decode_t<float, 64, 32>(p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace lisa
