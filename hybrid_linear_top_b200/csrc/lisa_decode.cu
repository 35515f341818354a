// LISA decode step on sm_100a: one kernel, one thread-block cluster of NC CTAs
// (NC = 16, 8 or 4; see the launcher) per (sequence b, KV head g).
//
// Method: arXiv 2607.19358 (LISA).  Abstract: a Lightning Indexer keeps the
// top-M tokens of the context for a sparse softmax attention, a linear
// attention runs beside it and a gate fuses the two.  gptget.net digest,
// method section: phi = identity with a state matrix S_t; indexer = ReLU dot
// products of small query/key projections.  Exact formulas: include/lisa.h.
//
// Work of one cluster (CTA rank r of NC):
//   1. stream its contiguous slice of the (b, g) indexer-key cache through a
//      TMA ring and score every key, keeping 32-bit order keys in
//      shared memory (NC = 16: 4 stages of 32 KB; NC <= 8: 2 stages, so two
//      CTAs fit one SM).  bf16: 2-D tiled TMA with a 64/128-byte swizzle and warp
//      tensor-core MMAs (keys x indexer heads); fp32: 1-D bulk copies and one
//      thread per key on the CUDA cores.  Meanwhile the columns
//      [r*d/NC, (r+1)*d/NC) of the linear state of the G query heads are
//      loaded, updated (S += k^T v) and read out (o_lin = q S);
//   2. exact top-M in one round of distributed-shared-memory messages: each
//      CTA bins its keys (1024 range bins over the 8 octaves below its
//      largest key), takes its bound theta (the kl-th largest key's bin) and
//      a send threshold (fewer than SEG keys above it), and sends every other
//      CTA one fixed-size message: both values, its largest key and its keys
//      above the threshold, in position order (st.async onto the receiver's
//      mbarrier).  With lb = min theta, the messages hold every key >= lb iff
//      every threshold is <= lb; then each CTA finds the M-th key exactly
//      from the candidates (range histograms, a one-warp resolve) and emits
//      the whole ascending index list itself.  Otherwise a cluster-wide
//      radix select (histograms summed over distributed shared memory)
//      builds the list in CTA 0;
//   3. gather M/NC of the selected K/V rows, partial softmax for the G heads;
//   4. every CTA sends each other CTA its partials of that CTA's columns
//      (st.async onto a second mbarrier); each merges its column slice,
//      applies the gate and stores.
// The wide form (nw CTAs per (b, g)) streams and scores over nw CTAs and
// hands the keys to the last cluster through a workspace.  Nothing else
// leaves the cluster but the outputs, the state and the appended cache row.
#include <cooperative_groups.h>
#include <string.h>

#include "lisa_internal.h"
#include "lisa_common.cuh"
#include "lisa_select.cuh"

namespace cg = cooperative_groups;

namespace lisa {

constexpr int kDecThreads = 256;
constexpr int kStages = 4;        // ring stages at most (the launcher picks 2 or 4)
constexpr int kStageBytes = 32768;  // ring stage size at most (the launcher picks 16 or 32 KB)

template <typename T, int DI>
struct ScoreGeom {
  static constexpr int RB = DI * (int)sizeof(T);                              // key row bytes
  // keys per ring stage of `stage_bytes`
  static __host__ __device__ int sub(int stage_bytes) { return (stage_bytes / RB) < 256 ? stage_bytes / RB : 256; }
  static constexpr bool kMma = sizeof(T) == 2;                                // bf16: swizzled tiles + MMA
};

struct DecLayout {
  int region0, xin, pout, pin;
  int keys, hist, tot, misc, sel, qs, qi, ks, vs, kis, gl, klin, vlin, olin, logit, sidx, wred, bars, total;
};

// Candidate slots each CTA of an NC-CTA cluster sends in the top-M exchange:
// 1024 over the cluster, but 128 each for 4 CTAs (two such CTAs share an SM).
__host__ __device__ constexpr int dec_seg(int NC) { return NC <= 4 ? 128 : 1024 / NC; }
// Words of one candidate message: a 4-word header (bound, largest key, send
// threshold, count) and dec_seg(NC) keys and positions.
__host__ __device__ constexpr int dec_msg_words(int NC) { return 4 + 2 * dec_seg(NC); }
// Floats of one merge message: a sender's partial outputs of the G heads on
// the receiver's D / NC columns, then its G (max, sum) pairs; 16-byte multiple.
__host__ __device__ constexpr int dec_merge_words(int G, int D, int NC) { return (G * (D / NC) + 2 * G + 3) & ~3; }

__host__ __device__ inline int align16(int x) { return (x + 15) & ~15; }

// Byte offsets of the dynamic shared-memory carve-up, relative to a
// 1024-byte aligned base (host and device agree; `total` includes the slack
// needed to align the base).  region0 holds the TMA ring (scoring), later the
// gathered K / V rows (attention) followed by the merge messages (pout: this
// CTA's, pin: the other CTAs').  Another CTA writes into pin only after it
// has this CTA's candidate message, which is sent after the last ring stage
// is consumed; candidate messages (xin) arrive while this CTA may still be
// scoring, so they have a region of their own.
__host__ __device__ inline DecLayout dec_layout(int kpc_max, int L_max, int M, int G, int D, int DI, int esize,
                                                int NC, int stages = kStages, int stage_bytes = kStageBytes,
                                                bool lin_kv = false, bool wide = false) {
  DecLayout L;
  const int rpc = M / NC;
  const int kv = 2 * rpc * (D * esize + 16);
  const int ring = stages * stage_bytes;
  const int mw = dec_merge_words(G, D, NC);
  const int kvm = align16(kv) + 2 * NC * mw * 4;      // K / V rows, then [NC][mw] pout and [NC][mw] pin
  const int r0 = ring > kvm ? ring : kvm;
  int off = 0;
  L.region0 = off; off += align16(r0);
  L.pout = L.region0 + align16(kv);                   // [NC owners] this CTA's merge messages
  L.pin = L.pout + NC * mw * 4;                       // [NC senders] merge messages for this CTA's columns
  L.xin = off; off += NC * dec_msg_words(NC) * 4;     // [NC senders] candidate messages (own in slot rank)
  L.keys = off; off += align16(kpc_max * 4);
  L.hist = off; off += 8 * 256 * 4;
  L.tot = off; off += 256 * 4;
  L.misc = off; off += 64 * 4;
  L.sel = off; off += align16(M * 4);
  L.qs = off; off += align16(G * D * 4);
  L.qi = off; off += align16(kMaxR * DI * 4 + kMaxR * 4);
  L.ks = off; off += align16(D * 4);
  L.vs = off; off += align16(D * 4);
  L.kis = off; off += align16(DI * 4);
  L.gl = off; off += align16(G * 4);
  L.klin = off; off += lin_kv ? align16(G * D * 4) : 0;   // linear-branch k, v per query head (variant)
  L.vlin = off; off += lin_kv ? align16(G * D * 4) : 0;
  L.olin = off; off += align16(G * (D / NC) * 4);
  {
    const int a = G * rpc * 4, bred = 8 * 8 * (D / NC) * 4;   // logits, or the o_lin reduction scratch
    L.logit = off; off += align16(a > bred ? a : bred);
  }
  L.sidx = off; off += align16(rpc * 4);
  L.wred = off; off += wide ? align16(2 * 8 * D * 4) : 0;   // wide form: [2 heads][8 warps][D] readout sums
  L.bars = off; off += (kStages + 2) * 8;             // ring stages, candidate messages, merge messages
  L.total = align16(off) + 1024;
  return L;
}

// Warp 0 scans 256 bins from the top and finds the one holding the rem-th
// largest key: misc[0] = bin, misc[1] = keys in higher bins.  Other lanes idle.
__device__ __forceinline__ void dec_find_bucket(const uint32_t *tot, uint32_t *misc, uint32_t rem) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = tot[255 - (8 * lane + j)];
      sum += c[j];
    }
    uint32_t inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const uint32_t exc = inc - sum;
    if (exc < rem && rem <= inc) {
      uint32_t cum = exc;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (cum + c[j] >= rem) {
          misc[0] = 255u - (uint32_t)(8 * lane + j);
          misc[1] = cum;
          break;
        }
        cum += c[j];
      }
    }
  }
}

template <typename T, int D, int DI, int NC, bool WIDE = false>
__global__ void __launch_bounds__(kDecThreads, (NC <= 8 && sizeof(T) == 2) ? 2 : 1)
    decode_cluster_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap kmap) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  using SG = ScoreGeom<T, DI>;
  constexpr int RB = SG::RB;                     // indexer-key row bytes
  constexpr int NCH = RB / 16;                   // 16-byte chunks per key row
  constexpr int VEC = 16 / (int)sizeof(T);       // elements per chunk
  constexpr int COLS = D / NC;                   // state / output columns of this CTA
  constexpr int QPR = COLS / 4;                  // float4 per state row slice
  constexpr int ITER = (D * QPR + kDecThreads - 1) / kDecThreads;
  constexpr int HP = (16 / ITER) < 8 ? (16 / ITER < 1 ? 1 : 16 / ITER) : 8;   // state heads held in registers at once
  constexpr int ROWB = D * (int)sizeof(T);       // K / V row bytes
  constexpr int RS = ROWB + 16;                  // padded K / V row stride in shared memory
  constexpr int SL = ROWB / 16;                  // 16-byte slices per K / V row

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  // Cluster form: the NC CTAs of one cluster serve (b, g); CTA `rank` scores
  // key slice `rank` and owns state columns slab `rank`.  Wide form: NSL CTAs
  // (NSL / NC clusters) serve (b, g); CTA `slice` scores key slice `slice`
  // and updates state rows slab `slice`, and the last cluster to finish
  // selects and attends.
  const int NSL = WIDE ? p.nw : NC;
  const int bg = blockIdx.x / NSL;
  const int slice = WIDE ? (int)(blockIdx.x % NSL) : rank;
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G, M = p.M, R = p.R;
  const int rpc = M / NC;

  // 1024-byte aligned base: the swizzled TMA tiles depend on address bits 4..9
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int NS = p.stages;
  const int SUB = p.stage_keys;                  // keys per ring stage
  const int STB = SUB * RB;                      // bytes per ring stage
  const bool lin_kv = p.k_lin != nullptr;  // variant: linear-branch k, v of its own per query head
  const DecLayout lay = dec_layout(p.kpc_max, p.L_max, M, G, D, DI, (int)sizeof(T), NC, NS, STB, lin_kv, WIDE);
  unsigned char *ring = smem + lay.region0;
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem + lay.keys);
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem + lay.hist);
  uint32_t *tot = reinterpret_cast<uint32_t *>(smem + lay.tot);
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + lay.misc);
  int *sel = reinterpret_cast<int *>(smem + lay.sel);
  float *qs = reinterpret_cast<float *>(smem + lay.qs);
  float *qis = reinterpret_cast<float *>(smem + lay.qi);   // [R][DI] indexer queries, then [R] weights
  float *ks = reinterpret_cast<float *>(smem + lay.ks);
  float *vs = reinterpret_cast<float *>(smem + lay.vs);
  float *kis = reinterpret_cast<float *>(smem + lay.kis);   // the new token's indexer key
  float *gls = reinterpret_cast<float *>(smem + lay.gl);    // gate logits of the G heads
  float *klin = reinterpret_cast<float *>(smem + lay.klin); // [G][D] (variant only)
  float *vlin = reinterpret_cast<float *>(smem + lay.vlin); // [G][D] (variant only)
  const int MW = dec_merge_words(G, D, NC);            // floats per merge message
  float *pout = reinterpret_cast<float *>(smem + lay.pout);   // [NC owners][MW] this CTA's merge messages
  float *pin = reinterpret_cast<float *>(smem + lay.pin);     // [NC senders][MW] messages for this CTA's columns
  float *olin = reinterpret_cast<float *>(smem + lay.olin);
  float *logit = reinterpret_cast<float *>(smem + lay.logit);
  int *sidx = reinterpret_cast<int *>(smem + lay.sidx);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.bars);

  // barrier init touches shared memory only: before the wait on the previous kernel
  uint64_t *mbx = &bars[kStages];          // candidate messages of the other CTAs (top-M exchange)
  uint64_t *mbm = &bars[kStages + 1];      // merge messages of the other CTAs
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
    mbar_init(mbx, 1);
    mbar_init(mbm, 1);
    fence_mbar_init();
    // armed once: each completes when the other NC - 1 CTAs' messages are in
    mbar_arrive_expect_tx(mbx, (uint32_t)((NC - 1) * dec_msg_words(NC) * 4));
    mbar_arrive_expect_tx(mbm, (uint32_t)((NC - 1) * dec_merge_words(G, D, NC) * 4));
    if constexpr (WIDE) misc[60] = 0u;   // "this cluster holds the last arrival" (wide form)
  }
  if (p.independent) {
    // The caller declared this step independent of the launch before it on the
    // stream: no wait, and the launch after it may start at once.
    grid_dep_launch();
  } else {
    // Everything read below may have been written by the previous kernel.
    grid_dep_wait();
  }
  if (p.debug_flags & LISA_DEBUG_FORCE_TIMEOUT) {
    // Failure-path test: no copy has been issued, so the first ring stage
    // never completes and the bounded wait runs out.  Every CTA of the
    // cluster returns here, before any cluster barrier or copy.
    __syncthreads();                     // the barriers are initialised
    const bool done = mbar_wait_bounded(&bars[0], 0u, 20000ull);
    if (!done && tid == 0) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
    return;
  }

  const int t = p.pos[b];                  // in flight while the loads below are issued
  const T *kidx_cache = reinterpret_cast<const T *>(p.kidx_cache) + (size_t)bg * p.L_max * DI;
  const T *kidx_new = reinterpret_cast<const T *>(p.kidx) + (size_t)bg * DI;

  // ---------------------------------------------------------------- early loads
  const T *qin = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + g * G) * D;
  const T *kin = reinterpret_cast<const T *>(p.k) + (size_t)bg * D;
  const T *vin = reinterpret_cast<const T *>(p.v) + (size_t)bg * D;
  const T *qidx_in = reinterpret_cast<const T *>(p.qidx) + ((size_t)b * p.HI + g * R) * DI;
  const bool ext = p.sel_ext != nullptr;  // index lists given by the caller
  const bool window = p.window != 0 || ext;   // no indexer, no top-M: the window's lists or the given ones
  // The step's own rows as 16-byte chunks, [q of the G heads | k | v |
  // indexer queries of the R heads | new indexer key | linear-branch k, v of
  // the G heads (variant)], loaded into registers with every load in flight
  // at once (one DRAM round trip, not one per row), then widened into shared
  // memory below.
  const int o_k = G * D / VEC, o_v = o_k + D / VEC, o_qi = o_v + D / VEC;
  const int o_ki = o_qi + (window ? 0 : R * DI / VEC);
  const int o_kl = o_ki + (p.kidx ? DI / VEC : 0);
  const int o_vl = o_kl + (lin_kv ? G * D / VEC : 0);
  const int n_in = o_vl + (lin_kv ? G * D / VEC : 0);
  const size_t lin_off = ((size_t)b * p.Hq + g * G) * D;
  auto chunk_src = [&](int c) -> const uint4 * {
    if (c < o_k) return reinterpret_cast<const uint4 *>(qin) + c;
    if (c < o_v) return reinterpret_cast<const uint4 *>(kin) + (c - o_k);
    if (c < o_qi) return reinterpret_cast<const uint4 *>(vin) + (c - o_v);
    if (c < o_ki) return reinterpret_cast<const uint4 *>(qidx_in) + (c - o_qi);
    if (c < o_kl) return reinterpret_cast<const uint4 *>(kidx_new) + (c - o_ki);
    if (c < o_vl) return reinterpret_cast<const uint4 *>(reinterpret_cast<const T *>(p.k_lin) + lin_off) + (c - o_kl);
    return reinterpret_cast<const uint4 *>(reinterpret_cast<const T *>(p.v_lin) + lin_off) + (c - o_vl);
  };
  auto chunk_dst = [&](int c) -> float * {
    if (c < o_k) return qs + c * VEC;
    if (c < o_v) return ks + (c - o_k) * VEC;
    if (c < o_qi) return vs + (c - o_v) * VEC;
    if (c < o_ki) return qis + (c - o_qi) * VEC;
    if (c < o_kl) return kis + (c - o_ki) * VEC;
    if (c < o_vl) return klin + (c - o_kl) * VEC;
    return vlin + (c - o_vl) * VEC;
  };
  constexpr int kInRegs = 2;               // chunks per thread held in registers
  uint4 inr[kInRegs];
#pragma unroll
  for (int j = 0; j < kInRegs; ++j)
    if (tid + j * kDecThreads < n_in) inr[j] = *chunk_src(tid + j * kDecThreads);
  const float w_in = (!window && tid < R) ? p.w[(size_t)b * p.HI + g * R + tid] : 0.f;
  const float gl_in = tid < G ? p.gate[(size_t)b * p.Hq + g * G + tid] : 0.f;
  // state slab of the first (up to) HP query heads
  const int c0s = rank * COLS;
  const int cq = tid % QPR;                // same float4 column for every row this thread visits
  const int gA = min(G, HP);
  float4 sv[HP][ITER];
  if constexpr (!WIDE) {
#pragma unroll
    for (int hh = 0; hh < HP; ++hh) {
      if (hh >= gA) continue;
      const float *S = p.state + ((size_t)b * p.Hq + g * G + hh) * D * D;
#pragma unroll
      for (int it = 0; it < ITER; ++it) {
        const int idx = tid + it * kDecThreads;
        if (idx < D * QPR) sv[hh][it] = *reinterpret_cast<const float4 *>(S + (size_t)(idx / QPR) * D + c0s + cq * 4);
      }
    }
    // heads beyond the first HP: their slab rows requested into L2 now
    for (int i = tid; i < (G - gA) * D; i += kDecThreads)
      prefetch_l2(p.state + ((size_t)b * p.Hq + g * G + gA + i / D) * D * D + (size_t)(i % D) * D + c0s);
  }
  // wide form: this CTA updates state rows [r_lo, r_hi) of the group's G * D
  // rows (row r = key dim r % D of head r / D; the G heads of a group are
  // contiguous, so the slab is one contiguous block); at most two heads,
  // since the host keeps rps <= D
  constexpr int SQ = D / 4;                // float4 per state row
  constexpr int WIT = 2;                   // float4 of the slab per thread and pass
  const int rps = (G * D + NSL - 1) / NSL;
  const int r_lo = min(G * D, slice * rps), r_hi = min(G * D, r_lo + rps);
  const int nf = WIDE ? (r_hi - r_lo) * SQ : 0;
  float *Sg = p.state + ((size_t)b * p.Hq + g * G) * D * D;
  float4 svw[WIT];
  if constexpr (WIDE) {
#pragma unroll
    for (int it = 0; it < WIT; ++it) {
      const int f = tid + it * kDecThreads;
      if (f < nf) svw[it] = *reinterpret_cast<const float4 *>(Sg + (size_t)r_lo * D + (size_t)f * 4);
    }
    for (int f = tid * 8 + WIT * kDecThreads; f < nf; f += kDecThreads * 8)   // later passes: into L2
      prefetch_l2(Sg + (size_t)r_lo * D + (size_t)f * 4);
  }
  if (t < 0 || t >= p.L_max) {  // same value in every CTA of the cluster: all leave together
    if (rank == 0 && tid == 0) set_err(p.err_word, LISA_DEVERR_POS);
    return;
  }
  // Other CTAs write into this CTA's shared memory only after the matching
  // wait (after the key stream): by then every CTA has initialised and armed
  // its mbarriers.
  cluster_arrive_relaxed();
  const int n = t + 1;
  const int kpc = (((n + NSL - 1) / NSL) + 31) & ~31;
  // this CTA's key slice (the wide form's last cluster later takes wider ranges)
  int k0 = min(n, slice * kpc);
  int k1 = min(n, k0 + kpc);
  int cnt = k1 - k0;
  // no key stream when every position is selected (n <= M): nothing is scored
  const int nsub = (window || n <= M) ? 0 : (cnt + SUB - 1) / SUB;

  // ---------------------------------------------------------------- TMA ring
  // the indexer keys are read once per step: first out of L2
  const uint64_t stream_pol = l2_evict_first_policy();
  auto issue = [&](int i) {  // thread 0 only: sub-chunk i -> stage i % NS; two ring lengths ahead -> L2
    const int s_lo = k0 + i * SUB;
    const int s_hi = min(k1, s_lo + SUB);
    const int ncopy = max(0, min(s_hi, t) - s_lo);   // row t comes from the argument
    for (int ahead = (i < NS ? 1 : 2); ahead <= 2; ++ahead) {   // sub-chunks i + NS and i + 2 NS
      const int p_lo = s_lo + ahead * NS * SUB;
      const int np = max(0, min(min(k1, p_lo + SUB), t) - p_lo);
      if (np > 0) bulk_prefetch_l2_hint(kidx_cache + (size_t)p_lo * DI, (uint32_t)(np * RB), stream_pol);
    }
    uint64_t *bar = &bars[i % NS];
    unsigned char *dst = ring + (i % NS) * STB;
    if (ncopy > 0) {
      if constexpr (SG::kMma) {
        mbar_arrive_expect_tx(bar, (uint32_t)(SUB * RB));   // the whole box lands, out-of-range rows zero
        tma_load_2d_hint(dst, &kmap, 0, bg * p.L_max + s_lo, bar, stream_pol);
      } else {
        mbar_arrive_expect_tx(bar, (uint32_t)(ncopy * RB));
        bulk_g2s_hint(dst, kidx_cache + (size_t)s_lo * DI, (uint32_t)(ncopy * RB), bar, stream_pol);
      }
    } else {
      mbar_arrive(bar);
    }
  };
  if (tid == 0)
    for (int i = 0; i < min(NS, nsub); ++i) issue(i);
  // the step's rows into shared memory; the CTA whose key slice holds row t
  // also appends the new token's k, v and indexer key to the caches
  {
    const bool app = p.fuse_append && t >= k0 && t < k1;
    const size_t arow = (size_t)bg * p.L_max + t;
    auto put = [&](int c, const uint4 &u) {
      Vec16<T>::unpack(u, chunk_dst(c));
      if (!app) return;
      if (c >= o_k && c < o_v)
        reinterpret_cast<uint4 *>(reinterpret_cast<T *>(p.k_cache) + arow * D)[c - o_k] = u;
      else if (c >= o_v && c < o_qi)
        reinterpret_cast<uint4 *>(reinterpret_cast<T *>(p.v_cache) + arow * D)[c - o_v] = u;
      else if (c >= o_ki && c < o_kl)
        reinterpret_cast<uint4 *>(reinterpret_cast<T *>(p.kidx_cache) + arow * DI)[c - o_ki] = u;
    };
#pragma unroll
    for (int j = 0; j < kInRegs; ++j)
      if (tid + j * kDecThreads < n_in) put(tid + j * kDecThreads, inr[j]);
    for (int c = tid + kInRegs * kDecThreads; c < n_in; c += kDecThreads) put(c, *chunk_src(c));
    if (!window && tid < R) qis[kMaxR * DI + tid] = w_in;
    if (tid < G) gls[tid] = gl_in;
  }
  __syncthreads();
  // MMA operand B (indexer queries, heads = columns, padded to 8; the floats
  // hold bf16 values, so re-packing is exact) and the head weights of this lane
  uint32_t bq[DI / 16][2];
  float wq0 = 0.f, wq1 = 0.f;
  if (SG::kMma && !window) {
    const int nh = lane >> 2, kc = 2 * (lane & 3);
    const float *qr = qis + (nh < R ? nh : 0) * DI;
#pragma unroll
    for (int s = 0; s < DI / 16; ++s) {
      bq[s][0] = nh < R ? pack_bf16(qr[s * 16 + kc], qr[s * 16 + kc + 1]) : 0u;
      bq[s][1] = nh < R ? pack_bf16(qr[s * 16 + kc + 8], qr[s * 16 + kc + 9]) : 0u;
    }
    if (kc < R) wq0 = qis[kMaxR * DI + kc];
    if (kc + 1 < R) wq1 = qis[kMaxR * DI + kc + 1];
  }

  // ---------------------------------------------------------------- linear state
  // S_h <- S_h + k^T v on columns [c0s, c0s + COLS); o_lin[h][c] = sum_i q_h[i] S_h[i][c].
  // Runs while the first key stages are in flight.
  if constexpr (WIDE) {
    // rows [r_lo, r_hi): S[r][:] += k[r % D] v, and the partial readout
    // o_lin[h][:] += q_h[r % D] S[r][:] of the (at most two) heads of the
    // slab, summed over the CTA into this CTA's slot of the workspace
    const int h_lo = r_lo / D;
    const int quad = tid % SQ;             // the same column quad for every float4 of this thread
    float vq[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) vq[j] = vs[quad * 4 + j];
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int f0 = 0; f0 < nf; f0 += WIT * kDecThreads) {
      float4 cur[WIT];
#pragma unroll
      for (int it = 0; it < WIT; ++it) {
        const int f = f0 + tid + it * kDecThreads;
        if (f < nf) cur[it] = f0 == 0 ? svw[it] : *reinterpret_cast<const float4 *>(Sg + (size_t)r_lo * D + (size_t)f * 4);
      }
#pragma unroll
      for (int it = 0; it < WIT; ++it) {
        const int f = f0 + tid + it * kDecThreads;
        if (f < nf) {
          const int r = r_lo + f / SQ, i = r % D, hh = r / D;
          const float ki = ks[i], qi = qs[hh * D + i];
          float4 sn = cur[it];
          sn.x = fmaf(ki, vq[0], sn.x);
          sn.y = fmaf(ki, vq[1], sn.y);
          sn.z = fmaf(ki, vq[2], sn.z);
          sn.w = fmaf(ki, vq[3], sn.w);
          *reinterpret_cast<float4 *>(Sg + (size_t)r * D + quad * 4) = sn;
          // the slab's first head, or the second (compile-time indices only)
          const float q0 = hh == h_lo ? qi : 0.f, q1 = hh == h_lo ? 0.f : qi;
          acc[0][0] = fmaf(q0, sn.x, acc[0][0]);
          acc[0][1] = fmaf(q0, sn.y, acc[0][1]);
          acc[0][2] = fmaf(q0, sn.z, acc[0][2]);
          acc[0][3] = fmaf(q0, sn.w, acc[0][3]);
          acc[1][0] = fmaf(q1, sn.x, acc[1][0]);
          acc[1][1] = fmaf(q1, sn.y, acc[1][1]);
          acc[1][2] = fmaf(q1, sn.z, acc[1][2]);
          acc[1][3] = fmaf(q1, sn.w, acc[1][3]);
        }
      }
    }
#pragma unroll
    for (int o = SQ; o < 32; o <<= 1)        // lanes of a warp with the same quad
#pragma unroll
      for (int sl = 0; sl < 2; ++sl)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[sl][j] += __shfl_xor_sync(0xffffffffu, acc[sl][j], o);
    float *wred = reinterpret_cast<float *>(smem + lay.wred);   // [2][8 warps][D]
    if (lane < SQ)
#pragma unroll
      for (int sl = 0; sl < 2; ++sl)
#pragma unroll
        for (int j = 0; j < 4; ++j) wred[(sl * 8 + warp) * D + quad * 4 + j] = acc[sl][j];
    __syncthreads();
    float *part = p.wpart + ((size_t)bg * NSL + slice) * 2 * D;
    for (int c = tid; c < 2 * D; c += kDecThreads) {
      float o = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) o += wred[((c / D) * 8 + w8) * D + c % D];
      part[c] = o;
    }
  } else {
    float vj[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) vj[j] = vs[c0s + cq * 4 + j];
    float *red = logit;                  // scratch [HP heads][8 warps][COLS]
    for (int h0 = 0; h0 < G; h0 += HP) {
      const int hn = min(HP, G - h0);
      if (h0 > 0) {                      // heads beyond the first HP are loaded now
#pragma unroll
        for (int hh = 0; hh < HP; ++hh) {
          if (hh >= hn) continue;
          const float *S = p.state + ((size_t)b * p.Hq + g * G + h0 + hh) * D * D;
#pragma unroll
          for (int it = 0; it < ITER; ++it) {
            const int idx = tid + it * kDecThreads;
            if (idx < D * QPR)
              sv[hh][it] = *reinterpret_cast<const float4 *>(S + (size_t)(idx / QPR) * D + c0s + cq * 4);
          }
        }
      }
      __syncthreads();                   // red is free
#pragma unroll
      for (int hh = 0; hh < HP; ++hh) {
        if (hh >= hn) continue;
        float *S = p.state + ((size_t)b * p.Hq + g * G + h0 + hh) * D * D;
        const float *qh = qs + (h0 + hh) * D;
        const float *kh = ks;            // the attention's k, or the head's own (variant)
        float vh[4] = {vj[0], vj[1], vj[2], vj[3]};
        if (lin_kv) {
          kh = klin + (h0 + hh) * D;
#pragma unroll
          for (int j = 0; j < 4; ++j) vh[j] = vlin[(h0 + hh) * D + c0s + cq * 4 + j];
        }
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int it = 0; it < ITER; ++it) {
          const int idx = tid + it * kDecThreads;
          if (idx < D * QPR) {
            const int i = idx / QPR;
            const float ki = kh[i], qi = qh[i];
            float4 sn = sv[hh][it];
            sn.x = fmaf(ki, vh[0], sn.x);
            sn.y = fmaf(ki, vh[1], sn.y);
            sn.z = fmaf(ki, vh[2], sn.z);
            sn.w = fmaf(ki, vh[3], sn.w);
            *reinterpret_cast<float4 *>(S + (size_t)i * D + c0s + cq * 4) = sn;
            a0 = fmaf(qi, sn.x, a0);
            a1 = fmaf(qi, sn.y, a1);
            a2 = fmaf(qi, sn.z, a2);
            a3 = fmaf(qi, sn.w, a3);
          }
        }
#pragma unroll
        for (int o = QPR; o < 32; o <<= 1) {
          a0 += __shfl_xor_sync(0xffffffffu, a0, o);
          a1 += __shfl_xor_sync(0xffffffffu, a1, o);
          a2 += __shfl_xor_sync(0xffffffffu, a2, o);
          a3 += __shfl_xor_sync(0xffffffffu, a3, o);
        }
        if (lane < QPR) {
          float *rw = red + (hh * 8 + warp) * COLS + lane * 4;
          rw[0] = a0;
          rw[1] = a1;
          rw[2] = a2;
          rw[3] = a3;
        }
      }
      __syncthreads();
      for (int i = tid; i < hn * COLS; i += kDecThreads) {
        const int hh = i / COLS, c = i % COLS;
        float o = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) o += red[(hh * 8 + w8) * COLS + c];
        olin[(h0 + hh) * COLS + c] = o;
      }
    }
  }

  // ---------------------------------------------------------------- indexer scores
  // Smallest and largest order key this thread writes (for the top-M's range
  // histogram).  The cache row of position t may be stale (its key is
  // replaced below from the argument row), so it is left out, and the new
  // key goes in when it is written.
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  auto note_key = [&](uint32_t u) {
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  };
  for (int i = 0; i < nsub; ++i) {
    const int stage = i % NS;
    if (!mbar_wait_bounded(&bars[stage], (uint32_t)((i / NS) & 1)) && tid == 0)
      set_err(p.err_word, LISA_DEVERR_TIMEOUT);
    const int s_lo = k0 + i * SUB;
    const int nk = min(k1, s_lo + SUB) - s_lo;
    const unsigned char *st = ring + stage * STB;
    if constexpr (SG::kMma) {
      // tiles of 16 keys; A = keys (row-major, swizzled by TMA), B = queries
      const uint32_t st_u32 = smem_u32(st);
      for (int tile = warp; tile * 16 < nk; tile += kDecThreads / 32) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        const int row = tile * 16 + (lane & 15);
        const int swz = RB == 128 ? (row & 7) : ((row >> 1) & 3);
#pragma unroll
        for (int s = 0; s < DI / 16; ++s) {
          const int chunk = 2 * s + (lane >> 4);
          uint32_t a[4];
          ldmatrix_x4(st_u32 + row * RB + ((chunk ^ swz) << 4), a[0], a[1], a[2], a[3]);
          mma_16816_bf16(d, a, bq[s]);
        }
        // columns 2*(lane&3), +1 are indexer heads; rows lane/4 and lane/4 + 8
        float p0 = fmaf(wq1, fmaxf(d[1], 0.f), wq0 * fmaxf(d[0], 0.f));
        float p1 = fmaf(wq1, fmaxf(d[3], 0.f), wq0 * fmaxf(d[2], 0.f));
        p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
        p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
        p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
        p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
        if ((lane & 3) == 0) {
          const int r0 = tile * 16 + (lane >> 2);
          if (r0 < nk) {
            const uint32_t u = score_key(p0);
            keys[s_lo - k0 + r0] = u;
            if (s_lo + r0 != t) note_key(u);
          }
          if (r0 + 8 < nk) {
            const uint32_t u = score_key(p1);
            keys[s_lo - k0 + r0 + 8] = u;
            if (s_lo + r0 + 8 != t) note_key(u);
          }
        }
      }
    } else {
      // one thread per key; chunk order rotated by the row so a wavefront
      // touches different bank groups
      const float *wsm = qis + kMaxR * DI;
      for (int kk = tid; kk < nk; kk += kDecThreads) {
        const unsigned char *row = st + kk * RB;
        float acc[kMaxR][2];
#pragma unroll
        for (int r = 0; r < kMaxR; ++r) acc[r][0] = acc[r][1] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < NCH; ++c0) {
          const int c = (c0 + kk) & (NCH - 1);
          float x[VEC];
          Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(row + c * 16), x);
#pragma unroll
          for (int r = 0; r < kMaxR; ++r) {
            if (r < R) {
              const float *qr = qis + r * DI + c * VEC;
#pragma unroll
              for (int j = 0; j < VEC; ++j) acc[r][j & 1] = fmaf(qr[j], x[j], acc[r][j & 1]);
            }
          }
        }
        float score = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxR; ++r)
          if (r < R) score = fmaf(wsm[r], fmaxf(acc[r][0] + acc[r][1], 0.f), score);
        const uint32_t u = score_key(score);
        keys[s_lo - k0 + kk] = u;
        if (s_lo + kk != t) note_key(u);
      }
    }
    __syncthreads();   // every thread is done with this stage
    if (tid == 0 && i + NS < nsub) issue(i + NS);
  }
  // the new token's score, from the argument row (its cache row may be stale)
  if (!window && n > M && t >= k0 && t < k1 && warp == 0) {
    const float *wsm = qis + kMaxR * DI;
    float score = 0.f;
    for (int r = 0; r < R; ++r) {
      float dot = 0.f;
      for (int c = lane; c < DI; c += 32) dot = fmaf(qis[r * DI + c], kis[c], dot);
      dot = warp_sum(dot);
      score = fmaf(wsm[r], fmaxf(dot, 0.f), score);
    }
    if (lane == 0) {
      const uint32_t u = score_key(score);
      keys[t - k0] = u;
      note_key(u);
    }
  }

  __syncthreads();

  // ---------------------------------------------------------------- top-M
  cluster_wait();                        // every CTA of the cluster runs and has armed its mbarriers
  // Wide form: every CTA of (b, g) arrives once, after publishing its slice in
  // the workspace.  The CTA that arrives last returns the counter to zero and
  // flags every CTA of its cluster; that cluster alone goes on (with every
  // slice visible to it), the others leave.  Only local shared memory is read
  // after the barrier, so a leaving CTA is never read by another.
  auto wide_arrive = [&]() -> bool {
    __threadfence();                     // this thread's workspace writes come before the arrival
    __syncthreads();
    if (tid == 0) {
      const unsigned old = atomicAdd(p.wcount + bg, 1u);
      if (old == (unsigned)NSL - 1u) {
        atomicExch(p.wcount + bg, 0u);
        __threadfence();
        for (int r = 0; r < NC; ++r) cluster.map_shared_rank(misc, r)[60] = 1u;
      }
    }
    cluster.sync();
    const bool last = misc[60] != 0u;
    if (last) __threadfence();
    return last;
  };
  int *sel0 = cluster.map_shared_rank(sel, 0);
  // Every CTA builds the whole index list in its own shared memory, except on
  // the cluster-wide radix path, which builds it in CTA 0 (local_list false).
  bool local_list = true;
  if (window) {
    if (ext) {                           // the caller's list of this (b, group)
      const int *src = p.sel_ext + ((size_t)b * p.sel_groups + (p.sel_groups == 1 ? 0 : g)) * M;
      for (int j = tid; j < M; j += kDecThreads) sel[j] = src[j];
    } else {                             // the M (= W) most recent positions t-M+1 .. t, or the whole prefix
      for (int j = tid; j < M; j += kDecThreads) sel[j] = n <= M ? (j < n ? j : -1) : t - M + 1 + j;
    }
  } else if (n > M) {
    if constexpr (WIDE) {
      // publish this slice's order keys and arrive; the last cluster's rank r
      // then takes the contiguous positions of NSL / NC slices
      {
        uint32_t *wk = p.wkeys + (size_t)bg * p.wkeys_stride + k0;
        for (int j = tid; j < cnt; j += kDecThreads) wk[j] = keys[j];
      }
      if (!wide_arrive()) return;
      const int spr = (NSL / NC) * kpc;
      k0 = min(n, rank * spr);
      k1 = min(n, k0 + spr);
      cnt = k1 - k0;
      const uint32_t *wk = p.wkeys + (size_t)bg * p.wkeys_stride + k0;
      for (int j = tid; j < cnt; j += kDecThreads) keys[j] = __ldcg(wk + j);
      __syncthreads();
    }
    constexpr int SEG = dec_seg(NC);                    // candidate slots each CTA sends
    constexpr int XW = dec_msg_words(NC);
    constexpr int SLOTS = NC * SEG / kDecThreads;       // candidate slots per thread
    static_assert(SLOTS * kDecThreads == NC * SEG && SLOTS <= 4, "slots");
    uint32_t *xin = reinterpret_cast<uint32_t *>(smem + lay.xin);   // [NC][XW]
    uint32_t *xo = xin + rank * XW;                     // this CTA's message, built in its own slot
    uint32_t *fh = hist + 1024;                         // bins of this CTA's keys
    uint32_t *sbin = hist;                              // bins of the exact select
    // kl: keys each CTA vouches for; covered: keys vouched for in all (at least
    // M when every CTA that holds keys holds kl of them)
    const int kw = WIDE ? (NSL / NC) * kpc : kpc;       // keys per CTA of the selecting cluster
    const int ns = (n + kw - 1) / kw;                   // CTAs that hold keys
    const int kl = (M + ns - 1) / ns;
    int covered = 0;
    for (int r = 0; r < NC; ++r) {
      const int cr = min(n, (r + 1) * kw) - min(n, r * kw);
      if (cr >= kl) covered += kl;
    }
    // (a) this CTA's keys into a 1024-bin range histogram over the 8 octaves
    //     below its largest key (order keys within 8 << 23 of it).  Its bound
    //     theta_r is the lower edge of the bin of its kl-th largest key (at
    //     least kl keys are >= theta_r); its send threshold is the lower edge
    //     of the bin above the one holding its SEG-th largest key (fewer than
    //     SEG keys are >= it), or 0 (every key) when it holds at most SEG.
    uint32_t vmin = kmin, vmax = kmax;                  // from the scoring pass
    if constexpr (WIDE) {                               // the reloaded keys of this CTA's range
      vmin = 0xFFFFFFFFu;
      vmax = 0u;
      for (int j = tid; j < cnt; j += kDecThreads) {
        const uint32_t u = keys[j];
        vmin = min(vmin, u);
        vmax = max(vmax, u);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 0) {
      tot[warp] = vmin;
      tot[8 + warp] = vmax;
    }
    for (int i = tid; i < 2048; i += kDecThreads) hist[i] = 0;   // fh and sbin
    __syncthreads();
#pragma unroll
    for (int w8 = 0; w8 < kDecThreads / 32; ++w8) {
      vmin = min(vmin, tot[w8]);
      vmax = max(vmax, tot[8 + w8]);
    }
    uint32_t theta = 0xFFFFFFFFu, tsend = 0u;          // theta: neutral for the minimum
    if (cnt > 0) {                                      // uniform in the CTA
      const uint32_t lo = (vmax - vmin) > (8u << 23) ? vmax - (8u << 23) : vmin;
      const uint32_t sh = (vmax - lo) < 1024u ? 0u : (uint32_t)(32 - __clz(vmax - lo)) - 10u;
      for (int j = tid; j < cnt; j += kDecThreads) {
        const uint32_t u = keys[j];
        if (u >= lo) atomicAdd(&fh[(u - lo) >> sh], 1u);
      }
      __syncthreads();
      find_bin1024_two<kDecThreads>(fh, (uint32_t)kl, (uint32_t)SEG, misc);
      if (cnt >= kl) theta = misc[0] <= 1023u ? lo + (misc[0] << sh) : vmin;   // fewer than kl keys >= lo: all
      if (cnt > SEG) {
        if (misc[4] <= 1023u) {
          const uint64_t e = (uint64_t)lo + ((uint64_t)(misc[4] + 1u) << sh);
          tsend = e > 0xFFFFFFFFull ? 0xFFFFFFFFu : (uint32_t)e;
        } else {
          tsend = lo;                                   // fewer than SEG keys >= lo
        }
      }
    } else {
      vmax = 0u;
    }
    auto prefetch_kv = [&](int pos) {
      const size_t row = ((size_t)bg * p.L_max + pos) * D;
      const char *kr = reinterpret_cast<const char *>(reinterpret_cast<const T *>(p.k_cache) + row);
      const char *vr = reinterpret_cast<const char *>(reinterpret_cast<const T *>(p.v_cache) + row);
#pragma unroll
      for (int c = 0; c < ROWB; c += 128) {
        prefetch_l2(kr + c);
        prefetch_l2(vr + c);
      }
    };
    // (b) keys >= tsend, in position order, into this CTA's message; warp w
    //     owns a contiguous run of keys
    {
      const int cw = (((cnt + 7) / 8) + 31) & ~31;
      const int j0 = min(cnt, warp * cw), j1 = min(cnt, j0 + cw);
      uint32_t wc = 0;
      for (int base = j0; base < j1; base += 32) {
        const int j = base + lane;
        wc += __popc(__ballot_sync(0xffffffffu, j < j1 && keys[j] >= tsend));
      }
      if (lane == 0) misc[24 + warp] = wc;
      __syncthreads();
      uint32_t off = 0, total = 0;
#pragma unroll
      for (int w8 = 0; w8 < kDecThreads / 32; ++w8) {
        const uint32_t c = misc[24 + w8];
        off += w8 < warp ? c : 0u;
        total += c;
      }
      if (total <= (uint32_t)SEG) {
        const unsigned lt = (1u << lane) - 1u;
        for (int base = j0; base < j1; base += 32) {
          const int j = base + lane;
          const bool act = j < j1 && keys[j] >= tsend;
          const unsigned am = __ballot_sync(0xffffffffu, act);
          if (act) {
            const uint32_t o = off + __popc(am & lt);
            xo[4 + o] = keys[j];
            xo[4 + SEG + o] = (uint32_t)(k0 + j);
          }
          off += __popc(am);
        }
      }
      if (tid == 0) {
        xo[0] = theta;
        xo[1] = vmax;
        xo[2] = tsend;
        xo[3] = total <= (uint32_t)SEG ? total : 0x80000000u;   // the top bit: too many to send
      }
    }
    __syncthreads();                                    // the message is complete
    // (c) the message to every other CTA of the cluster (its slot `rank`,
    //     counted on its candidate mbarrier), then the K and V rows of this
    //     CTA's likely selected keys (>= theta, all in its message when the
    //     exchange holds) into L2 while the others' messages arrive
    {
      constexpr int CH = XW / 4;                        // 16-byte chunks
      const uint32_t src = smem_u32(xo), xbar = smem_u32(mbx);
      for (int i = tid; i < (NC - 1) * CH; i += kDecThreads) {
        const int dd = i / CH, q = i % CH;
        const uint32_t d = (uint32_t)(dd < rank ? dd : dd + 1);
        st_async_v4(mapa_u32(src + 16u * q, d), *reinterpret_cast<const uint4 *>(xo + 4 * q), mapa_u32(xbar, d));
      }
    }
    if (!(xo[3] & 0x80000000u))
      for (int j = tid; j < (int)xo[3]; j += kDecThreads) {
        const int pos = (int)xo[4 + SEG + j];
        if (xo[4 + j] >= theta && pos != t) prefetch_kv(pos);
      }
    if (!mbar_wait_cluster_bounded(mbx, 0u)) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
    // (d) the bound lb = min_r theta_r (when the CTAs vouch for M keys
    //     together; else 0) and the largest key, from the headers.  The
    //     messages hold every key >= lb iff no CTA overflowed and every send
    //     threshold is <= lb; the same answer in every thread of every CTA.
    uint32_t th_r = 0xFFFFFFFFu, mx_r = 0u, ts_r = 0u, ct_r = 0u;
    if (lane < NC) {
      const uint4 h = *reinterpret_cast<const uint4 *>(xin + lane * XW);
      th_r = h.x;
      mx_r = h.y;
      ts_r = h.z;
      ct_r = h.w;
    }
    uint32_t lbv = th_r, hiv = mx_r;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lbv = min(lbv, __shfl_xor_sync(0xffffffffu, lbv, o));
      hiv = max(hiv, __shfl_xor_sync(0xffffffffu, hiv, o));
    }
    const uint32_t lb = covered >= M ? lbv : 0u;
    const bool exch_ok = __all_sync(0xffffffffu, (ct_r & 0x80000000u) == 0u && ts_r <= lb);
    local_list = exch_ok;
    if (exch_ok) {
      // the rest of this CTA's candidates (lb <= key < theta) into L2 as well:
      // they are all in its own message (every threshold is <= lb)
      for (int j = tid; j < (int)xo[3]; j += kDecThreads) {
        const uint32_t u = xo[4 + j];
        const int pos = (int)xo[4 + SEG + j];
        if (u >= lb && u < theta && pos != t) prefetch_kv(pos);
      }
      // (e) the candidates, in position order: slot s = (warp * SLOTS + i) *
      //     32 + lane is entry s % SEG of message s / SEG; valid when that
      //     entry was sent and its key is >= lb
      uint32_t cku[SLOTS];
      int cpp[SLOTS];
      bool cv[SLOTS];
#pragma unroll
      for (int i = 0; i < SLOTS; ++i) {
        const int s = (warp * SLOTS + i) * 32 + lane;
        const uint32_t *m = xin + (s / SEG) * XW;
        const int j = s % SEG;
        cv[i] = j < (int)m[3];
        cku[i] = cv[i] ? m[4 + j] : 0u;
        cpp[i] = cv[i] ? (int)m[4 + SEG + j] : -1;
        cv[i] = cv[i] && cku[i] >= lb;
      }
      // (f) the exact M-th key K*: 1024-bin range histograms over [lb, largest],
      //     narrowed until the bin holding it is one value or holds at most 32
      //     keys (ranked in warp 0); need_eq = keys equal to K* the top M takes
      uint32_t kstar = 0u, need_eq = 0u;
      bool rok = false;
      {
        uint32_t lbx = lb, ubx = hiv, rem = (uint32_t)M;
        uint32_t shx = (ubx - lbx) < 1024u ? 0u : (uint32_t)(32 - __clz(ubx - lbx)) - 10u;
        uint32_t *mem = tot + 128;                      // the keys of one bin, at most 32
#pragma unroll 1
        for (int iter = 0; iter < 4; ++iter) {
          if (iter > 0) {
            for (int i = tid; i < 1024; i += kDecThreads) sbin[i] = 0;
            __syncthreads();
          }
#pragma unroll
          for (int i = 0; i < SLOTS; ++i)
            if (cv[i] && cku[i] >= lbx && cku[i] <= ubx) atomicAdd(&sbin[(cku[i] - lbx) >> shx], 1u);
          __syncthreads();
          find_bin1024<kDecThreads>(sbin, rem, misc);
          const uint32_t bin = misc[0];
          if (bin > 1023u) break;                       // inconsistent counts (uniform)
          rem -= misc[1];
          const uint32_t cb = misc[2];
          const uint32_t blo = lbx + (bin << shx);
          if (shx == 0u) {
            kstar = blo;
            need_eq = rem;
            rok = true;
            break;
          }
          if (cb <= 32u) {
            if (tid == 0) misc[7] = 0xFFFFFFFFu;
#pragma unroll
            for (int i = 0; i < SLOTS; ++i) {
              if (cv[i] && cku[i] >= lbx && cku[i] <= ubx && ((cku[i] - lbx) >> shx) == bin) {
                const uint32_t s = atomicAdd(&misc[3], 1u);
                if (s < 32u) mem[s] = cku[i];
              }
            }
            __syncthreads();
            if (warp == 0) {
              const uint32_t x = lane < (int)cb ? mem[lane] : 0u;
              uint32_t gt = 0, ge = 0;
              for (int j = 0; j < (int)cb; ++j) {
                const uint32_t y = __shfl_sync(0xffffffffu, x, j);
                gt += y > x ? 1u : 0u;
                ge += y >= x ? 1u : 0u;
              }
              if (lane < (int)cb && gt < rem && rem <= ge) {
                misc[5] = x;
                misc[7] = rem - gt;
              }
            }
            __syncthreads();
            kstar = misc[5];
            need_eq = misc[7];
            rok = need_eq != 0xFFFFFFFFu;
            break;
          }
          const uint64_t top = (uint64_t)blo + ((1ull << shx) - 1ull);
          lbx = blo;
          ubx = top > (uint64_t)ubx ? ubx : (uint32_t)top;
          shx = shx > 10u ? shx - 10u : 0u;
        }
      }
      if (!rok) {
        if (tid == 0) set_err(p.err_word, LISA_DEVERR_CHECK);
        for (int j = tid; j < M; j += kDecThreads) sel[j] = -1;
      } else {
        // (g) the ascending index list: every key > K*, and the first need_eq
        //     keys equal to K* in position order; each warp's slots by
        //     ballots, the warps' offsets from their totals
        unsigned bgt[SLOTS], beq[SLOTS];
        uint32_t ngt = 0, neq = 0;
#pragma unroll
        for (int i = 0; i < SLOTS; ++i) {
          bgt[i] = __ballot_sync(0xffffffffu, cv[i] && cku[i] > kstar);
          beq[i] = __ballot_sync(0xffffffffu, cv[i] && cku[i] == kstar);
          ngt += __popc(bgt[i]);
          neq += __popc(beq[i]);
        }
        if (lane == 0) {
          misc[16 + warp] = ngt;
          misc[24 + warp] = neq;
        }
        __syncthreads();
        uint32_t gb = 0, eb = 0, gtot = 0, etot = 0;
#pragma unroll
        for (int w8 = 0; w8 < kDecThreads / 32; ++w8) {
          const uint32_t a = misc[16 + w8], c = misc[24 + w8];
          gb += w8 < warp ? a : 0u;
          eb += w8 < warp ? c : 0u;
          gtot += a;
          etot += c;
        }
        bool bad = gtot + need_eq != (uint32_t)M || etot < need_eq;
        const unsigned lt = (1u << lane) - 1u;
#pragma unroll
        for (int i = 0; i < SLOTS; ++i) {
          const bool gt = (bgt[i] >> lane) & 1u, eq = (beq[i] >> lane) & 1u;
          const uint32_t pe = eb + __popc(beq[i] & lt);
          if (gt || (eq && pe < need_eq)) {
            const uint32_t o = gb + __popc(bgt[i] & lt) + min(pe, need_eq);
            if (o < (uint32_t)M && cpp[i] >= 0 && cpp[i] < n) sel[o] = cpp[i];
            else bad = true;
          }
          gb += __popc(bgt[i]);
          eb += __popc(beq[i]);
        }
        if (bad) set_err(p.err_word, LISA_DEVERR_CHECK);
      }
    } else {
      // (h) the messages miss keys >= lb (a CTA had too many to send, or
      //     sent too few): cluster-wide radix select over all keys
      uint32_t prefix = 0, pmask = 0, rem = (uint32_t)M;
      bool ok = true;
      const int iters = (cnt + kDecThreads - 1) / kDecThreads;
#pragma unroll 1
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        // Written here, read by every CTA after the cluster barrier below, and
        // rewritten two passes later, after another cluster barrier.
        uint32_t *H = hist + (pass & 1) * 256;
        __syncthreads();
        H[tid] = 0;                            // 256 threads, 256 bins
        __syncthreads();
        for (int it = 0; it < iters; ++it) {
          const int j = tid + it * kDecThreads;
          uint32_t u = 0;
          bool act = false;
          if (j < cnt) {
            u = keys[j];
            act = (u & pmask) == prefix;
          }
          const uint32_t dig = (u >> shift) & 255u;
          const unsigned am = __ballot_sync(0xffffffffu, act);
          if (act) {
            const unsigned peers = __match_any_sync(am, dig);
            if (lane == __ffs(peers) - 1) atomicAdd(&H[dig], (uint32_t)__popc(peers));
          }
        }
        cluster.sync();                        // every CTA's histogram of this pass is complete
        {
          uint32_t s = 0;
#pragma unroll
          for (int r = 0; r < NC; ++r) s += cluster.map_shared_rank(H, r)[tid];
          tot[tid] = s;
        }
        if (tid == 0) misc[0] = 0xFFFFFFFFu;
        __syncthreads();
        dec_find_bucket(tot, misc, rem);
        __syncthreads();
        const uint32_t dig = misc[0];
        const uint32_t above = misc[1];
        if (dig > 255u) {                      // inconsistent counts: cannot happen for valid keys
          ok = false;
          continue;                            // keep every cluster barrier matched
        }
        rem -= above;
        prefix |= dig << shift;
        pmask |= 255u << shift;
      }
      if (!ok) {
        if (tid == 0) set_err(p.err_word, LISA_DEVERR_CHECK);
        prefix = 0xFFFFFFFFu;                  // nothing is above; emits no more than need_eq = 0
        rem = 0;
      }
      const uint32_t kstar = prefix, need_eq = rem;

      // counts of keys above / equal to K* in this CTA's slice, then cluster prefix
      const int per_warp = (((cnt + 7) / 8) + 31) & ~31;
      const int c0w = warp * per_warp;
      const int c1w = min(cnt, c0w + per_warp);
      uint32_t gw = 0, ew = 0;
      for (int base = c0w; base < c1w; base += 32) {
        const int j = base + lane;
        const uint32_t u = j < c1w ? keys[j] : 0u;
        gw += __popc(__ballot_sync(0xffffffffu, j < c1w && u > kstar));
        ew += __popc(__ballot_sync(0xffffffffu, j < c1w && u == kstar));
      }
      __syncthreads();
      if (lane == 0) {
        misc[8 + warp] = gw;
        misc[16 + warp] = ew;
      }
      __syncthreads();
      if (tid == 0) {
        uint32_t sg = 0, se = 0;
        for (int w8 = 0; w8 < 8; ++w8) {
          const uint32_t a = misc[8 + w8], c = misc[16 + w8];
          misc[8 + w8] = sg;       // exclusive prefix within the CTA
          misc[16 + w8] = se;
          sg += a;
          se += c;
        }
        misc[2] = sg;              // CTA totals, read by the other CTAs
        misc[3] = se;
      }
      cluster.sync();
      uint32_t gb = 0, eb = 0;
      for (int r = 0; r < rank; ++r) {
        const uint32_t *mr = cluster.map_shared_rank(misc, r);
        gb += mr[2];
        eb += mr[3];
      }
      uint32_t gcur = gb + misc[8 + warp], ecur = eb + misc[16 + warp];
      const unsigned lt = (1u << lane) - 1u;
      for (int base = c0w; base < c1w; base += 32) {
        const int j = base + lane;
        const uint32_t u = j < c1w ? keys[j] : 0u;
        const unsigned bgt = __ballot_sync(0xffffffffu, j < c1w && u > kstar);
        const unsigned beq = __ballot_sync(0xffffffffu, j < c1w && u == kstar);
        const uint32_t pe = ecur + __popc(beq & lt);
        const bool gt = (bgt >> lane) & 1u, eq = (beq >> lane) & 1u;
        if (gt || (eq && pe < need_eq)) {
          const uint32_t o = gcur + __popc(bgt & lt) + min(pe, need_eq);
          if (o < (uint32_t)M) sel0[o] = k0 + j;
          else set_err(p.err_word, LISA_DEVERR_CHECK);
        }
        gcur += __popc(bgt);
        ecur += __popc(beq);
      }
      if (!ok && rank == 0)
        for (int j = tid; j < M; j += kDecThreads) sel[j] = -1;
    }
  } else {
    if constexpr (WIDE) {
      if (!wide_arrive()) return;
    }
    for (int j = tid; j < M; j += kDecThreads) sel[j] = j < n ? j : -1;
  }
  // the ascending index list: this CTA's own copy, or CTA 0's after the
  // cluster-wide radix path (the same answer in every CTA)
  const int *selp = sel;
  if (local_list) {
    __syncthreads();
  } else {
    cluster.sync();                          // CTA 0 holds the full ascending index list
    selp = sel0;
  }
  if constexpr (WIDE) {
    // o_lin of this CTA's output columns: the partial readouts of the CTAs
    // whose state rows belong to each head, in a fixed order
    for (int i = tid; i < G * COLS; i += kDecThreads) {
      const int hh = i / COLS, c = i % COLS;
      const int w_a = (hh * D) / rps, w_b = min(NSL - 1, ((hh + 1) * D - 1) / rps);
      float o = 0.f;
      for (int w = w_a; w <= w_b; ++w)
        o += __ldcg(p.wpart + (((size_t)bg * NSL + w) * 2 + (hh - (w * rps) / D)) * D + c0s + c);
      olin[i] = o;
    }
  }
  if (rank == 0 && p.idx_out)
    for (int j = tid; j < M; j += kDecThreads) p.idx_out[(size_t)bg * M + j] = selp[j];

  // The next kernel on the stream may be scheduled from here on: its CTAs
  // wait in their prologue, so a later trigger keeps them from holding SM
  // slots through this kernel's key stream and selection.  (An independent
  // step has let it start already.)
  if (!p.independent) grid_dep_launch();
  // ---------------------------------------------------------------- sparse attention (this CTA's rows)
  unsigned char *kvs = ring;                 // [rpc] K rows then [rpc] V rows, stride RS
  for (int r = tid; r < rpc; r += kDecThreads) {
    int s = selp[rank * rpc + r];
    if (s < -1 || s > t) {
      set_err(p.err_word, LISA_DEVERR_CHECK);
      s = -1;
    }
    sidx[r] = s;
  }
  __syncthreads();
  {
    // every 16-byte piece in flight at once (asynchronous copies; rows of
    // unselected slots are zero-filled)
    const T *kc = reinterpret_cast<const T *>(p.k_cache) + (size_t)bg * p.L_max * D;
    const T *vc = reinterpret_cast<const T *>(p.v_cache) + (size_t)bg * p.L_max * D;
    const uint32_t kvs_base = smem_u32(kvs);
    for (int i = tid; i < rpc * SL; i += kDecThreads) {
      const int r = i / SL, sl = i % SL;
      const int s = sidx[r];
      const T *kr = (s == t) ? kin : kc + (size_t)(s < 0 ? 0 : s) * D;
      const T *vr = (s == t) ? vin : vc + (size_t)(s < 0 ? 0 : s) * D;
      cp_async16(kvs_base + r * RS + sl * 16, kr + sl * VEC, s >= 0);
      cp_async16(kvs_base + (rpc + r) * RS + sl * 16, vr + sl * VEC, s >= 0);
    }
    cp_async_commit();
    cp_async_wait_all();
  }
  __syncthreads();
  // bf16 with whole 16-row k-steps: both products on the tensor cores (warp
  // MMAs; query heads are the 16 rows of the A operand)
  const bool mma_attn = SG::kMma && (rpc % 16) == 0;
  if (mma_attn) {
    // logits[hh][r] = q_h . k_r / sqrt(d): A = q (heads x d), B = K rows (d x rows)
    const int g4 = lane >> 2, t2 = (lane & 3) * 2;
    const uint32_t kvs_u32 = smem_u32(kvs);
    for (int nt = warp; nt < rpc / 8; nt += kDecThreads / 32) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks2 = 0; ks2 < D / 32; ++ks2) {
        uint32_t bk[4];
        ldmatrix_x4(kvs_u32 + (nt * 8 + (lane & 7)) * RS + ks2 * 64 + (lane >> 3) * 16, bk[0], bk[1], bk[2], bk[3]);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int k0q = (2 * ks2 + h2) * 16 + t2;
          uint32_t a[4];
          a[0] = g4 < G ? pack_bf16(qs[g4 * D + k0q], qs[g4 * D + k0q + 1]) : 0u;
          a[1] = g4 + 8 < G ? pack_bf16(qs[(g4 + 8) * D + k0q], qs[(g4 + 8) * D + k0q + 1]) : 0u;
          a[2] = g4 < G ? pack_bf16(qs[g4 * D + k0q + 8], qs[g4 * D + k0q + 9]) : 0u;
          a[3] = g4 + 8 < G ? pack_bf16(qs[(g4 + 8) * D + k0q + 8], qs[(g4 + 8) * D + k0q + 9]) : 0u;
          mma_16816_bf16(c, a, bk + 2 * h2);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int hh = g4 + (j >> 1) * 8, r = nt * 8 + t2 + (j & 1);
        if (hh < G) logit[hh * rpc + r] = sidx[r] >= 0 ? c[j] * p.scale : -INFINITY;
      }
    }
  } else {
    // logits[hh][r] = q_h . k_r / sqrt(d)
    for (int i = tid; i < G * rpc; i += kDecThreads) {
      const int hh = i / rpc, r = i % rpc;
      float l = -INFINITY;
      if (sidx[r] >= 0) {
        const float *qh = qs + hh * D;
        const unsigned char *kr = kvs + r * RS;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
        for (int sl = 0; sl < SL; ++sl) {
          float x[VEC];
          Vec16<T>::unpack(*reinterpret_cast<const uint4 *>(kr + sl * 16), x);
#pragma unroll
          for (int j = 0; j < VEC; j += 2) {
            a0 = fmaf(qh[sl * VEC + j], x[j], a0);
            a1 = fmaf(qh[sl * VEC + j + 1], x[j + 1], a1);
          }
        }
        l = (a0 + a1) * p.scale;
      }
      logit[hh * rpc + r] = l;
    }
  }
  __syncthreads();
  // this CTA's partial output of head hh, column d: into the merge message
  // for the CTA that owns column d
  auto put_part = [&](int hh, int d, float v) { pout[(d / COLS) * MW + hh * COLS + d % COLS] = v; };
  // per head: local max and sum of exponentials over this CTA's rows
  for (int hh = warp; hh < G; hh += 8) {
    float m = -INFINITY;
    for (int r = lane; r < rpc; r += 32) m = fmaxf(m, logit[hh * rpc + r]);
    m = warp_max(m);
    float l = 0.f;
    for (int r = lane; r < rpc; r += 32) {
      const float x = logit[hh * rpc + r];
      const float e = (x == -INFINITY) ? 0.f : expf(x - m);
      logit[hh * rpc + r] = e;
      l += e;
    }
    l = warp_sum(l);
    // (max, sum) of this head go to every owner's merge message
    for (int o = lane; o < NC; o += 32) {
      pout[o * MW + G * COLS + 2 * hh] = m;
      pout[o * MW + G * COLS + 2 * hh + 1] = l;
    }
  }
  __syncthreads();
  if (mma_attn) {
    // o_part[hh][d] = sum_r e[hh][r] v_r[d]: A = e (heads x rows) as bf16 hi + lo
    // pairs, B = V rows (rows x d) through transposing matrix loads
    const int g4 = lane >> 2, t2 = (lane & 3) * 2;
    const uint32_t v_u32 = smem_u32(kvs + rpc * RS);
    for (int np = warp; np < D / 16; np += kDecThreads / 32) {     // pairs of 8-column tiles
      float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
      for (int ks = 0; ks < rpc / 16; ++ks) {
        uint32_t bv[4];
        const int m = lane >> 3;
        ldmatrix_x4_trans(v_u32 + (ks * 16 + (m & 1) * 8 + (lane & 7)) * RS + (np * 16 + (m >> 1) * 8) * 2, bv[0],
                          bv[1], bv[2], bv[3]);
        float e[8];
        const int r0 = ks * 16 + t2;
        e[0] = g4 < G ? logit[g4 * rpc + r0] : 0.f;
        e[1] = g4 < G ? logit[g4 * rpc + r0 + 1] : 0.f;
        e[2] = g4 + 8 < G ? logit[(g4 + 8) * rpc + r0] : 0.f;
        e[3] = g4 + 8 < G ? logit[(g4 + 8) * rpc + r0 + 1] : 0.f;
        e[4] = g4 < G ? logit[g4 * rpc + r0 + 8] : 0.f;
        e[5] = g4 < G ? logit[g4 * rpc + r0 + 9] : 0.f;
        e[6] = g4 + 8 < G ? logit[(g4 + 8) * rpc + r0 + 8] : 0.f;
        e[7] = g4 + 8 < G ? logit[(g4 + 8) * rpc + r0 + 9] : 0.f;
        uint32_t ahi[4], alo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          ahi[j] = pack_bf16(e[2 * j], e[2 * j + 1]);
          const float h0 = __bfloat162float(__float2bfloat16_rn(e[2 * j]));
          const float h1 = __bfloat162float(__float2bfloat16_rn(e[2 * j + 1]));
          alo[j] = pack_bf16(e[2 * j] - h0, e[2 * j + 1] - h1);
        }
        mma_16816_bf16(c0, ahi, bv);
        mma_16816_bf16(c0, alo, bv);
        mma_16816_bf16(c1, ahi, bv + 2);
        mma_16816_bf16(c1, alo, bv + 2);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int hh = g4 + (j >> 1) * 8, d = np * 16 + t2 + (j & 1);
        if (hh < G) {
          put_part(hh, d, c0[j]);
          put_part(hh, d + 8, c1[j]);
        }
      }
    }
  } else {
    // o_part[hh][d] = sum_r e[hh][r] v_r[d]
    for (int i = tid; i < G * D; i += kDecThreads) {
      const int hh = i / D, d = i % D;
      const float *e = logit + hh * rpc;
      const T *vcol = reinterpret_cast<const T *>(kvs + rpc * RS) + d;
      float a = 0.f;
      for (int r = 0; r < rpc; ++r) a = fmaf(e[r], Dt<T>::to_f(vcol[(size_t)r * (RS / sizeof(T))]), a);
      put_part(hh, d, a);
    }
  }
  // ---------------------------------------------------------------- merge + gate, columns of this CTA
  // Each CTA sends, to every other CTA r, its partial outputs of r's columns
  // [r*D/NC, (r+1)*D/NC) and its (max, sum) per head (counted on r's merge
  // mbarrier), then merges the NC partials of its own columns once the others'
  // have arrived.
  __syncthreads();                             // the merge messages are complete
  {
    const int CH = MW / 4;                     // 16-byte chunks per message
    const uint32_t dst0 = smem_u32(pin + rank * MW), mbar = smem_u32(mbm);
    for (int i = tid; i < (NC - 1) * CH; i += kDecThreads) {
      const int dd = i / CH, q = i % CH;
      const uint32_t d = (uint32_t)(dd < rank ? dd : dd + 1);
      st_async_v4(mapa_u32(dst0 + 16u * q, d), *reinterpret_cast<const uint4 *>(pout + d * MW + 4 * q),
                  mapa_u32(mbar, d));
    }
  }
  // The matching wait ends the kernel: no CTA leaves while another may still
  // be sending to it.
  cluster_arrive_relaxed();
  if (!mbar_wait_cluster_bounded(mbm, 0u)) set_err(p.err_word, LISA_DEVERR_TIMEOUT);
  for (int i = tid; i < G * COLS; i += kDecThreads) {
    const int hh = i / COLS, c = i % COLS, d = c0s + c;
    auto msg = [&](int r) -> const float * { return r == rank ? pout + rank * MW : pin + r * MW; };
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < NC; ++r) mx = fmaxf(mx, msg(r)[G * COLS + 2 * hh]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int r = 0; r < NC; ++r) {
      const float *mr = msg(r);
      const float m_r = mr[G * COLS + 2 * hh];
      if (m_r == -INFINITY) continue;
      const float f = expf(m_r - mx);
      num = fmaf(f, mr[hh * COLS + c], num);
      den = fmaf(f, mr[G * COLS + 2 * hh + 1], den);
    }
    const int h = g * G + hh;
    const float o_sp = num / den;
    const float o_lin = olin[hh * COLS + c];
    const float gam = 1.f / (1.f + expf(-gls[hh]));
    reinterpret_cast<T *>(p.out)[((size_t)b * p.Hq + h) * D + d] = Dt<T>::from_f(gam * o_sp + (1.f - gam) * o_lin);
  }
  cluster_wait();
}

// ============================================================ launcher
template <typename T, int D, int DI, int NC, bool WIDE = false>
static cudaError_t launch_cluster_t(const DecodeParams &p, const CUtensorMap &kmap, cudaStream_t st) {
  auto kern = decode_cluster_kernel<T, D, DI, NC, WIDE>;
  const DecLayout lay = dec_layout(p.kpc_max, p.L_max, p.M, p.G, D, DI, (int)sizeof(T), NC, p.stages,
                                   p.stage_keys * ScoreGeom<T, DI>::RB, p.k_lin != nullptr, WIDE);
  cudaError_t e = prepare_kernel(kern, lay.total);
  if (e != cudaSuccess) return e;
  if (NC > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = NC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.B * p.Hkv * (WIDE ? p.nw : NC));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = lay.total;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, p, kmap);
}

// 16 when a 16-CTA cluster of this kernel can be scheduled on this device, else 8.
template <typename T, int D, int DI>
static int pick_cluster(const DecodeParams &p) {
  auto kern = decode_cluster_kernel<T, D, DI, 16>;
  const int kpc = (((p.L_max + 15) / 16) + 31) & ~31;
  const DecLayout lay = dec_layout(kpc, p.L_max, p.M, p.G, D, DI, (int)sizeof(T), 16, kStages, kStageBytes,
                                   p.k_lin != nullptr);
  if (prepare_kernel(kern, lay.total) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 8;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 16;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(16);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = lay.total;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 8;
  }
  return nclusters > 0 ? 16 : 8;
}

template <typename T, int D, int DI>
static cudaError_t launch_decode_t(DecodeParams p, cudaStream_t st) {
  // whether 16-CTA clusters can be scheduled depends on the device and the
  // shared-memory footprint: cache per (device, footprint)
  static int cache_dev[8] = {-1, -1, -1, -1, -1, -1, -1, -1};
  static int cache_key[8], cache_ok16[8], cache_sms[8];
  static int next = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  const int key = p.L_max * 2 + (p.k_lin ? 1 : 0) + (p.M << 20) + (p.G << 28);
  int ok16 = -1, sms = 0;
  for (int i = 0; i < 8; ++i)
    if (cache_dev[i] == dev && cache_key[i] == key) {
      ok16 = cache_ok16[i];
      sms = cache_sms[i];
    }
  if (ok16 < 0) {
    ok16 = pick_cluster<T, D, DI>(p) == 16 ? 1 : 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      sms = 148;
    }
    const int slot = next++ & 7;
    cache_dev[slot] = dev;
    cache_key[slot] = key;
    cache_ok16[slot] = ok16;
    cache_sms[slot] = sms;
  }
  if (p.nw > 0) {
    // the wide form: nw CTAs (clusters of 8, 2 ring stages) per (b, g); the
    // last cluster's ranks each take nw / 8 key slices
    if constexpr (sizeof(T) == 2) {
      p.nc = 8;
      p.stages = 2;
      p.stage_keys = ScoreGeom<T, DI>::sub(32768);
      p.kpc_max = (p.nw / 8) * ((((p.L_max + p.nw - 1) / p.nw) + 31) & ~31);
      CUtensorMap kmap;
      memset(&kmap, 0, sizeof(kmap));
      using SG = ScoreGeom<T, DI>;
      if (!make_tmap_2d(&kmap, p.kidx_cache, (int)sizeof(T), (unsigned long long)DI,
                        (unsigned long long)p.B * p.Hkv * p.L_max, (unsigned long long)SG::RB, DI, p.stage_keys,
                        SG::RB))
        return cudaErrorInvalidValue;
      return launch_cluster_t<T, D, DI, 8, true>(p, kmap, st);
    }
    return cudaErrorInvalidValue;
  }
  // CTAs per (sequence, KV head): 16 keeps one small step short; with many
  // (sequence, KV head) pairs in the launch, fewer CTAs per pair (two per SM)
  // spend less SM time per step.
  int nc = p.split_req > 16 ? 16 : p.split_req;   // 32, 64 (the wide form) where it does not apply: 16
  if (nc == 0) {
    const int pairs = p.B * p.Hkv;
    nc = pairs * 16 <= sms ? 16 : pairs * 8 <= 2 * sms ? 8 : 4;
  }
  if (nc == 16 && !ok16) nc = 8;
  if (nc == 4 && dec_layout((((p.L_max + 3) / 4) + 31) & ~31, p.L_max, p.M, p.G, D, DI, (int)sizeof(T), 4, 2,
                            kStageBytes, p.k_lin != nullptr).total >
                     227 * 1024)
    nc = 8;
  p.nc = nc;
  // 16 CTAs: 4 stages of 32 KB; fewer: 2 stages, so two CTAs fit one SM
  p.stages = nc == 16 ? 4 : 2;
  p.stage_keys = ScoreGeom<T, DI>::sub(32768);
  p.kpc_max = (((p.L_max + nc - 1) / nc) + 31) & ~31;
  CUtensorMap kmap;
  memset(&kmap, 0, sizeof(kmap));
  if (ScoreGeom<T, DI>::kMma && !p.sel_ext) {   // given lists: no key stream
    using SG = ScoreGeom<T, DI>;
    if (!make_tmap_2d(&kmap, p.kidx_cache, (int)sizeof(T), (unsigned long long)DI,
                      (unsigned long long)p.B * p.Hkv * p.L_max, (unsigned long long)SG::RB, DI, p.stage_keys, SG::RB))
      return cudaErrorInvalidValue;
  }
  if (nc == 16) return launch_cluster_t<T, D, DI, 16>(p, kmap, st);
  if (nc == 4) return launch_cluster_t<T, D, DI, 4>(p, kmap, st);
  return launch_cluster_t<T, D, DI, 8>(p, kmap, st);
}

// Workspace of the wide form, sized for nw CTAs per (b, g): arrival counters,
// per-CTA partial readouts and the order keys (each block 256-byte aligned).
size_t decode_wide_workspace_bytes(int B, int Hkv, int G, int D, int L_max, int nw) {
  (void)G;
  const size_t pairs = (size_t)B * Hkv;
  auto r256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return r256(pairs * 4) + r256(pairs * nw * 2 * D * 4) + r256(pairs * (size_t)((L_max + 3) & ~3) * 4);
}

// The library's choice never takes the wide form: measured on a B200 at the
// 1.5B shape (16K context), one wide step (128 CTAs) took 24-25 us against
// about 20 us for one 16-CTA cluster, because its publish / arrival / reload
// steps cost more than the faster key stream saves.  It stays available on
// request (decode_split 32 or 64).
int decode_wide_nw(int B, int Hkv, int G, int D, int DI, int dtype, int sms) {
  (void)B; (void)Hkv; (void)G; (void)D; (void)DI; (void)dtype; (void)sms;
  return 0;
}

// Dynamic shared memory of the wide form (bf16; ring stages of at most 32 KB).
int decode_wide_smem_bytes(int L_max, int M, int G, int D, int DI, int nw) {
  const int kpc = (nw / 8) * ((((L_max + nw - 1) / nw) + 31) & ~31);
  return dec_layout(kpc, L_max, M, G, D, DI, 2, 8, 2, kStageBytes, false, true).total;
}

int decode_smem_bytes(int L_max, int M, int G, int D, int DI, int esize, int nc, bool lin_kv) {
  const int kpc = (((L_max + nc - 1) / nc) + 31) & ~31;
  return dec_layout(kpc, L_max, M, G, D, DI, esize, nc, kStages, kStageBytes, lin_kv).total;
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
