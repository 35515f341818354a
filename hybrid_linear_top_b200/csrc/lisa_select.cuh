// Exact block-wide top-M selection over order keys (see score_key()).
//
// Selection rule (a definition of this library; the LISA pages only say
// "top-M"): the first min(M, n) positions in the order (key descending,
// position ascending), written in ascending position order, padded with -1.
//
// Three methods:
//  * block_topm_sampled (long rows in global memory): a bound from a 1/8 (or
//    sparser) block sample of the keys, then one pass of 16-byte loads that
//    compacts the keys above it per warp; the exact K* and the ordered
//    emission work on those per-warp segments.  Falls back to the next
//    method when fewer than M keys pass the bound or a segment is full.
//  * block_topm_bounded (long rows): every thread keeps its 4 largest keys;
//    the bin of the M-th largest of those values gives a bound lb with at
//    least M keys >= lb; the keys >= lb are compacted in position order; the
//    exact M-th key K* comes from 1024-bin range histograms (range_kth); an
//    ordered compaction emits the positions.
//  * block_topm (short rows, and rows where too many keys pass the bound):
//    MSB-first radix select over the 32-bit key in four 8-bit digits finds K*
//    and how many entries equal to K* are still needed; one ordered
//    ballot/popc pass then emits the positions.  After the first digit only
//    the keys of the threshold bucket are revisited.
#pragma once

#include "lisa_common.cuh"

namespace lisa {

struct TopmShared {
  uint32_t hist[256];
  uint32_t wg[32];      // per-warp counts of keys > K*
  uint32_t we[32];      // per-warp counts of keys == K*
  uint32_t bc_digit;
  uint32_t bc_above;
  uint32_t cand_n;
};

// Warp-aggregated histogram add of `dig` for lanes with `act`.
__device__ __forceinline__ void hist_add(uint32_t *hist, bool act, uint32_t dig) {
  const unsigned am = __ballot_sync(0xffffffffu, act);
  if (act) {
    const unsigned peers = __match_any_sync(am, dig);
    const int lane = threadIdx.x & 31;
    if (lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (uint32_t)__popc(peers));
  }
}

// Warp 0 scans the 256 bins from the top and finds the bucket holding the
// rem-th largest key; writes bc_digit / bc_above.  Call between barriers.
__device__ __forceinline__ void find_bucket(TopmShared &sm, uint32_t rem) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t c[8];
    uint32_t tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = sm.hist[255 - (8 * lane + j)];
      tot += c[j];
    }
    uint32_t inc = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const uint32_t exc = inc - tot;
    if (exc < rem && rem <= inc) {
      uint32_t cum = exc;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (cum + c[j] >= rem) {
          sm.bc_digit = 255u - (uint32_t)(8 * lane + j);
          sm.bc_above = cum;
          break;
        }
        cum += c[j];
      }
    }
  }
}

// keys: n order keys (shared or global memory), position i has key keys[i].
// cand: shared scratch of cand_cap uint32.  out: M int32 (global).
// Must be called by all NT threads of the block.
// Returns false (and writes -1 everywhere) if an internal check failed.
template <int NT>
__device__ bool block_topm(const uint32_t *keys, int n, int M, int *out, TopmShared &sm, uint32_t *cand,
                           int cand_cap) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  if (n <= M) {
    for (int i = tid; i < M; i += NT) out[i] = i < n ? i : -1;
    return true;
  }

  uint32_t prefix = 0, pmask = 0, rem = (uint32_t)M;
  bool use_cand = false;
  int cand_n = 0;

#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    // every thread has read the previous pass's bucket before it is cleared
    __syncthreads();
    for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    if (use_cand) {
      for (int base = 0; base < cand_n; base += NT) {
        const int i = base + tid;
        uint32_t u = 0;
        bool act = false;
        if (i < cand_n) {
          u = cand[i];
          act = (u & pmask) == prefix;
        }
        hist_add(sm.hist, act, (u >> shift) & 255u);
      }
    } else {
      for (int base = 0; base < n; base += NT) {
        const int i = base + tid;
        uint32_t u = 0;
        bool act = false;
        if (i < n) {
          u = keys[i];
          act = (u & pmask) == prefix;
        }
        hist_add(sm.hist, act, (u >> shift) & 255u);
      }
    }
    if (tid == 0) sm.bc_digit = 0xFFFFFFFFu;
    __syncthreads();
    find_bucket(sm, rem);
    __syncthreads();
    const uint32_t dig = sm.bc_digit;
    if (dig > 255u) {  // counts inconsistent: cannot happen for a valid key array
      for (int i = tid; i < M; i += NT) out[i] = -1;
      return false;
    }
    const uint32_t above = sm.bc_above;
    const uint32_t in_bucket = sm.hist[dig];
    rem -= above;
    prefix |= dig << shift;
    pmask |= 255u << shift;

    if (pass == 0 && (int)in_bucket <= cand_cap) {
      // copy the keys of the threshold bucket to the candidate list
      if (tid == 0) sm.cand_n = 0;
      __syncthreads();
      for (int base = 0; base < n; base += NT) {
        const int i = base + tid;
        uint32_t u = 0;
        bool act = false;
        if (i < n) {
          u = keys[i];
          act = (u & pmask) == prefix;
        }
        const unsigned am = __ballot_sync(0xffffffffu, act);
        uint32_t wbase = 0;
        if (lane == 0 && am) wbase = atomicAdd(&sm.cand_n, (uint32_t)__popc(am));
        wbase = __shfl_sync(0xffffffffu, wbase, 0);
        if (act) cand[wbase + __popc(am & ((1u << lane) - 1u))] = u;
      }
      __syncthreads();
      cand_n = (int)sm.cand_n;
      use_cand = true;
    }
  }
  const uint32_t kstar = prefix;
  const uint32_t need_eq = rem;  // >= 1

  // ordered emission: warp w owns a contiguous chunk of positions
  const int per_warp = (((n + NW - 1) / NW) + 31) & ~31;
  const int c0 = warp * per_warp;
  const int c1 = min(n, c0 + per_warp);
  uint32_t g = 0, e = 0;
  for (int base = c0; base < c1; base += 32) {
    const int i = base + lane;
    const uint32_t u = i < c1 ? keys[i] : 0u;
    g += __popc(__ballot_sync(0xffffffffu, i < c1 && u > kstar));
    e += __popc(__ballot_sync(0xffffffffu, i < c1 && u == kstar));
  }
  if (lane == 0) {
    sm.wg[warp] = g;
    sm.we[warp] = e;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t vg = lane < NW ? sm.wg[lane] : 0u;
    uint32_t ve = lane < NW ? sm.we[lane] : 0u;
    uint32_t ig = vg, ie = ve;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t yg = __shfl_up_sync(0xffffffffu, ig, o);
      const uint32_t ye = __shfl_up_sync(0xffffffffu, ie, o);
      if (lane >= o) {
        ig += yg;
        ie += ye;
      }
    }
    if (lane < NW) {
      sm.wg[lane] = ig - vg;
      sm.we[lane] = ie - ve;
    }
  }
  __syncthreads();
  g = sm.wg[warp];
  e = sm.we[warp];
  const unsigned lt = (1u << lane) - 1u;
  bool bad = false;
  for (int base = c0; base < c1; base += 32) {
    const int i = base + lane;
    const uint32_t u = i < c1 ? keys[i] : 0u;
    const unsigned bg = __ballot_sync(0xffffffffu, i < c1 && u > kstar);
    const unsigned be = __ballot_sync(0xffffffffu, i < c1 && u == kstar);
    const uint32_t pe = e + __popc(be & lt);
    const bool gt = (bg >> lane) & 1u;
    const bool eq = (be >> lane) & 1u;
    if (gt || (eq && pe < need_eq)) {
      const uint32_t o = g + __popc(bg & lt) + min(pe, need_eq);
      if (o < (uint32_t)M) out[o] = i;
      else bad = true;
    }
    g += __popc(bg);
    e += __popc(be);
  }
  return !__syncthreads_or(bad);
}


// ---------------------------------------------------------------- range-histogram select helpers
// CTA-wide (NT = 256 threads, 4 bins each): the bin of fh[0..1024) (higher bin
// = larger keys) that holds the rem-th largest key, counting from the top.
// misc[0] = bin (0xFFFFFFFF if the counts hold fewer than rem keys), misc[1] =
// keys in higher bins, misc[2] = keys in the bin; misc[3] is zeroed.  Uses
// misc[8..15].  Ends with a barrier.
template <int NT>
__device__ void find_bin1024(const uint32_t *fh, uint32_t rem, uint32_t *misc) {
  static_assert(NT * 4 == 1024, "four bins per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = 1023 - 4 * tid;
  const uint32_t c0 = fh[b0], c1 = fh[b0 - 1], c2 = fh[b0 - 2], c3 = fh[b0 - 3];
  const uint32_t c = c0 + c1 + c2 + c3;
  uint32_t inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) misc[8 + warp] = inc;
  if (tid == 0) {
    misc[0] = 0xFFFFFFFFu;
    misc[3] = 0;
  }
  __syncthreads();
  uint32_t off = 0;
#pragma unroll
  for (int w8 = 0; w8 < NT / 32; ++w8) off += w8 < warp ? misc[8 + w8] : 0u;
  const uint32_t exc = off + inc - c;
  if (exc < rem && rem <= exc + c) {
    const uint32_t cc[4] = {c0, c1, c2, c3};
    uint32_t cum = exc;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (cum < rem && rem <= cum + cc[j]) {
        misc[0] = (uint32_t)(b0 - j);
        misc[1] = cum;
        misc[2] = cc[j];
      }
      cum += cc[j];
    }
  }
  __syncthreads();
}

// find_bin1024 for two ranks in one scan: misc[0..2] for rank ra, misc[4..6]
// for rank rb (bin, keys in higher bins, keys in the bin; bin 0xFFFFFFFF when
// the counts hold fewer keys than the rank), misc[7] = keys in all bins;
// misc[3] is zeroed.  Uses misc[8..15].  Ends with a barrier.
template <int NT>
__device__ void find_bin1024_two(const uint32_t *fh, uint32_t ra, uint32_t rb, uint32_t *misc) {
  static_assert(NT * 4 == 1024, "four bins per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = 1023 - 4 * tid;
  const uint32_t cc[4] = {fh[b0], fh[b0 - 1], fh[b0 - 2], fh[b0 - 3]};
  const uint32_t c = cc[0] + cc[1] + cc[2] + cc[3];
  uint32_t inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) misc[8 + warp] = inc;
  if (tid == 0) {
    misc[0] = 0xFFFFFFFFu;
    misc[4] = 0xFFFFFFFFu;
    misc[3] = 0;
  }
  __syncthreads();
  uint32_t off = 0, all = 0;
#pragma unroll
  for (int w8 = 0; w8 < NT / 32; ++w8) {
    off += w8 < warp ? misc[8 + w8] : 0u;
    all += misc[8 + w8];
  }
  const uint32_t exc = off + inc - c;
  if (tid == 0) misc[7] = all;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint32_t rem = k == 0 ? ra : rb;
    if (exc < rem && rem <= exc + c) {
      uint32_t cum = exc;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (cum < rem && rem <= cum + cc[j]) {
          misc[4 * k] = (uint32_t)(b0 - j);
          misc[4 * k + 1] = cum;
          misc[4 * k + 2] = cc[j];
        }
        cum += cc[j];
      }
    }
  }
  __syncthreads();
}

// CTA-wide exclusive prefix sums of two counters, plus their totals.  Uses
// misc[32..47].
template <int NT>
__device__ __forceinline__ void cta_scan2(uint32_t a, uint32_t b, uint32_t &ea, uint32_t &eb, uint32_t &ta,
                                          uint32_t &tb, uint32_t *misc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t ya = __shfl_up_sync(0xffffffffu, ia, o), yb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += ya;
      ib += yb;
    }
  }
  __syncthreads();
  if (lane == 31) {
    misc[32 + warp] = ia;
    misc[40 + warp] = ib;
  }
  __syncthreads();
  uint32_t wa = 0, wb = 0;
  ta = 0;
  tb = 0;
  for (int w8 = 0; w8 < NT / 32; ++w8) {
    if (w8 < warp) {
      wa += misc[32 + w8];
      wb += misc[40 + w8];
    }
    ta += misc[32 + w8];
    tb += misc[40 + w8];
  }
  ea = wa + ia - a;
  eb = wb + ib - b;
}

// Exact M-th largest key K* among keys ck[0..nc) that all lie in [lo, hi]:
// 1024-bin range histograms narrowed until one bin holds <= 32 keys (ranked
// in one warp) or is a single value.  Writes K* and need_eq = how many keys
// equal to K* the top M takes; returns false if the counts are inconsistent.
// fh: 1024 words of shared scratch; misc: 64 words.  All NT threads call it.
template <int NT>
__device__ bool range_kth(const uint32_t *ck, int nc, uint32_t lo, uint32_t hi, uint32_t M, uint32_t *fh,
                          uint32_t *misc, uint32_t *members, uint32_t &kstar, uint32_t &need_eq) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t lbx = lo, ubx = hi, rem = M;
  uint32_t shx = (hi - lo) < 1024u ? 0u : (uint32_t)(32 - __clz(hi - lo)) - 10u;
#pragma unroll 1
  for (int iter = 0; iter < 4; ++iter) {
    for (int i = tid; i < 1024; i += NT) fh[i] = 0;
    __syncthreads();
    for (int j = tid; j < nc; j += NT) {
      const uint32_t u = ck[j];
      if (u >= lbx && u <= ubx) atomicAdd(&fh[(u - lbx) >> shx], 1u);
    }
    __syncthreads();
    find_bin1024<NT>(fh, rem, misc);
    const uint32_t bin = misc[0];
    if (bin > 1023u) return false;
    rem -= misc[1];
    const uint32_t cb = misc[2];
    const uint32_t blo = lbx + (bin << shx);
    if (shx == 0) {
      kstar = blo;
      need_eq = rem;
      return true;
    }
    if (cb <= 32) {
      for (int j = tid; j < nc; j += NT) {
        const uint32_t u = ck[j];
        if (u >= blo && u <= ubx && ((u - lbx) >> shx) == bin) {
          const uint32_t s = atomicAdd(&misc[3], 1u);
          if (s < 32) members[s] = u;
        }
      }
      __syncthreads();
      if (warp == 0) {
        const uint32_t x = lane < (int)cb ? members[lane] : 0u;
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
      __syncthreads();
      return true;
    }
    const unsigned long long top = (unsigned long long)blo + (1ull << shx) - 1ull;
    lbx = blo;
    ubx = top < ubx ? (uint32_t)top : ubx;
    shx = shx > 10u ? shx - 10u : 0u;
    __syncthreads();
  }
  return false;
}

struct BoundedShared {
  uint32_t fh[1024];
  uint32_t misc[64];
  uint32_t members[32];
};

// Top-M of keys[0..n) (shared memory, n > M, n >= 8 * NT) through a bound:
// every thread keeps the 4 largest of its keys; the bin holding the M-th
// largest of those 4 * NT values gives lb with at least M keys >= lb; the keys
// >= lb are compacted in position order into (ck, cp); the exact K* among them
// and an ordered compaction emit the ascending index list.
// Returns 1 when done, 0 when more than cap keys pass the bound (nothing
// written; the caller selects another way), -1 on an internal check failure.
template <int NT>
__device__ int block_topm_bounded(const uint32_t *keys, int n, int M, int *out, BoundedShared &sm, uint32_t *ck,
                                  int *cp, int cap) {
  static_assert(NT == 256, "256 threads");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // (1) the 4 largest keys of each thread
  uint32_t t0 = 0, t1 = 0, t2 = 0, t3 = 0;
  for (int i = tid; i < n; i += NT) {
    uint32_t u = keys[i];
    if (u > t3) {
      t3 = u;
      if (t3 > t2) { const uint32_t x = t2; t2 = t3; t3 = x; }
      if (t2 > t1) { const uint32_t x = t1; t1 = t2; t2 = x; }
      if (t1 > t0) { const uint32_t x = t0; t0 = t1; t1 = x; }
    }
  }
  // range of those values
  uint32_t vmin = t3, vmax = t0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  if (lane == 0) {
    sm.misc[16 + warp] = vmin;
    sm.misc[24 + warp] = vmax;
  }
  for (int i = tid; i < 1024; i += NT) sm.fh[i] = 0;
  __syncthreads();
#pragma unroll
  for (int w8 = 0; w8 < NT / 32; ++w8) {
    vmin = min(vmin, sm.misc[16 + w8]);
    vmax = max(vmax, sm.misc[24 + w8]);
  }
  // (2) lb = lower edge of the bin of the M-th largest of the 4 * NT values
  const uint32_t sh = (vmax - vmin) < 1024u ? 0u : (uint32_t)(32 - __clz(vmax - vmin)) - 10u;
  atomicAdd(&sm.fh[(t0 - vmin) >> sh], 1u);
  atomicAdd(&sm.fh[(t1 - vmin) >> sh], 1u);
  atomicAdd(&sm.fh[(t2 - vmin) >> sh], 1u);
  atomicAdd(&sm.fh[(t3 - vmin) >> sh], 1u);
  __syncthreads();
  find_bin1024<NT>(sm.fh, (uint32_t)M, sm.misc);
  if (sm.misc[0] > 1023u) return -1;
  const uint32_t lb = vmin + (sm.misc[0] << sh);
  // (3) keys >= lb in position order: warp w owns a contiguous run
  const int cw = (((n + 7) / 8) + 31) & ~31;
  const int j0 = min(n, warp * cw), j1 = min(n, j0 + cw);
  uint32_t wc = 0;
  for (int base = j0; base < j1; base += 32) {
    const int j = base + lane;
    wc += __popc(__ballot_sync(0xffffffffu, j < j1 && keys[j] >= lb));
  }
  if (lane == 0) sm.misc[48 + warp] = wc;
  __syncthreads();
  uint32_t off = 0, nc = 0;
#pragma unroll
  for (int w8 = 0; w8 < NT / 32; ++w8) {
    const uint32_t c = sm.misc[48 + w8];
    off += w8 < warp ? c : 0u;
    nc += c;
  }
  if (nc > (uint32_t)cap) return 0;               // the same answer in every thread
  {
    const unsigned lt = (1u << lane) - 1u;
    for (int base = j0; base < j1; base += 32) {
      const int j = base + lane;
      const bool act = j < j1 && keys[j] >= lb;
      const unsigned am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t o = off + __popc(am & lt);
        ck[o] = keys[j];
        cp[o] = j;
      }
      off += __popc(am);
    }
  }
  __syncthreads();
  // (4) exact K* among the candidates
  uint32_t kstar = 0, need_eq = 0;
  if (!range_kth<NT>(ck, (int)nc, lb, vmax, (uint32_t)M, sm.fh, sm.misc, sm.members, kstar, need_eq)) return -1;
  // (5) ordered emission from the candidate list: thread-contiguous runs
  const int per = ((int)nc + NT - 1) / NT;
  const int c0 = min((int)nc, tid * per), c1 = min((int)nc, c0 + per);
  uint32_t cgt = 0, ceq = 0;
  for (int c = c0; c < c1; ++c) {
    const uint32_t u = ck[c];
    cgt += u > kstar ? 1u : 0u;
    ceq += u == kstar ? 1u : 0u;
  }
  uint32_t eg, ee, tg, te;
  cta_scan2<NT>(cgt, ceq, eg, ee, tg, te, sm.misc);
  bool bad = tg + need_eq != (uint32_t)M || te < need_eq;
  for (int c = c0; c < c1; ++c) {
    const uint32_t u = ck[c];
    if (u > kstar) {
      const uint32_t o = eg + min(ee, need_eq);
      if (o < (uint32_t)M) out[o] = cp[c];
      else bad = true;
      ++eg;
    } else if (u == kstar) {
      if (ee < need_eq) {
        const uint32_t o = eg + ee;
        if (o < (uint32_t)M) out[o] = cp[c];
        else bad = true;
      }
      ++ee;
    }
  }
  return __syncthreads_or(bad) ? -1 : 1;
}

// Top-M of a long row keys[0..n) (global memory, 16-byte aligned and readable
// up to n rounded up to 4; n >= 8 * NT, n > M) with one pass over the keys:
//  (1) a bound from a sample: the first 16 keys (one 64-byte block) of every
//      step-th group of 128, at most 4 blocks per thread, so the sample adds
//      no DRAM traffic to the pass that follows.  lb = the lower edge of the
//      1024-bin range bin (over the 8 octaves below the sample's largest
//      key) that holds the sample's r-th largest key, r chosen so that about
//      2M keys of the row are expected at or above lb;
//  (2) one pass of 16-byte loads: warp w compacts the keys >= lb of its
//      contiguous run, in position order, into its own segment of (ck, cp)
//      (cap / NW entries each) and tracks their largest key;
//  (3) fewer than M keys >= lb, or a full segment: returns 0 and the caller's
//      exact paths run.  Else the exact M-th key K* by range histograms over
//      the segments, and each warp emits its segment's share of the
//      ascending index list at offsets from the warps' counts.
// Returns 1 (done), 0 (bound unusable) or -1 (inconsistent counts).
template <int NT>
__device__ __forceinline__ int block_topm_sampled(const uint32_t *keys, int n, int M, int *out, BoundedShared &sm, uint32_t *ck,
                                  int *cp, int cap) {
  static_assert(NT == 256, "256 threads");
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int segcap = cap / NW;
  // (1) the sample: groups g = i * step (i < ng) of 128 keys, keys [128 g, 128 g + 16)
  const int groups = n / 128;
  const int step = (groups + 255) / 256;
  const int ng = groups / step;                       // sampled groups, at most 256: 4 uint4 per thread
  const int nsv = ng * 4;
  uint4 sv[4];
  uint32_t vmin = 0xFFFFFFFFu, vmax = 0u;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int s = tid + k * NT;
    sv[k] = make_uint4(0u, 0u, 0u, 0u);
    if (s < nsv) {
      sv[k] = __ldcg(reinterpret_cast<const uint4 *>(keys + (size_t)(s >> 2) * step * 128 + (s & 3) * 4));
      vmin = min(vmin, min(min(sv[k].x, sv[k].y), min(sv[k].z, sv[k].w)));
      vmax = max(vmax, max(max(sv[k].x, sv[k].y), max(sv[k].z, sv[k].w)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  if (lane == 0) {
    sm.misc[48 + warp] = vmin;
    sm.misc[56 + warp] = vmax;
  }
  for (int i = tid; i < 1024; i += NT) sm.fh[i] = 0;
  __syncthreads();
#pragma unroll
  for (int w8 = 0; w8 < NW; ++w8) {
    vmin = min(vmin, sm.misc[48 + w8]);
    vmax = max(vmax, sm.misc[56 + w8]);
  }
  const uint32_t lo = (vmax - vmin) > (8u << 23) ? vmax - (8u << 23) : vmin;
  const uint32_t sh = (vmax - lo) < 1024u ? 0u : (uint32_t)(32 - __clz(vmax - lo)) - 10u;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (tid + k * NT < nsv) {
      const uint32_t w4[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (w4[q] >= lo) atomicAdd(&sm.fh[(w4[q] - lo) >> sh], 1u);
    }
  }
  __syncthreads();
  // about 2M keys at or above the r-th largest of the nsv * 4 sampled keys
  const long long r_ll = (2ll * M * nsv * 4 + n - 1) / n;
  const uint32_t r = (uint32_t)(r_ll < 1 ? 1 : r_ll);
  find_bin1024<NT>(sm.fh, r, sm.misc);
  const uint32_t lb = sm.misc[0] <= 1023u ? lo + (sm.misc[0] << sh) : lo;
  // (2) one pass: warp w's run [j0, j1) of positions, 128 per iteration
  const int cw = (((n + NW - 1) / NW) + 127) & ~127;
  const int j0 = min(n, warp * cw), j1 = min(n, j0 + cw);
  uint32_t *cks = ck + warp * segcap;
  int *cps = cp + warp * segcap;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t cnt = 0, cmax = 0u;
  // the next iteration's 16 bytes are requested before this one's are used
  uint4 vn = make_uint4(0u, 0u, 0u, 0u);
  if (j0 + 4 * lane < j1) vn = __ldcg(reinterpret_cast<const uint4 *>(keys + j0 + 4 * lane));
  for (int base = j0; base < j1; base += 128) {
    const int idx = base + 4 * lane;
    const uint4 v = vn;
    if (idx + 128 < j1) vn = __ldcg(reinterpret_cast<const uint4 *>(keys + idx + 128));
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    bool f[4];
    unsigned bl[4];
    uint32_t before = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      f[q] = idx + q < j1 && w4[q] >= lb;
      bl[q] = __ballot_sync(0xffffffffu, f[q]);
      before += __popc(bl[q] & lt);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (f[q]) {
        const uint32_t o = cnt + before;
        if (o < (uint32_t)segcap) {
          cks[o] = w4[q];
          cps[o] = idx + q;
        }
        cmax = max(cmax, w4[q]);
        ++before;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) cnt += __popc(bl[q]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
  if (lane == 0) {
    sm.misc[16 + warp] = cnt;
    sm.misc[24 + warp] = cmax;
  }
  __syncthreads();
  uint32_t total = 0, hi = 0;
  bool full = false;
#pragma unroll
  for (int w8 = 0; w8 < NW; ++w8) {
    total += sm.misc[16 + w8];
    hi = max(hi, sm.misc[24 + w8]);
    full = full || sm.misc[16 + w8] > (uint32_t)segcap;
  }
  if (full || total < (uint32_t)M) {                  // the same answer in every thread
    __syncthreads();                                  // read by all before the caller reuses sm
    return 0;
  }
  cnt = sm.misc[16 + warp];
  // (3) K*: 1024-bin range histograms over [lb, hi] of the segments, narrowed
  //     until the bin of the rem-th key is one value or holds <= 32 keys
  uint32_t kstar = 0, need_eq = 0;
  {
    uint32_t lbx = lb, ubx = hi, rem = (uint32_t)M;
    uint32_t shx = (ubx - lbx) < 1024u ? 0u : (uint32_t)(32 - __clz(ubx - lbx)) - 10u;
    bool done = false;
#pragma unroll 1
    for (int iter = 0; iter < 4 && !done; ++iter) {
      __syncthreads();                                // every thread is done with the previous bins
      for (int i = tid; i < 1024; i += NT) sm.fh[i] = 0;
      __syncthreads();
      for (int j = lane; j < (int)cnt; j += 32) {
        const uint32_t u = cks[j];
        if (u >= lbx && u <= ubx) atomicAdd(&sm.fh[(u - lbx) >> shx], 1u);
      }
      __syncthreads();
      find_bin1024<NT>(sm.fh, rem, sm.misc);
      const uint32_t bin = sm.misc[0];
      if (bin > 1023u) return -1;
      rem -= sm.misc[1];
      const uint32_t cb = sm.misc[2];
      const uint32_t blo = lbx + (bin << shx);
      if (shx == 0u) {
        kstar = blo;
        need_eq = rem;
        done = true;
      } else if (cb <= 32u) {
        if (tid == 0) sm.misc[7] = 0xFFFFFFFFu;
        for (int j = lane; j < (int)cnt; j += 32) {
          const uint32_t u = cks[j];
          if (u >= lbx && u <= ubx && ((u - lbx) >> shx) == bin) {
            const uint32_t s = atomicAdd(&sm.misc[3], 1u);
            if (s < 32u) sm.members[s] = u;
          }
        }
        __syncthreads();
        if (warp == 0) {
          const uint32_t x = lane < (int)cb ? sm.members[lane] : 0u;
          uint32_t gt = 0, ge = 0;
          for (int j = 0; j < (int)cb; ++j) {
            const uint32_t y = __shfl_sync(0xffffffffu, x, j);
            gt += y > x ? 1u : 0u;
            ge += y >= x ? 1u : 0u;
          }
          if (lane < (int)cb && gt < rem && rem <= ge) {
            sm.misc[5] = x;
            sm.misc[7] = rem - gt;
          }
        }
        __syncthreads();
        kstar = sm.misc[5];
        need_eq = sm.misc[7];
        if (need_eq == 0xFFFFFFFFu) return -1;
        done = true;
      } else {
        const uint64_t top = (uint64_t)blo + ((1ull << shx) - 1ull);
        lbx = blo;
        ubx = top > (uint64_t)ubx ? ubx : (uint32_t)top;
        shx = shx > 10u ? shx - 10u : 0u;
      }
    }
    if (!done) return -1;
  }
  // (4) the ascending index list: each warp counts its segment's keys > K*
  //     and == K*, then emits them at offsets from the earlier warps' counts
  uint32_t ngt = 0, neq = 0;
  for (int base = 0; base < (int)cnt; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < (int)cnt ? cks[j] : 0u;
    ngt += __popc(__ballot_sync(0xffffffffu, j < (int)cnt && u > kstar));
    neq += __popc(__ballot_sync(0xffffffffu, j < (int)cnt && u == kstar));
  }
  if (lane == 0) {
    sm.misc[32 + warp] = ngt;
    sm.misc[40 + warp] = neq;
  }
  __syncthreads();
  uint32_t gb = 0, eb = 0, gtot = 0, etot = 0;
#pragma unroll
  for (int w8 = 0; w8 < NW; ++w8) {
    const uint32_t a = sm.misc[32 + w8], c = sm.misc[40 + w8];
    gb += w8 < warp ? a : 0u;
    eb += w8 < warp ? c : 0u;
    gtot += a;
    etot += c;
  }
  bool bad = gtot + need_eq != (uint32_t)M || etot < need_eq;
  for (int base = 0; base < (int)cnt; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < (int)cnt ? cks[j] : 0u;
    const unsigned bgt = __ballot_sync(0xffffffffu, j < (int)cnt && u > kstar);
    const unsigned beq = __ballot_sync(0xffffffffu, j < (int)cnt && u == kstar);
    const uint32_t pe = eb + __popc(beq & lt);
    const bool gt = (bgt >> lane) & 1u, eq = (beq >> lane) & 1u;
    if (gt || (eq && pe < need_eq)) {
      const uint32_t o = gb + __popc(bgt & lt) + min(pe, need_eq);
      if (o < (uint32_t)M) out[o] = cps[j];
      else bad = true;
    }
    gb += __popc(bgt);
    eb += __popc(beq);
  }
  return __syncthreads_or(bad) ? -1 : 1;
}

}  // namespace lisa
