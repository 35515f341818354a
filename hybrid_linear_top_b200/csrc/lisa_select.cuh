// Exact block-wide top-M selection over order keys (see score_key()).
//
// Selection rule (a definition of this library; the LISA pages only say
// "top-M"): the first min(M, n) positions in the order (key descending,
// position ascending), written in ascending position order, padded with -1.
//
// Method: MSB-first radix select over the 32-bit key in four 8-bit digits
// finds the key K* of the M-th entry and how many entries equal to K* are
// still needed; one ordered ballot/popc pass then emits the positions.  After
// the first digit only the keys of the threshold bucket are revisited (they are
// copied to a small shared-memory list when they fit).
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

}  // namespace lisa
