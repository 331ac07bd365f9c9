// Block-wide radix select and ordered (stable) compaction.
//
// Both the per-group top-k of the anchor step and every PDDP cut pick "the m
// smallest of n keys, ties to the earlier position": top-k on the key
// ~order(score) over the key index, a PDDP cut on order(projection) over a
// node whose members are kept in ascending token order. The selection is
// found by a 3-pass radix select (11 + 11 + 10 bits) on the 32-bit keys and
// then written out in position order (the selected members, and separately
// the rest) from per-warp counts over contiguous ranges.
#pragma once

#include "common.cuh"

namespace tlsp {

constexpr int kSelectThreads = 512;
constexpr int kRadixBins = 2048;

struct SelectShared {
  uint32_t hist[kRadixBins];
  uint32_t warp_tot[kSelectThreads / 32];
  uint32_t warp_tot2[kSelectThreads / 32];
  uint32_t bcast[4];
};

// Finds the m-th smallest key (1 <= m <= n) among key(0..n-1).
// On return *T is that key and *need_eq is how many of the keys equal to T
// (the earliest ones) belong to the m smallest.
template <class KeyFn>
__device__ void radix_select(KeyFn key, int n, int m, SelectShared& sh, uint32_t* T,
                             int* need_eq) {
  uint32_t prefix = 0, prefix_mask = 0;
  uint32_t rank = (uint32_t)m;  // 1-based rank still to find inside the prefix
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const uint32_t dmask = (1u << widths[pass]) - 1u;
    for (int b = threadIdx.x; b < kRadixBins; b += kSelectThreads) sh.hist[b] = 0;
    __syncthreads();
    // Lanes whose keys fall in the same bin add once per warp (match.any):
    // neighbouring keys often share a bin, and same-address shared atomics
    // would otherwise serialise.
    for (int base = 0; base < n; base += kSelectThreads) {
      const int i = base + threadIdx.x;
      uint32_t bin = 0xffffffffu;
      if (i < n) {
        const uint32_t k = key(i);
        if ((k & prefix_mask) == prefix) bin = (k >> shift) & dmask;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin != 0xffffffffu && (int)(threadIdx.x & 31) == __ffs(peers) - 1)
        atomicAdd(&sh.hist[bin], (uint32_t)__popc(peers));
    }
    __syncthreads();
    // Each thread owns 4 consecutive bins; a block scan of the per-thread sums
    // locates the bin where the running count reaches `rank`.
    constexpr int per = kRadixBins / kSelectThreads;
    uint32_t local[per], lsum = 0;
#pragma unroll
    for (int q = 0; q < per; ++q) {
      local[q] = sh.hist[threadIdx.x * per + q];
      lsum += local[q];
    }
    // inclusive warp scan of lsum
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) sh.warp_tot[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += sh.warp_tot[w];
    const uint32_t excl = before + incl - lsum;
    if (excl < rank && rank <= excl + lsum) {
      uint32_t run = excl;
#pragma unroll
      for (int q = 0; q < per; ++q) {
        if (run < rank && rank <= run + local[q]) {
          sh.bcast[0] = (uint32_t)(threadIdx.x * per + q);
          sh.bcast[1] = rank - run;
        }
        run += local[q];
      }
    }
    __syncthreads();
    prefix |= sh.bcast[0] << shift;
    prefix_mask |= dmask << shift;
    rank = sh.bcast[1];
    __syncthreads();
  }
  *T = prefix;
  *need_eq = (int)rank;
}

// Selects the m smallest of key(0..n-1) (ties to the lower position) and
// emits them in position order: sel(pos_in_selection, i) for selected i and
// rest(pos_in_rest, i) for the others. 0 <= m <= n. Each warp owns one
// contiguous range of positions: a first pass counts its keys below and equal
// to the threshold, one block-wide exchange turns the counts into starting
// offsets, and a second pass writes its members with in-warp ballots.
template <class KeyFn, class SelFn, class RestFn>
__device__ void select_smallest_ordered(KeyFn key, int n, int m, SelectShared& sh, SelFn sel,
                                        RestFn rest) {
  constexpr int W = kSelectThreads / 32;
  uint32_t T = 0;
  int need_eq = 0;
  const bool take_all = (m >= n), take_none = (m <= 0);
  const bool cut = !take_all && !take_none;
  if (cut) radix_select(key, n, m, sh, &T, &need_eq);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int seg = (n + W * 32 - 1) / (W * 32) * 32;
  const int b0 = min(n, warp * seg), b1 = min(n, b0 + seg);
  uint32_t sel_run = take_all ? (uint32_t)b0 : 0u, eq_run = 0;
  if (cut) {
    uint32_t c_lt = 0, c_eq = 0;
    for (int base = b0; base < b1; base += 32) {
      const int i = base + lane;
      const bool valid = i < b1;
      const uint32_t k = valid ? key(i) : 0u;
      c_lt += __popc(__ballot_sync(0xffffffffu, valid && k < T));
      c_eq += __popc(__ballot_sync(0xffffffffu, valid && k == T));
    }
    if (lane == 0) {
      sh.warp_tot[warp] = c_lt;
      sh.warp_tot2[warp] = c_eq;
    }
    __syncthreads();
    uint32_t lt_before = 0;
    for (int w = 0; w < warp; ++w) {
      lt_before += sh.warp_tot[w];
      eq_run += sh.warp_tot2[w];
    }
    sel_run = lt_before + min(eq_run, (uint32_t)need_eq);
  }
  for (int base = b0; base < b1; base += 32) {
    const int i = base + lane;
    const bool valid = i < b1;
    bool s = valid && take_all;
    if (cut) {
      const uint32_t k = valid ? key(i) : 0u;
      const bool eq = valid && k == T;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const uint32_t eq_rank = eq_run + __popc(eqb & below);
      eq_run += __popc(eqb);
      s = (valid && k < T) || (eq && eq_rank < (uint32_t)need_eq);
    }
    const uint32_t sb = __ballot_sync(0xffffffffu, s);
    const uint32_t pos = sel_run + __popc(sb & below);
    if (valid) {
      if (s)
        sel(pos, i);
      else
        rest((uint32_t)i - pos, i);
    }
    sel_run += __popc(sb);
  }
}

}  // namespace tlsp
