// Block-wide radix select and ordered (stable) compaction.
//
// Both the per-group top-k of the anchor step and every PDDP cut pick "the m
// smallest of n keys, ties to the earlier position": top-k on the key
// ~order(score) over the key index, a PDDP cut on order(projection) over a
// node whose members are kept in ascending token order. The selection is
// found by a 3-pass radix select (11 + 11 + 10 bits) on the 32-bit keys and
// then written out by one in-order pass with block-wide prefix counts, so the
// selected members come out in position order and the rest in position order.
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

// Exclusive prefix of a 0/1 flag over the block, plus the block total.
__device__ __forceinline__ uint32_t block_excl_count(bool flag, uint32_t* warp_tot,
                                                     uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
  const uint32_t in_warp = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(ballot);
  __syncthreads();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSelectThreads / 32; ++w) {
    const uint32_t c = warp_tot[w];
    before += (w < warp) ? c : 0u;
    tot += c;
  }
  __syncthreads();
  total = tot;
  return before + in_warp;
}

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
    for (int i = threadIdx.x; i < n; i += kSelectThreads) {
      const uint32_t k = key(i);
      if ((k & prefix_mask) == prefix) atomicAdd(&sh.hist[(k >> shift) & dmask], 1u);
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
// rest(pos_in_rest, i) for the others. 0 <= m <= n.
template <class KeyFn, class SelFn, class RestFn>
__device__ void select_smallest_ordered(KeyFn key, int n, int m, SelectShared& sh, SelFn sel,
                                        RestFn rest) {
  uint32_t T = 0;
  int need_eq = 0;
  bool take_all = (m >= n), take_none = (m <= 0);
  if (!take_all && !take_none) radix_select(key, n, m, sh, &T, &need_eq);
  uint32_t run_sel = 0, run_eq = 0;
  for (int base = 0; base < n; base += kSelectThreads) {
    const int i = base + threadIdx.x;
    const bool valid = i < n;
    bool s;
    if (take_all || take_none) {
      s = valid && take_all;
    } else {
      const uint32_t k = valid ? key(i) : 0xffffffffu;
      const bool lt = valid && k < T;
      const bool eq = valid && k == T;
      uint32_t eq_tot;
      const uint32_t eq_rank = run_eq + block_excl_count(eq, sh.warp_tot2, eq_tot);
      run_eq += eq_tot;
      s = lt || (eq && eq_rank < (uint32_t)need_eq);
    }
    uint32_t sel_tot;
    const uint32_t pos = run_sel + block_excl_count(s, sh.warp_tot, sel_tot);
    if (valid) {
      if (s)
        sel(pos, i);
      else
        rest((uint32_t)i - pos, i);
    }
    run_sel += sel_tot;
  }
}

}  // namespace tlsp
