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

// Locates the bin of sh.hist where the running count reaches `rank`
// (1-based): sh.bcast[0] = bin, sh.bcast[1] = rank within that bin. Each
// thread owns kRadixBins / kSelectThreads consecutive bins; a block scan of the
// per-thread sums finds the owner. Ends with a barrier.
__device__ __forceinline__ void find_rank_bin(SelectShared& sh, uint32_t rank) {
  constexpr int per = kRadixBins / kSelectThreads;
  uint32_t local[per], lsum = 0;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    local[q] = sh.hist[threadIdx.x * per + q];
    lsum += local[q];
  }
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
    find_rank_bin(sh, rank);
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

// ---------------------------------------------------------------------------
// The same selection on n words staged in shared memory (16-byte aligned, room
// for a multiple of 4 words); key_of(word) gives the order key. Every pass
// reads 16 bytes per lane. Pass 0 builds the histogram of the top 11 bits;
// pass 1 the next 11 bits of the keys in the chosen bin, and it also lists
// those keys' positions in `cand` (up to cand_cap), so pass 2 scans only the
// candidates (all words again if the list overflowed). The output is written
// by two passes over contiguous per-warp ranges: per-lane counts, then one
// warp scan per 128 positions.

constexpr int kCandCap = 8192;

template <class KeyOf>
__device__ void smem_radix_select(const uint32_t* w, int n, int m, KeyOf key_of, SelectShared& sh,
                                  int* cand, uint32_t* T, int* need_eq) {
  const int t = threadIdx.x, lane = t & 31;
  const uint32_t below = (1u << lane) - 1u;
  const int n4 = n >> 2;
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  // pass 0: top 11 bits
  for (int b = t; b < kRadixBins; b += kSelectThreads) sh.hist[b] = 0;
  __syncthreads();
  for (int v = t; v < n4; v += kSelectThreads) {
    const uint4 u = w4[v];
    atomicAdd(&sh.hist[key_of(u.x) >> 21], 1u);
    atomicAdd(&sh.hist[key_of(u.y) >> 21], 1u);
    atomicAdd(&sh.hist[key_of(u.z) >> 21], 1u);
    atomicAdd(&sh.hist[key_of(u.w) >> 21], 1u);
  }
  for (int i = 4 * n4 + t; i < n; i += kSelectThreads) atomicAdd(&sh.hist[key_of(w[i]) >> 21], 1u);
  __syncthreads();
  find_rank_bin(sh, (uint32_t)m);
  const uint32_t b0 = sh.bcast[0];
  uint32_t rank = sh.bcast[1];
  __syncthreads();
  // pass 1: bits 10..20 of the keys in bin b0, and their positions
  for (int b = t; b < kRadixBins; b += kSelectThreads) sh.hist[b] = 0;
  if (t == 0) sh.bcast[2] = 0;
  __syncthreads();
  const int n_slots = (n + 3) >> 2;
  for (int base = 0; base < n_slots; base += kSelectThreads) {
    const int v = base + t;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (v < n_slots) u = w4[v];
    const uint32_t wq[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * v + q;
      const uint32_t k = key_of(wq[q]);
      const bool hit = i < n && (k >> 21) == b0;
      if (hit) atomicAdd(&sh.hist[(k >> 10) & 0x7ffu], 1u);
      const uint32_t bal = __ballot_sync(0xffffffffu, hit);
      if (bal) {
        uint32_t at = 0;
        if (lane == __ffs(bal) - 1) at = atomicAdd(&sh.bcast[2], (uint32_t)__popc(bal));
        at = __shfl_sync(0xffffffffu, at, __ffs(bal) - 1);
        const uint32_t pos = at + __popc(bal & below);
        if (hit && pos < (uint32_t)kCandCap) cand[pos] = i;
      }
    }
  }
  __syncthreads();
  const uint32_t n_cand = sh.bcast[2];
  find_rank_bin(sh, rank);
  const uint32_t prefix22 = (b0 << 11) | sh.bcast[0];  // top 22 bits
  rank = sh.bcast[1];
  __syncthreads();
  // pass 2: low 10 bits of the keys that share the top 22 bits
  for (int b = t; b < kRadixBins; b += kSelectThreads) sh.hist[b] = 0;
  __syncthreads();
  if (n_cand <= (uint32_t)kCandCap) {
    for (int c = t; c < (int)n_cand; c += kSelectThreads) {
      const uint32_t k = key_of(w[cand[c]]);
      if ((k >> 10) == prefix22) atomicAdd(&sh.hist[k & 0x3ffu], 1u);
    }
  } else {
    for (int i = t; i < n; i += kSelectThreads) {
      const uint32_t k = key_of(w[i]);
      if ((k >> 10) == prefix22) atomicAdd(&sh.hist[k & 0x3ffu], 1u);
    }
  }
  __syncthreads();
  find_rank_bin(sh, rank);
  *T = (prefix22 << 10) | sh.bcast[0];
  *need_eq = (int)sh.bcast[1];
  __syncthreads();
}

__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, int lane) {
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  return incl - v;
}

// Selects the m smallest keys among the n staged words (ties to the lower
// position), emitting sel(pos_in_selection, i) and rest(pos_in_rest, i) in
// position order. 0 <= m <= n.
template <class KeyOf, class SelFn, class RestFn>
__device__ void smem_select_ordered(const uint32_t* w, int n, int m, KeyOf key_of,
                                    SelectShared& sh, int* cand, SelFn sel, RestFn rest) {
  constexpr int W = kSelectThreads / 32;
  const bool take_all = (m >= n), take_none = (m <= 0);
  const bool cut = !take_all && !take_none;
  uint32_t T = 0;
  int need_eq = 0;
  if (cut) smem_radix_select(w, n, m, key_of, sh, cand, &T, &need_eq);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_slots = (n + 3) >> 2;
  const int seg = (n_slots + W - 1) / W;
  const int s0 = min(n_slots, warp * seg), s1 = min(n_slots, s0 + seg);
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  uint32_t sel_run = take_all ? (uint32_t)min(n, 4 * s0) : 0u, eq_run = 0;
  if (cut) {
    uint32_t c_lt = 0, c_eq = 0;
    for (int v = s0 + lane; v < s1; v += 32) {
      const uint4 u = w4[v];
      const uint32_t wq[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = 4 * v + q < n;
        const uint32_t k = key_of(wq[q]);
        c_lt += (valid && k < T) ? 1u : 0u;
        c_eq += (valid && k == T) ? 1u : 0u;
      }
    }
    c_lt = __reduce_add_sync(0xffffffffu, c_lt);
    c_eq = __reduce_add_sync(0xffffffffu, c_eq);
    if (lane == 0) {
      sh.warp_tot[warp] = c_lt;
      sh.warp_tot2[warp] = c_eq;
    }
    __syncthreads();
    uint32_t lt_before = 0;
    for (int w2 = 0; w2 < warp; ++w2) {
      lt_before += sh.warp_tot[w2];
      eq_run += sh.warp_tot2[w2];
    }
    sel_run = lt_before + min(eq_run, (uint32_t)need_eq);
  }
  for (int base = s0; base < s1; base += 32) {
    const int v = base + lane;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (v < s1) u = w4[v];
    const uint32_t wq[4] = {u.x, u.y, u.z, u.w};
    bool s[4];
    uint32_t cs = 0;
    if (cut) {
      bool lt[4], eq[4];
      uint32_t ce = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = v < s1 && 4 * v + q < n;
        const uint32_t k = key_of(wq[q]);
        lt[q] = valid && k < T;
        eq[q] = valid && k == T;
        ce += eq[q] ? 1u : 0u;
      }
      uint32_t eq_rank = eq_run;
      if (__any_sync(0xffffffffu, ce != 0)) {
        eq_rank += warp_excl_scan(ce, lane);
        eq_run += __reduce_add_sync(0xffffffffu, ce);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        s[q] = lt[q] || (eq[q] && eq_rank < (uint32_t)need_eq);
        eq_rank += eq[q] ? 1u : 0u;
        cs += s[q] ? 1u : 0u;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        s[q] = take_all && v < s1 && 4 * v + q < n;
        cs += s[q] ? 1u : 0u;
      }
    }
    uint32_t pos = sel_run + warp_excl_scan(cs, lane);
    sel_run += __reduce_add_sync(0xffffffffu, cs);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * v + q;
      if (v < s1 && i < n) {  // (the bounds hold by construction; they guard the writes)
        if (s[q]) {
          if (pos < (uint32_t)m) sel(pos, i);
          ++pos;
        } else if ((uint32_t)i - pos < (uint32_t)(n - m)) {
          rest((uint32_t)i - pos, i);
        }
      }
    }
  }
}

}  // namespace tlsp
