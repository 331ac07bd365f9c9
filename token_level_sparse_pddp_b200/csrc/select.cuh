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
// (1-based): sh.bcast[0] = bin, sh.bcast[1] = rank within that bin. Each of
// the block's NT threads (at most kSelectThreads) owns kRadixBins / NT
// consecutive bins; a block scan of the per-thread sums finds the owner. Ends
// with a barrier.
template <int NT = kSelectThreads>
__device__ __forceinline__ void find_rank_bin(SelectShared& sh, uint32_t rank) {
  static_assert(NT % 32 == 0 && NT <= kSelectThreads && kRadixBins % NT == 0, "block size");
  constexpr int per = kRadixBins / NT;
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
// for a multiple of 4 words). Every pass reads 16 bytes per lane. Pass 0
// replaces each word by its order key key_of(word) in place and builds the
// histogram of the top 11 bits; passes 1 and 2 scan the keys again and count
// only those that share the prefix found so far. The output is written by two
// passes over contiguous per-warp ranges: per-lane counts, then, per 128
// positions, four ballots whose popcounts give every member its offset.

template <int NT, class KeyOf>
__device__ void smem_radix_select(uint32_t* w, int n, int m, KeyOf key_of, SelectShared& sh,
                                  uint32_t* T, int* need_eq) {
  const int t = threadIdx.x;
  const int n4 = n >> 2;
  uint4* w4 = reinterpret_cast<uint4*>(w);
  for (int b = t; b < kRadixBins; b += NT) sh.hist[b] = 0;
  __syncthreads();
  for (int v = t; v < n4; v += NT) {
    uint4 u = w4[v];
    u.x = key_of(u.x);
    u.y = key_of(u.y);
    u.z = key_of(u.z);
    u.w = key_of(u.w);
    w4[v] = u;
    atomicAdd(&sh.hist[u.x >> 21], 1u);
    atomicAdd(&sh.hist[u.y >> 21], 1u);
    atomicAdd(&sh.hist[u.z >> 21], 1u);
    atomicAdd(&sh.hist[u.w >> 21], 1u);
  }
  for (int i = 4 * n4 + t; i < n; i += NT) {
    w[i] = key_of(w[i]);
    atomicAdd(&sh.hist[w[i] >> 21], 1u);
  }
  __syncthreads();
  find_rank_bin<NT>(sh, (uint32_t)m);
  uint32_t prefix = sh.bcast[0];  // top 11 bits
  uint32_t rank = sh.bcast[1];
  __syncthreads();
  for (int pass = 1; pass < 3; ++pass) {
    const int shift = pass == 1 ? 21 : 10;  // keys match when k >> shift == prefix
    const int dshift = pass == 1 ? 10 : 0;
    const uint32_t dmask = pass == 1 ? 0x7ffu : 0x3ffu;
    for (int b = t; b < kRadixBins; b += NT) sh.hist[b] = 0;
    __syncthreads();
    for (int v = t; v < n4; v += NT) {
      const uint4 u = w4[v];
      if ((u.x >> shift) == prefix) atomicAdd(&sh.hist[(u.x >> dshift) & dmask], 1u);
      if ((u.y >> shift) == prefix) atomicAdd(&sh.hist[(u.y >> dshift) & dmask], 1u);
      if ((u.z >> shift) == prefix) atomicAdd(&sh.hist[(u.z >> dshift) & dmask], 1u);
      if ((u.w >> shift) == prefix) atomicAdd(&sh.hist[(u.w >> dshift) & dmask], 1u);
    }
    for (int i = 4 * n4 + t; i < n; i += NT)
      if ((w[i] >> shift) == prefix) atomicAdd(&sh.hist[(w[i] >> dshift) & dmask], 1u);
    __syncthreads();
    find_rank_bin<NT>(sh, rank);
    prefix = (prefix << (pass == 1 ? 11 : 10)) | sh.bcast[0];
    rank = sh.bcast[1];
    __syncthreads();
  }
  *T = prefix;
  *need_eq = (int)rank;
}

// Selects the m smallest keys among the n staged words (ties to the lower
// position), emitting sel(pos_in_selection, i) and rest(pos_in_rest, i) in
// position order. 0 <= m <= n. The words are replaced by their keys. NT is the
// block's thread count (a multiple of 32, at most kSelectThreads); the result
// does not depend on it.
template <int NT = kSelectThreads, class KeyOf, class SelFn, class RestFn>
__device__ void smem_select_ordered(uint32_t* w, int n, int m, KeyOf key_of, SelectShared& sh,
                                    SelFn sel, RestFn rest) {
  constexpr int W = NT / 32;
  const bool take_all = (m >= n), take_none = (m <= 0);
  const bool cut = !take_all && !take_none;
  uint32_t T = 0;
  int need_eq = 0;
  if (cut) smem_radix_select<NT>(w, n, m, key_of, sh, &T, &need_eq);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int n_slots = (n + 3) >> 2;
  const int seg = (n_slots + W - 1) / W;
  const int s0 = min(n_slots, warp * seg), s1 = min(n_slots, s0 + seg);
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  uint32_t sel_run = take_all ? (uint32_t)min(n, 4 * s0) : 0u, eq_run = 0;
  if (cut) {
    uint32_t c_lt = 0, c_eq = 0;
    for (int v = s0 + lane; v < s1; v += 32) {
      const uint4 u = w4[v];
      const uint32_t k4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = 4 * v + q < n;
        c_lt += (valid && k4[q] < T) ? 1u : 0u;
        c_eq += (valid && k4[q] == T) ? 1u : 0u;
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
    const uint32_t k4[4] = {u.x, u.y, u.z, u.w};
    bool s[4];
    if (cut) {
      bool eq[4];
      bool any_eq = false;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = v < s1 && 4 * v + q < n;
        s[q] = valid && k4[q] < T;
        eq[q] = valid && k4[q] == T;
        any_eq |= eq[q];
      }
      if (__any_sync(0xffffffffu, any_eq)) {  // ties at the threshold: take the earliest
        uint32_t eb[4], rank = eq_run;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          eb[q] = __ballot_sync(0xffffffffu, eq[q]);
          rank += __popc(eb[q] & below);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          s[q] = s[q] || (eq[q] && rank < (uint32_t)need_eq);
          rank += eq[q] ? 1u : 0u;
          eq_run += __popc(eb[q]);
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) s[q] = take_all && v < s1 && 4 * v + q < n;
    }
    uint32_t pos = sel_run;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t sb = __ballot_sync(0xffffffffu, s[q]);
      pos += __popc(sb & below);
      sel_run += __popc(sb);
    }
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
