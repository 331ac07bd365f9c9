// Token-level KV selection (per-group top-k) and the single PDDP cut hook.
//
// MC-Sparse review, section 3: each query group keeps the individual KV
// tokens of highest exact score, not whole blocks. Ties go to the lower key
// index and the kept set is listed in ascending key order.
#include <algorithm>

#include "kernels.h"
#include "select.cuh"

namespace tlsp {

// ---------------------------------------------------------------------------
// Streaming top-k: the k largest of each score row (ties to the lower index),
// listed in ascending key order. Every pass streams the row from global
// memory (HBM or L2), so a CTA needs little shared memory and several run on
// each SM, hiding each other's latencies.
//
// Keys are the complemented order keys of the scores (largest score =
// smallest key) and the selection is "the k smallest keys". Per row:
//   1. histogram of the top 13 key bits -> the bin b0 holding the k-th key
//      (13 bits: group scores of attention rows span about an octave, and a
//      bin of 1/16 octave holds a few hundred of 32K keys);
//   2. each warp scans a contiguous segment of the row, counts its keys in
//      bins below b0 (all selected) and appends the keys of bin b0 (the
//      candidates) with their positions to a shared list;
//   3. two radix passes (10 + 9 bits) over the candidate list give the
//      exact k-th key T and how many keys equal to T are taken (the ones at
//      the lowest positions);
//   4. each warp writes its selected positions in order, its starting offset
//      coming from the per-warp counts.
// When bin b0 holds more candidates than the list does (a flat row, ties),
// step 3 streams the row instead, and the per-warp counts come from one more
// pass over it: the same result, more slowly.

constexpr int kStreamThreads = 256;
constexpr int kStreamWarps = kStreamThreads / 32;
constexpr int kStreamCtasPerSm = 4;
constexpr int kBins0 = 8192;  // first pass: key bits 31..19
constexpr int kCandCap = 2048;
constexpr int kStreamUnroll = 4;  // 16-byte loads in flight per thread in every pass

struct StreamShared {
  uint32_t hist[kBins0];
  uint32_t cand_key[kCandCap];
  int32_t cand_pos[kCandCap];
  uint32_t warp_lt[kStreamWarps], warp_eq[kStreamWarps];
  uint32_t scan[kStreamWarps];
  uint32_t bcast[2];
  uint32_t n_cand;
};

__device__ __forceinline__ uint32_t topk_key(float f) {
  // largest score first == smallest complemented order key
  return ~float_order_key(f);
}

// Bin of sh.hist[0 .. nbins) where the running count reaches `rank`
// (1-based) -> sh.bcast = {bin, rank within the bin}. Thread t owns bins
// t * nbins / 256 .. (t + 1) * nbins / 256 - 1. Starts and ends with a barrier.
__device__ __forceinline__ void stream_rank_bin(StreamShared& sh, int nbins, uint32_t rank) {
  const int per = nbins / kStreamThreads;
  const int b0 = threadIdx.x * per;
  __syncthreads();
  uint32_t lsum = 0;
  for (int q = 0; q < per; ++q) lsum += sh.hist[b0 + q];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh.scan[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp; ++w) before += sh.scan[w];
  const uint32_t excl = before + incl - lsum;
  if (excl < rank && rank <= excl + lsum) {
    uint32_t run = excl;
    for (int q = 0; q < per; ++q) {
      const uint32_t c = sh.hist[b0 + q];
      if (run < rank && rank <= run + c) {
        sh.bcast[0] = (uint32_t)(b0 + q);
        sh.bcast[1] = rank - run;
      }
      run += c;
    }
  }
  __syncthreads();
}

// Four consecutive keys of the row starting at position i (a multiple of 4);
// positions at or past n read as the largest key (never selected). `vec`:
// the row is 16-byte aligned and n is a multiple of 4.
__device__ __forceinline__ void load_keys4(const float* row, int i, int n, bool vec,
                                           uint32_t (&k4)[4]) {
  if (vec && i + 3 < n) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(row + i));
    k4[0] = topk_key(f.x);
    k4[1] = topk_key(f.y);
    k4[2] = topk_key(f.z);
    k4[3] = topk_key(f.w);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) k4[q] = i + q < n ? topk_key(__ldg(row + i + q)) : 0xffffffffu;
  }
}

// Dynamic shared memory: one StreamShared.
__global__ void __launch_bounds__(kStreamThreads, kStreamCtasPerSm)
topk_stream_kernel(const float* __restrict__ scores, int64_t rows, int n_kv, int k,
                   int32_t* __restrict__ indices) {
  extern __shared__ __align__(16) uint8_t stream_smem[];
  StreamShared& sh = *reinterpret_cast<StreamShared*>(stream_smem);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int n = n_kv;
  const uint32_t m = (uint32_t)k;
  // each warp's contiguous segment: whole 128-position blocks
  const int seg = (n + kStreamWarps * 128 - 1) / (kStreamWarps * 128) * 128;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* row = scores + r * (int64_t)n;
    int32_t* out = indices + r * (int64_t)k;
    const bool vec = (n % 4) == 0 && (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
    if (m >= (uint32_t)n) {  // every key
      for (int i = t; i < n; i += kStreamThreads) out[i] = i;
      continue;
    }
    // 1. histogram of the top 13 bits
    for (int b = t; b < kBins0; b += kStreamThreads) sh.hist[b] = 0;
    if (t == 0) sh.n_cand = 0;
    __syncthreads();
    for (int i0 = 4 * t; i0 < n; i0 += 4 * kStreamThreads * kStreamUnroll) {
      uint32_t kk[kStreamUnroll][4];
#pragma unroll
      for (int u = 0; u < kStreamUnroll; ++u)
        load_keys4(row, i0 + 4 * kStreamThreads * u, n, vec, kk[u]);
#pragma unroll
      for (int u = 0; u < kStreamUnroll; ++u)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (i0 + 4 * kStreamThreads * u + q < n) atomicAdd(&sh.hist[kk[u][q] >> 19], 1u);
    }
    stream_rank_bin(sh, kBins0, m);
    const uint32_t b0 = sh.bcast[0], r0 = sh.bcast[1];
    // 2. per-warp count below b0, candidates of bin b0 to the list
    uint32_t lt = 0;
    for (int base0 = s0; base0 < s1; base0 += 128 * kStreamUnroll) {
      uint32_t kk[kStreamUnroll][4];
#pragma unroll
      for (int u = 0; u < kStreamUnroll; ++u)
        load_keys4(row, base0 + 128 * u + 4 * lane, s1, vec, kk[u]);
#pragma unroll
      for (int u = 0; u < kStreamUnroll; ++u) {
        const int i = base0 + 128 * u + 4 * lane;
        uint32_t eqb[4], n_eq = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool valid = i + q < s1;
          lt += (valid && (kk[u][q] >> 19) < b0) ? 1u : 0u;
          eqb[q] = __ballot_sync(0xffffffffu, valid && (kk[u][q] >> 19) == b0);
          n_eq += __popc(eqb[q]);
        }
        if (n_eq) {
          uint32_t off = 0;
          if (lane == 0) off = atomicAdd(&sh.n_cand, n_eq);
          off = __shfl_sync(0xffffffffu, off, 0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (eqb[q] >> lane & 1u) {
              const uint32_t slot = off + __popc(eqb[q] & below);
              if (slot < (uint32_t)kCandCap) {
                sh.cand_key[slot] = kk[u][q];
                sh.cand_pos[slot] = i + q;
              }
            }
            off += __popc(eqb[q]);
          }
        }
      }
    }
    lt = __reduce_add_sync(0xffffffffu, lt);
    if (lane == 0) {
      sh.warp_lt[warp] = lt;
      sh.warp_eq[warp] = 0;
    }
    __syncthreads();
    const uint32_t n_cand = sh.n_cand;
    const bool listed = n_cand <= (uint32_t)kCandCap;
    // 3. the exact k-th key T below bin b0's prefix: bits 18..9, then 8..0
    uint32_t prefix = b0, rank = r0;
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 19 : 9;  // keys match when key >> shift == prefix
      const int dshift = pass == 0 ? 9 : 0;
      const int nbins = pass == 0 ? 1024 : 512;
      const uint32_t dmask = (uint32_t)nbins - 1u;
      for (int b = t; b < nbins; b += kStreamThreads) sh.hist[b] = 0;
      __syncthreads();
      if (listed) {
        for (uint32_t c = t; c < n_cand; c += kStreamThreads) {
          const uint32_t key = sh.cand_key[c];
          if ((key >> shift) == prefix) atomicAdd(&sh.hist[(key >> dshift) & dmask], 1u);
        }
      } else {
        for (int i = 4 * t; i < n; i += 4 * kStreamThreads) {
          uint32_t k4[4];
          load_keys4(row, i, n, vec, k4);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (i + q < n && (k4[q] >> shift) == prefix)
              atomicAdd(&sh.hist[(k4[q] >> dshift) & dmask], 1u);
        }
      }
      stream_rank_bin(sh, nbins, rank);
      prefix = (prefix << (pass == 0 ? 10 : 9)) | sh.bcast[0];
      rank = sh.bcast[1];
    }
    const uint32_t T = prefix, need_eq = rank;
    // per-warp counts of keys below T and equal to T
    if (listed) {
      for (uint32_t c = t; c < n_cand; c += kStreamThreads) {
        const uint32_t key = sh.cand_key[c];
        const int w = sh.cand_pos[c] / seg;
        if (key < T) atomicAdd(&sh.warp_lt[w], 1u);
        else if (key == T) atomicAdd(&sh.warp_eq[w], 1u);
      }
    } else {
      uint32_t c_lt = 0, c_eq = 0;
      for (int base = s0; base < s1; base += 128) {
        const int i = base + 4 * lane;
        uint32_t k4[4];
        load_keys4(row, i, s1, vec, k4);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool valid = i + q < s1;
          c_lt += (valid && (k4[q] >> 19) == b0 && k4[q] < T) ? 1u : 0u;
          c_eq += (valid && k4[q] == T) ? 1u : 0u;
        }
      }
      c_lt = __reduce_add_sync(0xffffffffu, c_lt);
      c_eq = __reduce_add_sync(0xffffffffu, c_eq);
      if (lane == 0) {
        sh.warp_lt[warp] += c_lt;
        sh.warp_eq[warp] = c_eq;
      }
    }
    __syncthreads();
    // 4. ordered write-out of this warp's segment
    uint32_t lt_before = 0, eq_run = 0;
    for (int w = 0; w < warp; ++w) {
      lt_before += sh.warp_lt[w];
      eq_run += sh.warp_eq[w];
    }
    uint32_t sel_run = lt_before + min(eq_run, need_eq);
    for (int base0 = s0; base0 < s1; base0 += 128 * kStreamUnroll) {
      uint32_t kk[kStreamUnroll][4];
#pragma unroll
      for (int u = 0; u < kStreamUnroll; ++u)
        load_keys4(row, base0 + 128 * u + 4 * lane, s1, vec, kk[u]);
#pragma unroll
      for (int u = 0; u < kStreamUnroll; ++u) {
        const int i = base0 + 128 * u + 4 * lane;
        bool s[4], eq[4], any_eq = false;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool valid = i + q < s1;
          s[q] = valid && kk[u][q] < T;
          eq[q] = valid && kk[u][q] == T;
          any_eq |= eq[q];
        }
        if (__any_sync(0xffffffffu, any_eq)) {  // ties at the threshold: the earliest are taken
          uint32_t eb[4], er = eq_run;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            eb[q] = __ballot_sync(0xffffffffu, eq[q]);
            er += __popc(eb[q] & below);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            s[q] = s[q] || (eq[q] && er < need_eq);
            er += eq[q] ? 1u : 0u;
            eq_run += __popc(eb[q]);
          }
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
          if (s[q]) {
            if (pos < m) out[pos] = i + q;  // (holds by construction; guards the write)
            ++pos;
          }
        }
      }
    }
    __syncthreads();  // shared state is reset for the next row
  }
}

// One PDDP cut of `members` (ascending token ids) on projections proj[token].
__global__ void __launch_bounds__(kSelectThreads)
split_kernel(const float* __restrict__ proj, const int32_t* __restrict__ members, int n,
             int n_left, int32_t* __restrict__ left, int32_t* __restrict__ right) {
  __shared__ SelectShared sh;
  auto key = [&](int i) -> uint32_t { return float_order_key(__ldg(proj + members[i])); };
  select_smallest_ordered(
      key, n, n_left, sh, [&](uint32_t pos, int i) { left[pos] = members[i]; },
      [&](uint32_t pos, int i) { right[pos] = members[i]; });
}

// ---------------------------------------------------------------------------
// Top-k with the row's key bins kept in shared memory: the row is read from
// global memory once. Same keys, bins and selection rule as the streaming
// kernel above; used when the row's 16-bit bins fit in shared memory.
//   A. one pass over the row: the histogram of the top 13 key bits, and each
//      key's 13-bit bin stored as 16 bits -> the bin b0 of the k-th key;
//   B. each warp scans its segment of the stored bins: counts bins below b0
//      and lists the positions in bin b0 (the candidates);
//   C. the candidates' full keys are read again (a few hundred, all at once),
//      two radix passes over them give T and how many keys equal to T are
//      taken, and each candidate's stored bin is replaced by a code (below,
//      equal to or above T);
//   D. each warp writes its selected positions in order from the stored bins.
// When bin b0 holds more keys than the candidate list, C streams the row.

constexpr int kBinThreads = 512;
constexpr int kBinWarps = kBinThreads / 32;
constexpr int kBinCandCap = 1024;
constexpr int kBinUnroll = 4;                 // 16-byte loads in flight per thread in pass A
constexpr uint16_t kCodeLt = 0xFFFD;          // candidate key below T (selected)
constexpr uint16_t kCodeEq = 0xFFFE;          // candidate key equal to T (ties: lowest positions)
constexpr uint16_t kCodeGt = 0xFFFF;          // above T, or past the row (not selected)
constexpr int kBinsMaxN = 94208;              // longest row whose bins fit beside the rest

struct BinShared {
  uint32_t hist[kBins0];
  uint32_t cand_key[kBinCandCap];
  int32_t cand_pos[kBinCandCap];
  uint32_t warp_lt[kBinWarps], warp_eq[kBinWarps];
  uint32_t scan[kBinWarps];
  uint32_t bcast[2];
  uint32_t n_cand;
};
constexpr size_t kBinsOffset = (sizeof(BinShared) + 15) / 16 * 16;  // the bins, 16-byte aligned

size_t topk_bins_smem(int n_kv) { return kBinsOffset + (size_t)(n_kv + 7) / 8 * 16; }

// Bin of h[0 .. nbins) where the running count reaches `rank` (1-based) ->
// bcast = {bin, rank within the bin}. Thread t owns bins t * per .. and
// sums them starting at a different one per lane, so a warp's reads fall in
// 32 different banks. Starts and ends with a barrier.
__device__ __forceinline__ void bins_rank(const uint32_t* h, int nbins, uint32_t rank,
                                          uint32_t* scan, uint32_t* bcast) {
  const int per = nbins / kBinThreads;
  const int b0 = threadIdx.x * per;
  __syncthreads();
  uint32_t lsum = 0;
  for (int q = 0; q < per; ++q) lsum += h[b0 + (q + threadIdx.x) % per];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp; ++w) before += scan[w];
  const uint32_t excl = before + incl - lsum;
  if (excl < rank && rank <= excl + lsum) {
    uint32_t run = excl;
    for (int q = 0; q < per; ++q) {
      const uint32_t c = h[b0 + q];
      if (run < rank && rank <= run + c) {
        bcast[0] = (uint32_t)(b0 + q);
        bcast[1] = rank - run;
      }
      run += c;
    }
  }
  __syncthreads();
}

// Exclusive prefix of v over the lanes of the warp.
__device__ __forceinline__ uint32_t warp_excl(uint32_t v, int lane) {
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  return incl - v;
}

// Dynamic shared memory: a BinShared, then the 16-bit bins of the row.
__global__ void __launch_bounds__(kBinThreads, 2)
topk_bins_kernel(const float* __restrict__ scores, int64_t rows, int n_kv, int k,
                 int32_t* __restrict__ indices) {
  extern __shared__ __align__(16) uint8_t bins_smem[];
  BinShared& sh = *reinterpret_cast<BinShared*>(bins_smem);
  uint16_t* bins = reinterpret_cast<uint16_t*>(bins_smem + kBinsOffset);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int n = n_kv;
  const int n8 = (n + 7) / 8 * 8;
  const uint32_t m = (uint32_t)k;
  // each warp's contiguous segment of positions: whole 256-position blocks
  const int seg = (n8 + kBinWarps * 256 - 1) / (kBinWarps * 256) * 256;
  const int s0 = min(n8, warp * seg), s1 = min(n8, s0 + seg);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* row = scores + r * (int64_t)n;
    int32_t* out = indices + r * (int64_t)k;
    const bool vec = (n % 4) == 0 && (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
    if (m >= (uint32_t)n) {  // every key
      for (int i = t; i < n; i += kBinThreads) out[i] = i;
      continue;
    }
    // A. histogram of the top 13 bits, bins to shared memory
    for (int b = t; b < kBins0; b += kBinThreads) sh.hist[b] = 0;
    if (t == 0) sh.n_cand = 0;
    __syncthreads();
    for (int i0 = 4 * t; i0 < n8; i0 += 4 * kBinThreads * kBinUnroll) {
      uint32_t kk[kBinUnroll][4];
#pragma unroll
      for (int u = 0; u < kBinUnroll; ++u)
        load_keys4(row, i0 + 4 * kBinThreads * u, n, vec, kk[u]);
#pragma unroll
      for (int u = 0; u < kBinUnroll; ++u) {
        const int i = i0 + 4 * kBinThreads * u;
        if (i < n8) {
          uint32_t b16[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (i + q < n) {
              b16[q] = kk[u][q] >> 19;
              atomicAdd(&sh.hist[b16[q]], 1u);
            } else {
              b16[q] = kCodeGt;
            }
          }
          *reinterpret_cast<uint2*>(bins + i) = make_uint2(b16[0] | (b16[1] << 16),
                                                          b16[2] | (b16[3] << 16));
        }
      }
    }
    bins_rank(sh.hist, kBins0, m, sh.scan, sh.bcast);
    const uint32_t b0 = sh.bcast[0], r0 = sh.bcast[1];
    // B. per-warp count below b0; positions of bin b0 to the candidate list
    uint32_t lt = 0;
    for (int base = s0; base < s1; base += 256) {
      // s1 is a multiple of 8: a lane's 8 bins are all inside the segment or
      // all past it (then they read as never selected, and nothing is loaded)
      const int i = base + 8 * lane;
      const uint4 v = i < s1 ? *reinterpret_cast<const uint4*>(bins + i)
                             : make_uint4(~0u, ~0u, ~0u, ~0u);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t eq_mask = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t b = (w[q >> 1] >> (16 * (q & 1))) & 0xffffu;
        lt += b < b0 ? 1u : 0u;
        eq_mask |= (b == b0 ? 1u : 0u) << q;
      }
      const uint32_t c = __popc(eq_mask);
      const uint32_t tot = __reduce_add_sync(0xffffffffu, c);
      if (tot) {
        uint32_t off = 0;
        if (lane == 0) off = atomicAdd(&sh.n_cand, tot);
        off = __shfl_sync(0xffffffffu, off, 0) + warp_excl(c, lane);
        for (int q = 0; q < 8; ++q) {
          if (eq_mask >> q & 1u) {
            if (off < (uint32_t)kBinCandCap) sh.cand_pos[off] = i + q;
            ++off;
          }
        }
      }
    }
    lt = __reduce_add_sync(0xffffffffu, lt);
    if (lane == 0) {
      sh.warp_lt[warp] = lt;
      sh.warp_eq[warp] = 0;
    }
    __syncthreads();
    const uint32_t n_cand = sh.n_cand;
    const bool listed = n_cand <= (uint32_t)kBinCandCap;
    // C. the exact k-th key T: candidates' keys, bits 18..9, then 8..0
    if (listed)
      for (uint32_t c = t; c < n_cand; c += kBinThreads)
        sh.cand_key[c] = topk_key(__ldg(row + sh.cand_pos[c]));
    uint32_t prefix = b0, rank = r0;
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 19 : 9;  // keys match when key >> shift == prefix
      const int dshift = pass == 0 ? 9 : 0;
      const int nbins = pass == 0 ? 1024 : 512;
      const uint32_t dmask = (uint32_t)nbins - 1u;
      __syncthreads();
      for (int b = t; b < nbins; b += kBinThreads) sh.hist[b] = 0;
      __syncthreads();
      if (listed) {
        for (uint32_t c = t; c < n_cand; c += kBinThreads) {
          const uint32_t key = sh.cand_key[c];
          if ((key >> shift) == prefix) atomicAdd(&sh.hist[(key >> dshift) & dmask], 1u);
        }
      } else {
        for (int i = 4 * t; i < n; i += 4 * kBinThreads) {
          uint32_t k4[4];
          load_keys4(row, i, n, vec, k4);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (i + q < n && (k4[q] >> shift) == prefix)
              atomicAdd(&sh.hist[(k4[q] >> dshift) & dmask], 1u);
        }
      }
      bins_rank(sh.hist, nbins, rank, sh.scan, sh.bcast);
      prefix = (prefix << (pass == 0 ? 10 : 9)) | sh.bcast[0];
      rank = sh.bcast[1];
    }
    const uint32_t T = prefix, need_eq = rank;
    // codes for the keys of bin b0, and the per-warp counts below / equal to T
    if (listed) {
      for (uint32_t c = t; c < n_cand; c += kBinThreads) {
        const uint32_t key = sh.cand_key[c];
        const int pos = sh.cand_pos[c];
        const uint16_t code = key < T ? kCodeLt : key == T ? kCodeEq : kCodeGt;
        bins[pos] = code;
        if (code == kCodeLt) atomicAdd(&sh.warp_lt[pos / seg], 1u);
        else if (code == kCodeEq) atomicAdd(&sh.warp_eq[pos / seg], 1u);
      }
    } else {
      uint32_t c_lt = 0, c_eq = 0;
      for (int i = s0 + lane; i < min(s1, n); i += 32) {
        if (bins[i] == b0) {
          const uint32_t key = topk_key(__ldg(row + i));
          const uint16_t code = key < T ? kCodeLt : key == T ? kCodeEq : kCodeGt;
          bins[i] = code;
          c_lt += code == kCodeLt ? 1u : 0u;
          c_eq += code == kCodeEq ? 1u : 0u;
        }
      }
      c_lt = __reduce_add_sync(0xffffffffu, c_lt);
      c_eq = __reduce_add_sync(0xffffffffu, c_eq);
      if (lane == 0) {
        sh.warp_lt[warp] += c_lt;
        sh.warp_eq[warp] = c_eq;
      }
    }
    __syncthreads();
    // D. ordered write-out of this warp's segment
    uint32_t lt_before = 0, eq_run = 0;
    for (int w = 0; w < warp; ++w) {
      lt_before += sh.warp_lt[w];
      eq_run += sh.warp_eq[w];
    }
    uint32_t sel_run = lt_before + min(eq_run, need_eq);
    for (int base = s0; base < s1; base += 256) {
      const int i = base + 8 * lane;
      const uint4 v = i < s1 ? *reinterpret_cast<const uint4*>(bins + i)
                             : make_uint4(~0u, ~0u, ~0u, ~0u);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t sel_mask = 0, eq_mask = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t b = (w[q >> 1] >> (16 * (q & 1))) & 0xffffu;
        sel_mask |= (b < b0 || b == kCodeLt ? 1u : 0u) << q;
        eq_mask |= (b == kCodeEq ? 1u : 0u) << q;
      }
      if (__any_sync(0xffffffffu, eq_mask != 0)) {  // ties at T: the earliest are taken
        uint32_t er = eq_run + warp_excl(__popc(eq_mask), lane);
        for (int q = 0; q < 8; ++q) {
          if (eq_mask >> q & 1u) {
            if (er < need_eq) sel_mask |= 1u << q;
            ++er;
          }
        }
        eq_run += __reduce_add_sync(0xffffffffu, __popc(eq_mask));
      }
      const uint32_t c = __popc(sel_mask);
      uint32_t pos = sel_run + warp_excl(c, lane);
      sel_run += __reduce_add_sync(0xffffffffu, c);
      for (int q = 0; q < 8; ++q) {
        if (sel_mask >> q & 1u) {
          if (pos < m) out[pos] = i + q;  // (holds by construction; guards the write)
          ++pos;
        }
      }
    }
    __syncthreads();  // shared state is reset for the next row
  }
}

int launch_topk(const float* scores, int64_t rows, int n_kv, int k, int32_t* indices,
                int* status, cudaStream_t stream) {
  (void)status;  // the selection kernels have no waits to time out
  if (rows == 0) return TLSP_OK;
  const int sms = device_sm_count();
  if (n_kv <= kBinsMaxN) {
    const size_t smem = topk_bins_smem(n_kv);
    TLSP_TRY(ensure_smem_limit((const void*)topk_bins_kernel, (int)topk_bins_smem(kBinsMaxN)));
    // as many CTAs as fit on an SM (228 KB, 1 KB of it reserved per CTA)
    const int per_sm = std::max(1, (int)((228u << 10) / (smem + 1024)));
    const int64_t grid = std::min<int64_t>(rows, (int64_t)per_sm * sms);
    topk_bins_kernel<<<(unsigned)grid, kBinThreads, smem, stream>>>(scores, rows, n_kv, k,
                                                                   indices);
    return check_launch();
  }
  TLSP_TRY(ensure_smem_limit((const void*)topk_stream_kernel, (int)sizeof(StreamShared)));
  const int64_t grid = std::min<int64_t>(rows, (int64_t)kStreamCtasPerSm * sms);
  topk_stream_kernel<<<(unsigned)grid, kStreamThreads, sizeof(StreamShared), stream>>>(
      scores, rows, n_kv, k, indices);
  return check_launch();
}

int launch_split(const float* proj, const int32_t* members, int n, int n_left, int32_t* left,
                 int32_t* right, cudaStream_t stream) {
  split_kernel<<<1, kSelectThreads, 0, stream>>>(proj, members, n, n_left, left, right);
  return check_launch();
}

}  // namespace tlsp
