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
// memory (HBM the first time, L2 after), so a CTA needs little shared memory
// and several run on each SM, hiding each other's latencies.
//
// Keys are the complemented order keys of the scores (largest score =
// smallest key) and the selection is "the k smallest keys". Per row:
//   1. histogram of the top 11 key bits -> the bin b0 holding the k-th key;
//   2. each warp scans a contiguous segment of the row, counts its keys in
//      bins below b0 (all selected) and appends the keys of bin b0 (the
//      candidates) with their positions to a shared list;
//   3. two radix passes (11 + 10 bits) over the candidate list give the
//      exact k-th key T and how many keys equal to T are taken (the ones at
//      the lowest positions);
//   4. each warp writes its selected positions in order, its starting offset
//      coming from the per-warp counts.
// When bin b0 holds more candidates than the list does (a very flat row),
// step 3 streams the row instead, and the per-warp counts come from one more
// pass over it: the same result, more slowly.

constexpr int kStreamThreads = 256;
constexpr int kStreamWarps = kStreamThreads / 32;
constexpr int kStreamCtasPerSm = 4;
constexpr int kCandCap = 3072;

struct StreamShared {
  uint32_t hist[kRadixBins];
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

// Bin of sh.hist where the running count reaches `rank` (1-based) ->
// sh.bcast = {bin, rank within the bin}. Starts and ends with a barrier.
__device__ __forceinline__ void stream_rank_bin(StreamShared& sh, uint32_t rank) {
  constexpr int per = kRadixBins / kStreamThreads;
  __syncthreads();
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
  if (lane == 31) sh.scan[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp; ++w) before += sh.scan[w];
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

__global__ void __launch_bounds__(kStreamThreads, kStreamCtasPerSm)
topk_stream_kernel(const float* __restrict__ scores, int64_t rows, int n_kv, int k,
                   int32_t* __restrict__ indices) {
  __shared__ StreamShared sh;
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
    // 1. histogram of the top 11 bits
    for (int b = t; b < kRadixBins; b += kStreamThreads) sh.hist[b] = 0;
    if (t == 0) sh.n_cand = 0;
    __syncthreads();
    for (int i = 4 * t; i < n; i += 4 * kStreamThreads) {
      uint32_t k4[4];
      load_keys4(row, i, n, vec, k4);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (i + q < n) atomicAdd(&sh.hist[k4[q] >> 21], 1u);
    }
    stream_rank_bin(sh, m);
    const uint32_t b0 = sh.bcast[0], r0 = sh.bcast[1];
    // 2. per-warp count below b0, candidates of bin b0 to the list
    uint32_t lt = 0;
    for (int base = s0; base < s1; base += 128) {
      const int i = base + 4 * lane;
      uint32_t k4[4];
      load_keys4(row, i, s1, vec, k4);
      uint32_t eqb[4], n_eq = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = i + q < s1;
        lt += (valid && (k4[q] >> 21) < b0) ? 1u : 0u;
        eqb[q] = __ballot_sync(0xffffffffu, valid && (k4[q] >> 21) == b0);
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
              sh.cand_key[slot] = k4[q];
              sh.cand_pos[slot] = i + q;
            }
          }
          off += __popc(eqb[q]);
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
    // 3. the exact k-th key T below bin b0's prefix: bits 20..10, then 9..0
    uint32_t prefix = b0, rank = r0;
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 21 : 10;  // keys match when key >> shift == prefix
      const int dshift = pass == 0 ? 10 : 0;
      const uint32_t dmask = pass == 0 ? 0x7ffu : 0x3ffu;
      for (int b = t; b < kRadixBins; b += kStreamThreads) sh.hist[b] = 0;
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
      stream_rank_bin(sh, rank);
      prefix = (prefix << (pass == 0 ? 11 : 10)) | sh.bcast[0];
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
          c_lt += (valid && (k4[q] >> 21) == b0 && k4[q] < T) ? 1u : 0u;
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
    for (int base = s0; base < s1; base += 128) {
      const int i = base + 4 * lane;
      uint32_t k4[4];
      load_keys4(row, i, s1, vec, k4);
      bool s[4], eq[4], any_eq = false;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = i + q < s1;
        s[q] = valid && k4[q] < T;
        eq[q] = valid && k4[q] == T;
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

int launch_topk(const float* scores, int64_t rows, int n_kv, int k, int32_t* indices,
                int* status, cudaStream_t stream) {
  (void)status;  // the streaming kernel has no waits to time out
  if (rows == 0) return TLSP_OK;
  const int64_t grid = std::min<int64_t>(rows, (int64_t)kStreamCtasPerSm * device_sm_count());
  topk_stream_kernel<<<(unsigned)grid, kStreamThreads, 0, stream>>>(scores, rows, n_kv, k,
                                                                   indices);
  return check_launch();
}

int launch_split(const float* proj, const int32_t* members, int n, int n_left, int32_t* left,
                 int32_t* right, cudaStream_t stream) {
  split_kernel<<<1, kSelectThreads, 0, stream>>>(proj, members, n, n_left, left, right);
  return check_launch();
}

}  // namespace tlsp
