// Tile-aligned query grouping by fast PDDP (principal direction divisive
// partitioning), MC-Sparse review section 3: similar queries are grouped
// into equal-size, tile-aligned groups.
//
// Per (batch, head) the token ids live in a permutation buffer `perm` whose
// node segments are contiguous and kept in ascending token order. The tree
// shape depends only on (n_q, group_size): a node at offset `off` with `cnt`
// tokens and `slots` leaf slots sends floor(slots/2)*gs tokens left, so
// every kernel recomputes a node's (off, cnt, slots) by walking its path bits
// from the root; no node table is stored. Per level:
//   1. moments        (large nodes only) count, mean and centred scatter
//                     matrix of each chunk of a node's rows;
//   2. reduce         combines a node's chunk records (pairwise-update
//                     formula) into its scatter matrix and mean;
//   3. direction      power iteration on the scatter matrix (computed in place
//                     for nodes handled as one chunk), sign fixed;
//   4. project        p_i = (x_i - mu) . v for every token of a split node;
//   5. split          radix-select cut at rank floor(slots/2)*gs, stable
//                     partition of the segment (ties: lower token id).
// After the last level leaf g is the segment [g*gs, (g+1)*gs) of perm.
// On the tensor-core path, levels whose nodes are handled as one chunk run
// steps 3-5 in one kernel: a CTA per node builds the scatter, iterates,
// projects the node's rows and cuts it.
// bf16 inputs with d = 128 take the tensor-core moments and direction kernels;
// the other shapes take the fp32 SIMT ones. Both write the same records.
#include <type_traits>

#include "kernels.h"
#include "select.cuh"
#include "tc_ptx.cuh"

namespace tlsp {

constexpr int kMomThreads = 256;
constexpr int kStageRows = 32;
constexpr int kPowerIters = 16;

struct NodeDesc {
  int off, cnt, slots;
  bool active;
};

__device__ __forceinline__ NodeDesc node_at(int n_q, int gs, int G, int level, int j) {
  NodeDesc nd{0, n_q, G, false};
  for (int b = level - 1; b >= 0; --b) {
    if (nd.slots == 1) return nd;  // passed through a leaf made at an earlier level
    const int ls = nd.slots / 2;
    if ((j >> b) & 1) {
      nd.off += ls * gs;
      nd.cnt -= ls * gs;
      nd.slots -= ls;
    } else {
      nd.cnt = ls * gs;
      nd.slots = ls;
    }
  }
  nd.active = nd.slots > 1;
  return nd;
}

// Partial-moment record: scatter [D*D], mean [D], count, padding.
template <int D>
struct Moments {
  static constexpr int kStride = D * D + 2 * D;
  static constexpr int kMu = D * D;
  static constexpr int kN = D * D + D;
};

// Count, mean and centred scatter of the rows perm[begin..end) of X.
// Each thread accumulates a (D/16) x (D/16) block of the D x D scatter.
// s_rows: kStageRows * D floats; s_mu: D floats; s_red: kMomThreads floats.
template <class T, int D>
__device__ void chunk_moments(const T* __restrict__ X, const int32_t* __restrict__ perm, int begin,
                              int end, float* s_rows, float* s_mu, float* s_red,
                              float (&acc)[D / 16][D / 16]) {
  constexpr int BLK = D / 16;
  const int t = threadIdx.x;
  // mean
  {
    constexpr int kLanesPerRow = D;                  // one thread per channel
    constexpr int kRowPar = kMomThreads / kLanesPerRow;  // rows in flight
    const int c = t % D, r0 = t / D;
    float s = 0.f;
    for (int r = begin + r0; r < end; r += kRowPar) s += to_f32(X[(int64_t)perm[r] * D + c]);
    s_red[t] = s;
    __syncthreads();
    if (t < D) {
      float tot = 0.f;
      for (int q = 0; q < kRowPar; ++q) tot += s_red[q * D + t];
      s_mu[t] = tot / (float)(end - begin);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < BLK; ++i)
#pragma unroll
    for (int j = 0; j < BLK; ++j) acc[i][j] = 0.f;
  const int bi = t / 16, bj = t % 16;
  for (int r0 = begin; r0 < end; r0 += kStageRows) {
    const int nr = min(kStageRows, end - r0);
    for (int e = t; e < kStageRows * D; e += kMomThreads) {
      const int r = e / D, c = e % D;
      s_rows[e] = r < nr ? to_f32(X[(int64_t)perm[r0 + r] * D + c]) - s_mu[c] : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      float a[BLK], b[BLK];
#pragma unroll
      for (int i = 0; i < BLK; ++i) a[i] = s_rows[r * D + bi * BLK + i];
#pragma unroll
      for (int j = 0; j < BLK; ++j) b[j] = s_rows[r * D + bj * BLK + j];
#pragma unroll
      for (int i = 0; i < BLK; ++i)
#pragma unroll
        for (int j = 0; j < BLK; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
}

template <class T, int D>
__global__ void __launch_bounds__(kMomThreads)
pddp_moments_kernel(const T* __restrict__ Q, const int32_t* __restrict__ perm, int n_q, int gs,
                    int G, int level, int cpn, int bh0, float* __restrict__ partials) {
  constexpr int BLK = D / 16;
  __shared__ float s_rows[kStageRows * D];
  __shared__ float s_mu[D];
  __shared__ float s_red[kMomThreads];
  const int j = blockIdx.y, hl = blockIdx.z, bh = bh0 + hl, c = blockIdx.x;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  const int len = (nd.cnt + cpn - 1) / cpn;
  const int begin = nd.off + c * len;
  const int end = min(nd.off + nd.cnt, begin + len);
  float* rec = partials + ((int64_t)(hl * (1 << level) + j) * cpn + c) * Moments<D>::kStride;
  if (begin >= end) {  // empty chunk: count 0
    if (threadIdx.x == 0) rec[Moments<D>::kN] = 0.f;
    return;
  }
  float acc[BLK][BLK];
  chunk_moments<T, D>(Q + (int64_t)bh * n_q * D, perm + (int64_t)bh * n_q, begin, end, s_rows,
                      s_mu, s_red, acc);
  const int bi = threadIdx.x / 16, bj = threadIdx.x % 16;
#pragma unroll
  for (int i = 0; i < BLK; ++i)
#pragma unroll
    for (int jj = 0; jj < BLK; ++jj) rec[(bi * BLK + i) * D + bj * BLK + jj] = acc[i][jj];
  if (threadIdx.x < D) rec[Moments<D>::kMu + threadIdx.x] = s_mu[threadIdx.x];
  if (threadIdx.x == 0) rec[Moments<D>::kN] = (float)(end - begin);
}

// Combines the cpn chunk records of a node into record 0 (scatter entries, in
// place) and node_mu: mu = sum_c n_c mu_c / n and
// C = sum_c [C_c + n_c (mu_c - mu)(mu_c - mu)^T], both in chunk order. Each CTA
// owns 256 entries of the D x D scatter; a thread reads and writes only its
// own entry, so the in-place update has no race.
template <int D>
__global__ void __launch_bounds__(256)
pddp_reduce_kernel(int n_q, int gs, int G, int level, int cpn, int bh0,
                   float* __restrict__ partials, float* __restrict__ node_mu) {
  __shared__ float s_mu[D];
  const int slice = blockIdx.x, j = blockIdx.y, hl = blockIdx.z, bh = bh0 + hl, t = threadIdx.x;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  float* recs = partials + (int64_t)(hl * (1 << level) + j) * cpn * Moments<D>::kStride;
  if (t < D) {
    float s = 0.f, n = 0.f;
    for (int c = 0; c < cpn; ++c) {
      const float* rec = recs + (int64_t)c * Moments<D>::kStride;
      const float nc = rec[Moments<D>::kN];
      if (nc > 0.f) {
        s += nc * rec[Moments<D>::kMu + t];
        n += nc;
      }
    }
    s_mu[t] = s / n;
  }
  __syncthreads();
  const int e = slice * 256 + t, a = e / D, b = e % D;
  float acc = 0.f;
  for (int c = 0; c < cpn; ++c) {
    const float* rec = recs + (int64_t)c * Moments<D>::kStride;
    const float nc = rec[Moments<D>::kN];
    if (!(nc > 0.f)) continue;
    const float da = rec[Moments<D>::kMu + a] - s_mu[a];
    const float db = rec[Moments<D>::kMu + b] - s_mu[b];
    acc += rec[e] + nc * da * db;
  }
  recs[e] = acc;
  if (slice == 0 && t < D) node_mu[((int64_t)bh * G + j) * D + t] = s_mu[t];
}

// Dynamic shared memory of pddp_direction_kernel.
template <int D>
constexpr size_t direction_smem_bytes() {
  return sizeof(float) * ((size_t)D * D + kStageRows * D + 4 * D + kMomThreads + 8);
}

template <class T, int D>
__global__ void __launch_bounds__(kMomThreads)
pddp_direction_kernel(const T* __restrict__ Q, const int32_t* __restrict__ perm, int n_q, int gs,
                      int G, int level, int cpn, int bh0, const float* __restrict__ partials,
                      float* __restrict__ node_mu, float* __restrict__ node_v) {
  constexpr int BLK = D / 16;
  extern __shared__ float smem[];
  float* s_C = smem;                      // D*D scatter (symmetric)
  float* s_rows = s_C + D * D;            // staging
  float* s_mu = s_rows + kStageRows * D;  // D
  float* s_v = s_mu + D;                  // D
  float* s_w = s_v + D;                   // D
  float* s_red = s_w + D + D;             // kMomThreads
  float* s_misc = s_red + kMomThreads;    // 8
  const int j = blockIdx.x, hl = blockIdx.y, bh = bh0 + hl, t = threadIdx.x;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  const int bi = t / 16, bj = t % 16;
  float acc[BLK][BLK];
  if (cpn <= 1) {
    chunk_moments<T, D>(Q + (int64_t)bh * n_q * D, perm + (int64_t)bh * n_q, nd.off,
                        nd.off + nd.cnt, s_rows, s_mu, s_red, acc);
  } else {  // scatter and mean combined by pddp_reduce_kernel (record 0, node_mu)
    const float* rec = partials + (int64_t)(hl * (1 << level) + j) * cpn * Moments<D>::kStride;
    if (t < D) s_mu[t] = node_mu[((int64_t)bh * G + j) * D + t];
#pragma unroll
    for (int i = 0; i < BLK; ++i)
#pragma unroll
      for (int jj = 0; jj < BLK; ++jj) acc[i][jj] = rec[(bi * BLK + i) * D + bj * BLK + jj];
  }
#pragma unroll
  for (int i = 0; i < BLK; ++i)
#pragma unroll
    for (int jj = 0; jj < BLK; ++jj) s_C[(bi * BLK + i) * D + bj * BLK + jj] = acc[i][jj];
  if (t < D) s_v[t] = rsqrtf((float)D);
  __syncthreads();
  // Power iteration v <- C v / |C v| (C symmetric: thread c reads column c).
  for (int it = 0; it < kPowerIters; ++it) {
    float w = 0.f;
    if (t < D) {
      for (int e = 0; e < D; ++e) w = fmaf(s_C[e * D + t], s_v[e], w);
      s_w[t] = w;
    }
    float sq = warp_sum(t < D ? w * w : 0.f);
    if ((t & 31) == 0) s_red[t >> 5] = sq;
    __syncthreads();
    if (t == 0) {
      float tot = 0.f;
      for (int q = 0; q < kMomThreads / 32; ++q) tot += s_red[q];
      s_misc[0] = sqrtf(tot);
    }
    __syncthreads();
    const float nw = s_misc[0];
    if (nw <= 1e-30f * (float)nd.cnt) {  // no spread: e_0 (uniform decision for the block)
      if (t < D) s_v[t] = (t == 0) ? 1.f : 0.f;
      __syncthreads();
      break;
    }
    if (t < D) s_v[t] = s_w[t] / nw;
    __syncthreads();
  }
  // Sign: the component of largest magnitude (lowest channel on ties) positive.
  if (t == 0) {
    int cmax = 0;
    for (int c = 1; c < D; ++c)
      if (fabsf(s_v[c]) > fabsf(s_v[cmax])) cmax = c;
    s_misc[1] = s_v[cmax] < 0.f ? -1.f : 1.f;
  }
  __syncthreads();
  const int64_t node = (int64_t)bh * G + j;  // 2^level <= G - 1 node slots per level
  if (t < D) {
    node_mu[node * D + t] = s_mu[t];
    node_v[node * D + t] = s_v[t] * s_misc[1];
  }
}

// Projection of the token at each position of perm on its node's direction
// (positions in leaves are skipped). A row is read as 16-byte vectors by a
// group of D * sizeof(T) / 16 lanes and reduced with shuffles; each group
// takes kProjRows rows and issues all their loads before it uses any, so the
// perm -> row -> reduce chains of the rows overlap.
constexpr int kProjRows = 4;

template <class T, int D>
__global__ void __launch_bounds__(256)
pddp_project_kernel(const T* __restrict__ Q, const int32_t* __restrict__ perm, int n_q, int gs,
                    int G, int level, const float* __restrict__ node_mu,
                    const float* __restrict__ node_v, uint32_t* __restrict__ seg_key,
                    float* __restrict__ trace, int64_t trace_level_stride) {
  constexpr int kVec = 16 / (int)sizeof(T);  // elements per 16-byte load
  constexpr int kLanes = D / kVec;           // lanes per row (8, 16 or 32)
  constexpr int kRows = 256 / kLanes;        // rows per pass of the block
  const int sub = threadIdx.x % kLanes;
  const int bh = blockIdx.y;
  int pos[kProjRows], node[kProjRows], token[kProjRows];
  bool live[kProjRows];
#pragma unroll
  for (int q = 0; q < kProjRows; ++q) {
    pos[q] = (blockIdx.x * kProjRows + q) * kRows + threadIdx.x / kLanes;
    live[q] = pos[q] < n_q;
    int off = 0, slots = G, j = 0;
    for (int b = 0; b < level && live[q]; ++b) {
      if (slots == 1) break;
      const int ls = slots / 2, boundary = off + ls * gs;
      if (pos[q] < boundary) {
        slots = ls;
        j = 2 * j;
      } else {
        off = boundary;
        slots -= ls;
        j = 2 * j + 1;
      }
    }
    live[q] = live[q] && slots > 1;
    node[q] = j;
    token[q] = live[q] ? perm[(int64_t)bh * n_q + pos[q]] : 0;
  }
  float x[kProjRows][kVec];
#pragma unroll
  for (int q = 0; q < kProjRows; ++q) {
    const T* xp = Q + ((int64_t)bh * n_q + token[q]) * D + sub * kVec;
    if constexpr (kVec == 8) {
      load8(xp, x[q]);
    } else {
      const float4 u = *reinterpret_cast<const float4*>(xp);
      x[q][0] = u.x; x[q][1] = u.y; x[q][2] = u.z; x[q][3] = u.w;
    }
  }
  float p[kProjRows];
#pragma unroll
  for (int q = 0; q < kProjRows; ++q) {
    p[q] = 0.f;
    const float4* mu =
        reinterpret_cast<const float4*>(node_mu + ((int64_t)bh * G + node[q]) * D + sub * kVec);
    const float4* v =
        reinterpret_cast<const float4*>(node_v + ((int64_t)bh * G + node[q]) * D + sub * kVec);
#pragma unroll
    for (int c = 0; c < kVec / 4; ++c) {
      const float4 m4 = mu[c], v4 = v[c];
      p[q] = fmaf(x[q][4 * c] - m4.x, v4.x, p[q]);
      p[q] = fmaf(x[q][4 * c + 1] - m4.y, v4.y, p[q]);
      p[q] = fmaf(x[q][4 * c + 2] - m4.z, v4.z, p[q]);
      p[q] = fmaf(x[q][4 * c + 3] - m4.w, v4.w, p[q]);
    }
  }
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1)
#pragma unroll
    for (int q = 0; q < kProjRows; ++q) p[q] += __shfl_xor_sync(0xffffffffu, p[q], o);
  if (sub == 0) {
#pragma unroll
    for (int q = 0; q < kProjRows; ++q) {
      if (!live[q]) continue;
      seg_key[(int64_t)bh * n_q + pos[q]] = float_order_key(p[q]);
      if (trace) trace[level * trace_level_stride + (int64_t)bh * n_q + token[q]] = p[q];
    }
  }
}

// Applies a cut to a node's perm segment p[0 .. n): o[j] is the index in p of
// the token that goes to position j (the ordered selection writes indices, not
// tokens, so it issues no load). The tokens are gathered into the staging
// words w (shared memory, n words, free by now) kGatherUnroll at a time, all
// loads before any store, and then written back; no global load waits on a
// global store. NT is the block's thread count.
constexpr int kGatherUnroll = 8;
template <int NT>
__device__ __forceinline__ void apply_partition(int32_t* p, const int32_t* o, uint32_t* w, int n) {
  for (int j0 = threadIdx.x; j0 < n; j0 += kGatherUnroll * NT) {
    int src[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int j = j0 + u * NT;
      src[u] = j < n ? min(max(o[j], 0), n - 1) : 0;  // (in range by construction)
    }
    int32_t val[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) val[u] = p[src[u]];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u)
      if (j0 + u * NT < n) w[j0 + u * NT] = (uint32_t)val[u];
  }
  __syncthreads();
  for (int j = threadIdx.x; j < n; j += NT) p[j] = (int32_t)w[j];
}

// One CTA per split node: cut at rank floor(slots/2)*gs on the segment keys,
// stable partition into tmp, then copy back into perm.
__global__ void __launch_bounds__(kSelectThreads)
pddp_split_kernel(int32_t* __restrict__ perm, int32_t* __restrict__ tmp,
                  const uint32_t* __restrict__ seg_key, int n_q, int gs, int G, int level) {
  __shared__ SelectShared sh;
  const int j = blockIdx.x, bh = blockIdx.y;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  const int64_t base = (int64_t)bh * n_q + nd.off;
  const int n_left = (nd.slots / 2) * gs;
  const uint32_t* keys = seg_key + base;
  int32_t* p = perm + base;
  int32_t* o = tmp + base;
  select_smallest_ordered(
      [&](int i) { return keys[i]; }, nd.cnt, n_left, sh,
      [&](uint32_t pos, int i) { o[pos] = p[i]; },
      [&](uint32_t pos, int i) { o[n_left + pos] = p[i]; });
  __syncthreads();
  for (int i = threadIdx.x; i < nd.cnt; i += kSelectThreads) p[i] = o[i];
}

// ------------------------------------------------------------ tensor-core path
// bf16 inputs with d = 128. The scatter of a run of rows is the Gram product
// D^T D of its centred rows d_i = x_i - s, computed on the tensor cores; s is
// the fp32 mean of the run's first 128 rows, already close to the run's mean.
// Each d is split into two bf16 parts, d = hi + lo + r with |r| <= 2^-18 |d|,
// and D^T D ~= hi^T hi + hi^T lo + lo^T hi accumulates in fp32 in TMEM (the
// dropped lo^T lo term is below 2^-16 of each product). Both operands of each
// MMA are the same shared-memory tile of 128 rows read MN-major (channels
// contiguous): A = tile^T (M = channel a, K = row), B = tile (N = channel b).
// The scatter about the run's own mean is then G - n m m^T, m = mean of d.

constexpr int kGT = 256;  // threads of the tensor-core PDDP kernels
constexpr int kGD = 128;  // channels
constexpr int kSub = 128; // rows per MMA batch
constexpr uint32_t kHalfB = kSub * 128;  // one 64-channel half of a tile: 128 rows x 128 B
constexpr uint32_t kTileB = 2 * kHalfB;  // one operand (hi or lo), 32 KB
constexpr uint64_t kGramWaitNs = 1000000000ull;

struct GramShared {
  float part[16][kGD];  // per row-offset channel sums
  float shift[kGD];
  float m[kGD];
  float v[kGD];
  float half[2][kGD];
  float red[8];
  uint64_t mbar, drain;
  uint32_t tmem_base;
};
constexpr uint32_t kGramSharedB = (sizeof(GramShared) + 1023) / 1024 * 1024;
constexpr size_t kGramSmem = 1024 + kGramSharedB + 2 * (size_t)kTileB;  // + slack to align
constexpr size_t kDirSmemNoGram = 1024 + kGramSharedB;
// A node's level finished inside the direction kernel keeps its order keys at
// the start of the Gram tiles and the selection state at their end.
constexpr uint32_t kFuseSelOffset =
    (2 * kTileB - (uint32_t)sizeof(SelectShared)) / 16 * 16;
constexpr int kFuseMaxKeys = (int)(kFuseSelOffset / 16 * 4);  // words, a multiple of 4

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t word_of(const uint4& v, int k) {
  return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}

// Splits (d0, d1) into packed bf16x2 high parts and low parts.
__device__ __forceinline__ void split_bf16x2(float d0, float d1, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(d0, d1);
  hi = *reinterpret_cast<uint32_t*>(&h);
  __nv_bfloat162 l = __floats2bfloat162_rn(d0 - bf16_lo(hi), d1 - bf16_hi(hi));
  lo = *reinterpret_cast<uint32_t*>(&l);
}

// Gram matrix of the rows perm[begin..end) of X ([n_q, 128] bf16, one head)
// about a shift: sum_i d_ia d_ib with d_i = x_i - sh.shift, split as d = hi +
// lo (bf16 parts) and taken as hi.hi + hi.lo + lo.hi. TMEM lane a receives
// hi.hi + lo.hi in columns [0, 128) and hi.lo in columns [128, 256): the first
// two come from one N = 256 MMA whose B operand is the hi tile followed by the
// lo tile (an M = 128 MMA costs the same at N = 256 as at N = 128), the third
// from one N = 128 MMA. On return sh.m holds the mean of
// d. Thread t handles the 16-byte chunk t % 16 of rows t / 16 + 16 i; the next
// batch is loaded into registers while the current one is converted and
// multiplied, and the perm entries of the batch after it are loaded with it.
// Returns false (status recorded, MMAs drained) after a wait that ran out; the
// result is the same for every thread of the block.
__device__ bool gram_tc(const __nv_bfloat16* __restrict__ X, const int32_t* __restrict__ perm,
                        int begin, int end, uint32_t tiles, GramShared& sh, uint32_t tmem,
                        int* status) {
  const int t = threadIdx.x;
  const int q = t & 15, ro = t >> 4;
  const int h = q >> 3, c8 = q & 7;  // 64-channel half, 16-byte chunk within it
  const int n = end - begin;
  const int nsub = (n + kSub - 1) / kSub;
  const uint4* Xv = reinterpret_cast<const uint4*>(X);
  uint4 cur[8], nxt[8];
  int ix[8];  // perm entries of the next batch whose rows are not yet requested
  auto fetch = [&](int sub) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = begin + sub * kSub + ro + 16 * i;
      ix[i] = (sub < nsub && r < end) ? perm[r] : -1;
    }
  };
  auto load = [&](uint4(&buf)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      buf[i] = ix[i] >= 0 ? __ldg(Xv + (int64_t)ix[i] * (kGD / 8) + q) : make_uint4(0, 0, 0, 0);
  };
  fetch(0);
  load(cur);
  fetch(1);
  {  // shift: mean of the first batch (rows past the end load as zeros)
    float s[8] = {};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        s[2 * k] += bf16_lo(word_of(cur[i], k));
        s[2 * k + 1] += bf16_hi(word_of(cur[i], k));
      }
#pragma unroll
    for (int k = 0; k < 8; ++k) sh.part[ro][q * 8 + k] = s[k];
    __syncthreads();
    if (t < kGD) {
      float tot = 0.f;
      for (int r = 0; r < 16; ++r) tot += sh.part[r][t];
      sh.shift[t] = tot / (float)min(n, kSub);
    }
    __syncthreads();
  }
  float sv[8], sum[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    sv[k] = sh.shift[q * 8 + k];
    sum[k] = 0.f;
  }
  const uint32_t hi_base = tiles, lo_base = tiles + kTileB;
  constexpr uint32_t idesc = ptx::idesc_bf16(128, 128, true, true);
  constexpr uint32_t idesc_wide = ptx::idesc_bf16(128, 256, true, true);
  bool ok = true;
  for (int sub = 0; sub < nsub; ++sub) {
    if (sub + 1 < nsub) {
      load(nxt);       // rows of batch sub + 1 (their perm entries arrived a batch ago)
      fetch(sub + 2);  // perm entries of batch sub + 2, in flight with those rows
    }
    // the tile is rewritten only after the previous batch's MMAs have read it
    if (sub > 0) ok = ptx::mbar_wait(&sh.mbar, (sub - 1) & 1, nullptr, kGramWaitNs);
    if (ok) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = ro + 16 * i;
        const bool valid = sub * kSub + r < n;
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t x = word_of(cur[i], k);
          const float d0 = valid ? bf16_lo(x) - sv[2 * k] : 0.f;
          const float d1 = valid ? bf16_hi(x) - sv[2 * k + 1] : 0.f;
          sum[2 * k] += d0;
          sum[2 * k + 1] += d1;
          split_bf16x2(d0, d1, hw[k], lw[k]);
        }
        const uint32_t off = h * kHalfB + r * 128 + ((c8 ^ (r & 7)) << 4);
        ptx::st_shared_v4(hi_base + off, hw[0], hw[1], hw[2], hw[3]);
        ptx::st_shared_v4(lo_base + off, lw[0], lw[1], lw[2], lw[3]);
      }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    if (t == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < kSub / 16; ++ks) {
        // (lo_base = hi_base + 2 * kHalfB: as an N = 256 operand the hi tile's two
        // 64-channel atoms are followed by the lo tile's)
        const uint64_t dh = ptx::sw128_desc(hi_base + ks * 2048, kHalfB, 1024);
        const uint64_t dl = ptx::sw128_desc(lo_base + ks * 2048, kHalfB, 1024);
        ptx::mma_ss(tmem, dh, dh, idesc_wide, (sub > 0 || ks > 0) ? 1u : 0u);
        ptx::mma_ss(tmem, dl, dh, idesc, 1u);
      }
      ptx::tc_commit(&sh.mbar);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
  }
  if (ok) ok = ptx::mbar_wait(&sh.mbar, (nsub - 1) & 1, nullptr, kGramWaitNs);
  if (__syncthreads_or(!ok)) {
    if (t == 0) {
      record_status(status, TLSP_ERR_TIMEOUT);
      ptx::tc_commit(&sh.drain);  // every MMA issued must land before TMEM is freed
      ptx::mbar_wait(&sh.drain, 0, nullptr, kGramWaitNs);
    }
    __syncthreads();
    return false;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) sh.part[ro][q * 8 + k] = sum[k];
  __syncthreads();
  if (t < kGD) {
    float tot = 0.f;
    for (int r = 0; r < 16; ++r) tot += sh.part[r][t];
    sh.m[t] = tot / (float)n;
  }
  __syncthreads();
  ptx::tc_fence_after();
  return true;
}

// Shared-memory carve-up and TMEM allocation common to the two kernels below.
struct GramCta {
  GramShared* sh;
  uint32_t tiles;
};
__device__ __forceinline__ GramCta gram_cta_layout(uint8_t* smem_raw) {
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  return {reinterpret_cast<GramShared*>(smem_raw + (base - raw)), base + kGramSharedB};
}
__device__ __forceinline__ uint32_t gram_cta_setup(GramShared& sh) {
  if (threadIdx.x == 0) {
    ptx::mbar_init(&sh.mbar, 1);
    ptx::mbar_init(&sh.drain, 1);
    ptx::fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    ptx::tmem_alloc(&sh.tmem_base, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  return sh.tmem_base;
}
__device__ __forceinline__ void gram_cta_release(uint32_t tmem) {
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
}

// This thread's 64 entries of the centred scatter held in TMEM: row
// a = 32 (warp % 4) + lane, columns e0 .. e0 + 63 with e0 = 64 (warp / 4):
// the sum of the two accumulator halves (hi.hi + lo.hi, and hi.lo), minus the
// shift correction n m_a m_b.
__device__ __forceinline__ void gram_row_part(uint32_t tmem, const GramShared& sh, float n,
                                              float (&C)[64]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a = 32 * (warp & 3) + lane, e0 = 64 * (warp >> 2);
  const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)e0;
  const float nma = n * sh.m[a];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t l[16], rr[16];
    ptx::tmem_ld16(tl + 16 * q, l);
    ptx::tmem_ld16(tl + 128 + 16 * q, rr);
    ptx::tmem_ld_wait(l);
    ptx::reg_barrier16(rr);
#pragma unroll
    for (int e = 0; e < 16; ++e)
      C[16 * q + e] = (__uint_as_float(l[e]) + __uint_as_float(rr[e])) - nma * sh.m[e0 + 16 * q + e];
  }
}

// Chunk records of the tensor-core path (same format as pddp_moments_kernel).
__global__ void __launch_bounds__(kGT, 2)
pddp_gram_tc_kernel(const __nv_bfloat16* __restrict__ Q, const int32_t* __restrict__ perm,
                    int n_q, int gs, int G, int level, int cpn, int bh0,
                    float* __restrict__ partials, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const GramCta cta = gram_cta_layout(smem_raw);
  GramShared& sh = *cta.sh;
  const int c = blockIdx.x, j = blockIdx.y, hl = blockIdx.z, bh = bh0 + hl, t = threadIdx.x;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  const int len = (nd.cnt + cpn - 1) / cpn;
  const int begin = nd.off + c * len;
  const int end = min(nd.off + nd.cnt, begin + len);
  float* rec = partials + ((int64_t)(hl * (1 << level) + j) * cpn + c) * Moments<kGD>::kStride;
  if (begin >= end) {
    if (t == 0) rec[Moments<kGD>::kN] = 0.f;
    return;
  }
  const uint32_t tmem = gram_cta_setup(sh);
  const bool ok = gram_tc(Q + (int64_t)bh * n_q * kGD, perm + (int64_t)bh * n_q, begin, end,
                          cta.tiles, sh, tmem, status);
  if (ok) {
    float C[64];
    gram_row_part(tmem, sh, (float)(end - begin), C);
    const int warp = t >> 5, a = 32 * (warp & 3) + (t & 31), e0 = 64 * (warp >> 2);
    float4* dst = reinterpret_cast<float4*>(rec + a * kGD + e0);
#pragma unroll
    for (int e = 0; e < 64; e += 4) dst[e / 4] = make_float4(C[e], C[e + 1], C[e + 2], C[e + 3]);
    if (t < kGD) rec[Moments<kGD>::kMu + t] = sh.shift[t] + sh.m[t];
    if (t == 0) rec[Moments<kGD>::kN] = (float)(end - begin);
  } else if (t == 0) {
    rec[Moments<kGD>::kN] = 0.f;
  }
  gram_cta_release(tmem);
}

// Projections of the node's rows perm[off .. off + cnt) on v about the node
// mean mu = sh.shift + sh.m, with the arithmetic of pddp_project_kernel (16
// lanes per row, 8 channels each, products summed in channel order, then a
// shuffle tree), so a projection here is bit-identical to one made there.
// keys[i] receives the order key of row off + i; trace, when given, the
// projection at the row's token. Rows just read for the Gram are mostly still
// in L2; the perm entries of kFuseRows rows are loaded before any of them.
constexpr int kFuseRows = 8;  // rows per 16-lane group and pass
__device__ __forceinline__ void project_node_tc(const __nv_bfloat16* __restrict__ X,
                                                const int32_t* __restrict__ permh, int off,
                                                int cnt, const GramShared& sh, uint32_t* keys,
                                                float* __restrict__ trace) {
  const int sub = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  float mu[8], vv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mu[e] = sh.shift[sub * 8 + e] + sh.m[sub * 8 + e];
    vv[e] = sh.v[sub * 8 + e];
  }
  for (int base = 0; base < cnt; base += (kGT / 16) * kFuseRows) {
    int tok[kFuseRows];
#pragma unroll
    for (int q = 0; q < kFuseRows; ++q) {
      const int i = base + r0 + (kGT / 16) * q;
      tok[q] = i < cnt ? permh[off + i] : -1;
    }
    float x[kFuseRows][8];
#pragma unroll
    for (int q = 0; q < kFuseRows; ++q) {
      if (tok[q] >= 0) {
        load8(X + (int64_t)tok[q] * kGD + sub * 8, x[q]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[q][e] = 0.f;
      }
    }
    float pr[kFuseRows];
#pragma unroll
    for (int q = 0; q < kFuseRows; ++q) {
      pr[q] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) pr[q] = fmaf(x[q][e] - mu[e], vv[e], pr[q]);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
#pragma unroll
      for (int q = 0; q < kFuseRows; ++q) pr[q] += __shfl_xor_sync(0xffffffffu, pr[q], o);
    if (sub == 0) {
#pragma unroll
      for (int q = 0; q < kFuseRows; ++q) {
        if (tok[q] < 0) continue;
        keys[base + r0 + (kGT / 16) * q] = float_order_key(pr[q]);
        if (trace) trace[tok[q]] = pr[q];
      }
    }
  }
}

// Node of position pos at `level` (as pddp_project_kernel walks it); false
// for positions in leaves made at earlier levels.
__device__ __forceinline__ bool live_node_of(int pos, int n_q, int gs, int G, int level, int& j) {
  int off = 0, slots = G;
  j = 0;
  if (pos >= n_q) return false;
  for (int b = 0; b < level; ++b) {
    if (slots == 1) return false;
    const int ls = slots / 2, boundary = off + ls * gs;
    if (pos < boundary) {
      slots = ls;
      j = 2 * j;
    } else {
      off = boundary;
      slots -= ls;
      j = 2 * j + 1;
    }
  }
  return slots > 1;
}

// pddp_project_kernel for bf16 rows of 128 channels, restructured for memory
// parallelism: each 16-lane group walks runs of kProjRun consecutive positions
// of one head (grid-stride), loading the next run's perm entries while the
// current run's rows are in flight, and keeps its node's mean and direction in
// registers while the positions stay in that node. A warp takes two runs per
// step (one per half) and steps while its first run is in range, so every
// shuffle has all 32 lanes. Per row the arithmetic is that of
// pddp_project_kernel, so the keys are bit-identical. Grid: (blocks per head,
// BH).
constexpr int kProjRun = 8;
constexpr int kProjBlocksPerSm = 3;
__global__ void __launch_bounds__(256, kProjBlocksPerSm)
pddp_project_tc_kernel(const __nv_bfloat16* __restrict__ Q, const int32_t* __restrict__ perm,
                       int n_q, int gs, int G, int level, const float* __restrict__ node_mu,
                       const float* __restrict__ node_v, uint32_t* __restrict__ seg_key,
                       float* __restrict__ trace, int64_t trace_level_stride) {
  const int sub = threadIdx.x & 15, half = (threadIdx.x >> 4) & 1, bh = blockIdx.y;
  const int wg = blockIdx.x * 8 + (threadIdx.x >> 5), step = gridDim.x * 16;
  const int nrun = (n_q + kProjRun - 1) / kProjRun;
  const int32_t* ph = perm + (int64_t)bh * n_q;
  const uint4* Xh = reinterpret_cast<const uint4*>(Q + (int64_t)bh * n_q * kGD);
  const float* mu_h = node_mu + (int64_t)bh * G * kGD + sub * 8;
  const float* v_h = node_v + (int64_t)bh * G * kGD + sub * 8;
  int tok[kProjRun];
  auto fetch = [&](int run) {
#pragma unroll
    for (int q = 0; q < kProjRun; ++q) {
      const int pos = run * kProjRun + q;
      tok[q] = (run < nrun && pos < n_q) ? ph[pos] : -1;
    }
  };
  fetch(2 * wg + half);
  int cur = -1;
  float mu[8], vv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mu[e] = vv[e] = 0.f;
  for (int base = 2 * wg; base < nrun; base += step) {  // (warp-uniform)
    const int run = base + half;
    uint4 raw[kProjRun];
    int tk[kProjRun];
#pragma unroll
    for (int q = 0; q < kProjRun; ++q) {
      tk[q] = tok[q];
      raw[q] = tk[q] >= 0 ? __ldg(Xh + (int64_t)tk[q] * (kGD / 8) + sub) : make_uint4(0, 0, 0, 0);
    }
    fetch(run + step);  // in flight with the rows above
    const int p0 = run * kProjRun;
    int j_first, j_last;
    const bool l_first = live_node_of(p0, n_q, gs, G, level, j_first);
    const bool l_last = live_node_of(min(p0 + kProjRun, n_q) - 1, n_q, gs, G, level, j_last);
    const bool one_node = l_first && l_last && j_first == j_last;
    float pr[kProjRun];
    bool live[kProjRun];
#pragma unroll
    for (int q = 0; q < kProjRun; ++q) {
      int j = j_first;
      live[q] = tk[q] >= 0 && (one_node || live_node_of(p0 + q, n_q, gs, G, level, j));
      pr[q] = 0.f;
      if (!live[q]) continue;
      if (j != cur) {
        const float4 m0 = *reinterpret_cast<const float4*>(mu_h + (int64_t)j * kGD);
        const float4 m1 = *reinterpret_cast<const float4*>(mu_h + (int64_t)j * kGD + 4);
        const float4 v0 = *reinterpret_cast<const float4*>(v_h + (int64_t)j * kGD);
        const float4 v1 = *reinterpret_cast<const float4*>(v_h + (int64_t)j * kGD + 4);
        mu[0] = m0.x; mu[1] = m0.y; mu[2] = m0.z; mu[3] = m0.w;
        mu[4] = m1.x; mu[5] = m1.y; mu[6] = m1.z; mu[7] = m1.w;
        vv[0] = v0.x; vv[1] = v0.y; vv[2] = v0.z; vv[3] = v0.w;
        vv[4] = v1.x; vv[5] = v1.y; vv[6] = v1.z; vv[7] = v1.w;
        cur = j;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t w = word_of(raw[q], k);
        pr[q] = fmaf(bf16_lo(w) - mu[2 * k], vv[2 * k], pr[q]);
        pr[q] = fmaf(bf16_hi(w) - mu[2 * k + 1], vv[2 * k + 1], pr[q]);
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
#pragma unroll
      for (int q = 0; q < kProjRun; ++q) pr[q] += __shfl_xor_sync(0xffffffffu, pr[q], o);
    if (sub == 0) {
#pragma unroll
      for (int q = 0; q < kProjRun; ++q) {
        if (!live[q]) continue;
        seg_key[(int64_t)bh * n_q + p0 + q] = float_order_key(pr[q]);
        if (trace) trace[level * trace_level_stride + (int64_t)bh * n_q + tk[q]] = pr[q];
      }
    }
  }
}

// Principal direction of one node. With cpn <= 1 the node's scatter is built
// here (tensor-core Gram over all its rows) and its mean written to node_mu;
// otherwise both come combined from pddp_reduce_kernel. The scatter stays in
// registers (thread: row a, 64 columns) for the 16 power iterations
// v <- C v / |C v|; the sign makes the component of largest magnitude (lowest
// channel on ties) positive.
// With `tmp` given (cpn <= 1 only) the kernel also finishes the node's level:
// the projections of its rows (project_node_tc; trace at trace_level when
// given), staged as order keys in the Gram tile region, and the cut at rank
// floor(slots/2)*gs with the stable partition of perm (as pddp_split_smem_kernel,
// through tmp). The node then needs no projection or split launch.
__global__ void __launch_bounds__(kGT, 2)
pddp_direction_tc_kernel(const __nv_bfloat16* __restrict__ Q, int32_t* __restrict__ perm,
                         int n_q, int gs, int G, int level, int cpn, int bh0,
                         const float* __restrict__ partials, float* __restrict__ node_mu,
                         float* __restrict__ node_v, int* status, int32_t* __restrict__ tmp,
                         float* __restrict__ trace_level) {
  extern __shared__ uint8_t smem_raw[];
  const GramCta cta = gram_cta_layout(smem_raw);
  GramShared& sh = *cta.sh;
  const int j = blockIdx.x, hl = blockIdx.y, bh = bh0 + hl, t = threadIdx.x, warp = t >> 5,
            lane = t & 31;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  const int a = 32 * (warp & 3) + lane, e0 = 64 * (warp >> 2);
  const int64_t node = (int64_t)bh * G + j;
  float C[64];
  if (cpn <= 1) {
    const uint32_t tmem = gram_cta_setup(sh);
    const bool ok = gram_tc(Q + (int64_t)bh * n_q * kGD, perm + (int64_t)bh * n_q, nd.off,
                            nd.off + nd.cnt, cta.tiles, sh, tmem, status);
    if (ok) {
      gram_row_part(tmem, sh, (float)nd.cnt, C);
      if (t < kGD) node_mu[node * kGD + t] = sh.shift[t] + sh.m[t];
    }
    gram_cta_release(tmem);
    if (!ok) return;
  } else {
    const float4* src = reinterpret_cast<const float4*>(
        partials + (int64_t)(hl * (1 << level) + j) * cpn * Moments<kGD>::kStride + a * kGD + e0);
#pragma unroll
    for (int e = 0; e < 64; e += 4) {
      const float4 u = src[e / 4];
      C[e] = u.x;
      C[e + 1] = u.y;
      C[e + 2] = u.z;
      C[e + 3] = u.w;
    }
  }
  if (t < kGD) sh.v[t] = rsqrtf((float)kGD);
  __syncthreads();
  for (int it = 0; it < kPowerIters; ++it) {
    float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
    for (int e = 0; e < 64; e += 4) {
      const float4 vv = *reinterpret_cast<const float4*>(&sh.v[e0 + e]);
      p0 = fmaf(C[e], vv.x, p0);
      p1 = fmaf(C[e + 1], vv.y, p1);
      p2 = fmaf(C[e + 2], vv.z, p2);
      p3 = fmaf(C[e + 3], vv.w, p3);
    }
    sh.half[warp >> 2][a] = (p0 + p1) + (p2 + p3);
    __syncthreads();
    float w = 0.f;
    if (t < kGD) {
      w = sh.half[0][t] + sh.half[1][t];
      const float sq = warp_sum(w * w);
      if (lane == 0) sh.red[warp] = sq;
    }
    __syncthreads();
    const float nw = sqrtf((sh.red[0] + sh.red[1]) + (sh.red[2] + sh.red[3]));
    if (nw <= 1e-30f * (float)nd.cnt) {  // no spread: e_0 (the same decision in every thread)
      if (t < kGD) sh.v[t] = t == 0 ? 1.f : 0.f;
      __syncthreads();
      break;
    }
    if (t < kGD) sh.v[t] = w / nw;
    __syncthreads();
  }
  if (warp == 0) {  // component of largest magnitude, lowest channel on ties
    float best = fabsf(sh.v[lane]);
    int cmax = lane;
#pragma unroll
    for (int c = lane + 32; c < kGD; c += 32)
      if (fabsf(sh.v[c]) > best) {
        best = fabsf(sh.v[c]);
        cmax = c;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oc = __shfl_xor_sync(0xffffffffu, cmax, o);
      if (ob > best || (ob == best && oc < cmax)) {
        best = ob;
        cmax = oc;
      }
    }
    if (lane == 0) sh.red[4] = sh.v[cmax] < 0.f ? -1.f : 1.f;
  }
  __syncthreads();
  const float vf = t < kGD ? sh.v[t] * sh.red[4] : 0.f;
  if (t < kGD) node_v[node * kGD + t] = vf;
  if (tmp == nullptr || cpn > 1) return;
  __syncthreads();  // every thread has read sh.v and sh.red[4]
  if (t < kGD) sh.v[t] = vf;
  // keys, then the selection state, in the Gram tiles (their MMAs completed)
  uint8_t* tiles = smem_raw + (cta.tiles - ptx::smem_u32(smem_raw));
  uint32_t* keys = reinterpret_cast<uint32_t*>(tiles);
  SelectShared& ssh = *reinterpret_cast<SelectShared*>(tiles + kFuseSelOffset);
  __syncthreads();
  const int64_t base = (int64_t)bh * n_q + nd.off;
  project_node_tc(Q + (int64_t)bh * n_q * kGD, perm + (int64_t)bh * n_q, nd.off, nd.cnt, sh, keys,
                  trace_level ? trace_level + (int64_t)bh * n_q : nullptr);
  __syncthreads();
  const int n_left = (nd.slots / 2) * gs;
  int32_t* p = perm + base;
  int32_t* o = tmp + base;
  smem_select_ordered<kGT>(
      keys, nd.cnt, n_left, [](uint32_t w) { return w; }, ssh,
      [&](uint32_t pos, int i) { o[pos] = i; },
      [&](uint32_t pos, int i) { o[n_left + pos] = i; });
  __syncthreads();
  apply_partition<kGT>(p, o, keys, nd.cnt);
}

// pddp_split_kernel with the node's keys staged in shared memory (nodes of
// at most kSplitSmemKeys tokens); the selection writes indices into tmp and
// apply_partition moves the tokens. Dynamic shared memory: keys rounded up to
// 4 words.
constexpr int kSplitSmemKeys = 52 * 1024;
__global__ void __launch_bounds__(kSelectThreads)
pddp_split_smem_kernel(int32_t* __restrict__ perm, int32_t* __restrict__ tmp,
                       const uint32_t* __restrict__ seg_key, int n_q, int gs, int G, int level) {
  extern __shared__ __align__(128) uint8_t split_smem[];
  __shared__ SelectShared sh;
  const int j = blockIdx.x, bh = blockIdx.y;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  uint32_t* keys = reinterpret_cast<uint32_t*>(split_smem);
  const int64_t base = (int64_t)bh * n_q + nd.off;
  for (int i = threadIdx.x; i < nd.cnt; i += kSelectThreads) keys[i] = seg_key[base + i];
  __syncthreads();
  const int n_left = (nd.slots / 2) * gs;
  int32_t* p = perm + base;
  int32_t* o = tmp + base;
  smem_select_ordered(
      keys, nd.cnt, n_left, [](uint32_t w) { return w; }, sh,
      [&](uint32_t pos, int i) { o[pos] = i; },
      [&](uint32_t pos, int i) { o[n_left + pos] = i; });
  __syncthreads();
  apply_partition<kSelectThreads>(p, o, keys, nd.cnt);
}

__global__ void pddp_init_kernel(int32_t* __restrict__ perm, int n_q, int64_t total) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < total) perm[i] = (int32_t)(i % n_q);
}

__global__ void pddp_emit_kernel(const int32_t* __restrict__ perm, int n_q, int gs, int G,
                                 int32_t* __restrict__ groups, int64_t total) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int64_t per = (int64_t)G * gs;
  const int64_t bh = i / per, q = i % per;
  groups[i] = q < n_q ? perm[bh * n_q + q] : -1;
}

// ----------------------------------------------------------------- host side

// Chunk records per head and tree level at most (see run_pddp_t).
constexpr int64_t kChunksPerHead = 32;

static int levels_of(int G) {
  int L = 0;
  while ((1 << L) < G) ++L;
  return L;
}

template <class T, int D>
static int run_pddp_t(const T* Q, int64_t BH, int n_q, int gs, int32_t* groups, float* trace,
                      const PddpWork& w, cudaStream_t st) {
  constexpr bool kTc = std::is_same<T, __nv_bfloat16>::value && D == kGD;
  const int G = (n_q + gs - 1) / gs;
  const int L = levels_of(G);
  const int64_t total = BH * n_q;
  pddp_init_kernel<<<(unsigned)ceil_div(total, 256), 256, 0, st>>>(w.perm, n_q, total);
  TLSP_TRY(check_launch());
  if (kTc) {
    TLSP_TRY(ensure_smem_limit((const void*)pddp_gram_tc_kernel, (int)kGramSmem));
    TLSP_TRY(ensure_smem_limit((const void*)pddp_direction_tc_kernel, (int)kGramSmem));
  }
  TLSP_TRY(ensure_smem_limit((const void*)pddp_split_smem_kernel,
                             (int)((size_t)kSplitSmemKeys * 4)));
  if (!kTc) {
    TLSP_TRY(ensure_smem_limit((const void*)pddp_direction_kernel<T, D>,
                               (int)direction_smem_bytes<D>()));
  }
  for (int level = 0; level < L; ++level) {
    const int64_t nodes = 1 << level;
    const int64_t max_rows = ceil_div(n_q, nodes) + gs;
    // Chunks per node depend only on the node sizes (never on how many heads
    // the call holds or on the device), so a head's groups are the same
    // whether it is grouped alone or with others: at most kChunksPerHead
    // records per head and level, each chunk at least two MMA batches (tensor
    // cores) or about 256 rows (SIMT).
    int64_t cpn = kTc ? ceil_div(max_rows, 2 * kSub) : ceil_div(max_rows, 256);
    cpn = std::min<int64_t>(cpn, std::max<int64_t>(1, kChunksPerHead / nodes));
    if (cpn < 2) cpn = 1;
    // levels whose nodes build their own scatter also project and cut them there
    const bool fused = kTc && cpn == 1 && max_rows <= kFuseMaxKeys;
    // heads whose chunk records fit in the workspace at once
    const int64_t hb = cpn > 1 ? std::max<int64_t>(1, w.partial_slots / (nodes * cpn)) : BH;
    for (int64_t h0 = 0; h0 < BH; h0 += hb) {
      const unsigned nh = (unsigned)std::min<int64_t>(hb, BH - h0);
      if (cpn > 1) {
        const dim3 grid((unsigned)cpn, (unsigned)nodes, nh);
        if constexpr (kTc) {
          pddp_gram_tc_kernel<<<grid, kGT, kGramSmem, st>>>(Q, w.perm, n_q, gs, G, level,
                                                            (int)cpn, (int)h0, w.partials,
                                                            w.status);
        } else {
          pddp_moments_kernel<T, D><<<grid, kMomThreads, 0, st>>>(Q, w.perm, n_q, gs, G, level,
                                                                  (int)cpn, (int)h0, w.partials);
        }
        TLSP_TRY(check_launch());
        pddp_reduce_kernel<D><<<dim3(D * D / 256, (unsigned)nodes, nh), 256, 0, st>>>(
            n_q, gs, G, level, (int)cpn, (int)h0, w.partials, w.node_mu);
        TLSP_TRY(check_launch());
      }
      if constexpr (kTc) {
        pddp_direction_tc_kernel<<<dim3((unsigned)nodes, nh), kGT,
                                   cpn > 1 ? kDirSmemNoGram : kGramSmem, st>>>(
            Q, w.perm, n_q, gs, G, level, (int)cpn, (int)h0, w.partials, w.node_mu, w.node_v,
            w.status, fused ? w.tmp : nullptr, fused && trace ? trace + level * total : nullptr);
      } else {
        pddp_direction_kernel<T, D><<<dim3((unsigned)nodes, nh), kMomThreads,
                                      direction_smem_bytes<D>(), st>>>(
            Q, w.perm, n_q, gs, G, level, (int)cpn, (int)h0, w.partials, w.node_mu, w.node_v);
      }
      TLSP_TRY(check_launch());
    }
    if (fused) continue;
    if constexpr (kTc) {
      // one resident wave of blocks in all, at most one 16-lane group per run
      const int64_t runs = ceil_div(n_q, kProjRun);
      const int64_t per_head = std::max<int64_t>(
          1, std::min<int64_t>(ceil_div(kProjBlocksPerSm * (int64_t)device_sm_count(), BH),
                               ceil_div(runs, 16)));
      pddp_project_tc_kernel<<<dim3((unsigned)per_head, (unsigned)BH), 256, 0, st>>>(
          Q, w.perm, n_q, gs, G, level, w.node_mu, w.node_v, w.seg_key, trace, total);
    } else {
      constexpr int kRowsPerBlock = 256 / (D * (int)sizeof(T) / 16) * kProjRows;
      pddp_project_kernel<T, D>
          <<<dim3((unsigned)ceil_div(n_q, kRowsPerBlock), (unsigned)BH), 256, 0, st>>>(
              Q, w.perm, n_q, gs, G, level, w.node_mu, w.node_v, w.seg_key, trace, total);
    }
    TLSP_TRY(check_launch());
    if (max_rows <= kSplitSmemKeys) {
      const size_t smem = (size_t)((max_rows + 3) & ~3) * 4;
      pddp_split_smem_kernel<<<dim3((unsigned)nodes, (unsigned)BH), kSelectThreads, smem, st>>>(
          w.perm, w.tmp, w.seg_key, n_q, gs, G, level);
    } else {
      pddp_split_kernel<<<dim3((unsigned)nodes, (unsigned)BH), kSelectThreads, 0, st>>>(
          w.perm, w.tmp, w.seg_key, n_q, gs, G, level);
    }
    TLSP_TRY(check_launch());
  }
  const int64_t out_total = BH * (int64_t)G * gs;
  pddp_emit_kernel<<<(unsigned)ceil_div(out_total, 256), 256, 0, st>>>(w.perm, n_q, gs, G, groups,
                                                                       out_total);
  return check_launch();
}

int run_pddp(const void* Q, bool bf16, int d, int64_t BH, int n_q, int gs, int32_t* groups,
             float* trace, const PddpWork& w, cudaStream_t st) {
  if (bf16) {
    if (d == 128) return run_pddp_t<__nv_bfloat16, 128>((const __nv_bfloat16*)Q, BH, n_q, gs, groups, trace, w, st);
    return run_pddp_t<__nv_bfloat16, 64>((const __nv_bfloat16*)Q, BH, n_q, gs, groups, trace, w, st);
  }
  if (d == 128) return run_pddp_t<float, 128>((const float*)Q, BH, n_q, gs, groups, trace, w, st);
  return run_pddp_t<float, 64>((const float*)Q, BH, n_q, gs, groups, trace, w, st);
}

}  // namespace tlsp
