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
//   1. pddp_moments   (large nodes only) count, mean and centred scatter
//                     matrix of each chunk of a node's rows;
//   2. pddp_direction combines the chunk moments (pairwise-update formula),
//                     runs the power iteration and fixes the sign;
//   3. pddp_project   p_i = (x_i - mu) . v for every token of a split node;
//   4. pddp_split     radix-select cut at rank floor(slots/2)*gs, stable
//                     partition of the segment (ties: lower token id).
// After the last level leaf g is the segment [g*gs, (g+1)*gs) of perm.
#include "kernels.h"
#include "select.cuh"

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
                    int G, int level, int cpn, float* __restrict__ partials) {
  constexpr int BLK = D / 16;
  __shared__ float s_rows[kStageRows * D];
  __shared__ float s_mu[D];
  __shared__ float s_red[kMomThreads];
  const int j = blockIdx.y, bh = blockIdx.z, c = blockIdx.x;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  const int len = (nd.cnt + cpn - 1) / cpn;
  const int begin = nd.off + c * len;
  const int end = min(nd.off + nd.cnt, begin + len);
  float* rec = partials + ((int64_t)(bh * (1 << level) + j) * cpn + c) * Moments<D>::kStride;
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

// Dynamic shared memory of pddp_direction_kernel.
template <int D>
constexpr size_t direction_smem_bytes() {
  return sizeof(float) * ((size_t)D * D + kStageRows * D + 4 * D + kMomThreads + 8);
}

template <class T, int D>
__global__ void __launch_bounds__(kMomThreads)
pddp_direction_kernel(const T* __restrict__ Q, const int32_t* __restrict__ perm, int n_q, int gs,
                      int G, int level, int cpn, const float* __restrict__ partials,
                      float* __restrict__ node_mu, float* __restrict__ node_v) {
  constexpr int BLK = D / 16;
  extern __shared__ float smem[];
  float* s_C = smem;                      // D*D scatter (symmetric)
  float* s_rows = s_C + D * D;            // staging
  float* s_mu = s_rows + kStageRows * D;  // D
  float* s_v = s_mu + D;                  // D
  float* s_w = s_v + D;                   // D
  float* s_muc = s_w + D;                 // D
  float* s_red = s_muc + D;               // kMomThreads
  float* s_misc = s_red + kMomThreads;    // 8
  const int j = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const NodeDesc nd = node_at(n_q, gs, G, level, j);
  if (!nd.active) return;
  const int bi = t / 16, bj = t % 16;
  float acc[BLK][BLK];
  if (cpn <= 1) {
    chunk_moments<T, D>(Q + (int64_t)bh * n_q * D, perm + (int64_t)bh * n_q, nd.off,
                        nd.off + nd.cnt, s_rows, s_mu, s_red, acc);
  } else {
    const float* recs = partials + (int64_t)(bh * (1 << level) + j) * cpn * Moments<D>::kStride;
    // overall mean
    if (t < D) {
      float s = 0.f, n = 0.f;
      for (int c = 0; c < cpn; ++c) {
        const float nc = recs[c * Moments<D>::kStride + Moments<D>::kN];
        if (nc > 0.f) {
          s += nc * recs[c * Moments<D>::kStride + Moments<D>::kMu + t];
          n += nc;
        }
      }
      s_mu[t] = s / n;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < BLK; ++i)
#pragma unroll
      for (int jj = 0; jj < BLK; ++jj) acc[i][jj] = 0.f;
    for (int c = 0; c < cpn; ++c) {
      const float* rec = recs + c * Moments<D>::kStride;
      const float nc = rec[Moments<D>::kN];
      if (!(nc > 0.f)) continue;
      if (t < D) s_muc[t] = rec[Moments<D>::kMu + t] - s_mu[t];
      __syncthreads();
      float a[BLK], b[BLK];
#pragma unroll
      for (int i = 0; i < BLK; ++i) a[i] = s_muc[bi * BLK + i];
#pragma unroll
      for (int jj = 0; jj < BLK; ++jj) b[jj] = s_muc[bj * BLK + jj];
#pragma unroll
      for (int i = 0; i < BLK; ++i)
#pragma unroll
        for (int jj = 0; jj < BLK; ++jj)
          acc[i][jj] += rec[(bi * BLK + i) * D + bj * BLK + jj] + nc * a[i] * b[jj];
      __syncthreads();
    }
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

// One warp per position of perm: projection of the token there on its node's
// direction (positions in leaves are skipped).
template <class T, int D>
__global__ void __launch_bounds__(256)
pddp_project_kernel(const T* __restrict__ Q, const int32_t* __restrict__ perm, int n_q, int gs,
                    int G, int level, const float* __restrict__ node_mu,
                    const float* __restrict__ node_v, uint32_t* __restrict__ seg_key,
                    float* __restrict__ trace, int64_t trace_level_stride) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  if (warp >= n_q) return;
  const int pos = warp;
  int off = 0, cnt = n_q, slots = G, j = 0;
  for (int b = 0; b < level; ++b) {
    if (slots == 1) return;
    const int ls = slots / 2, boundary = off + ls * gs;
    if (pos < boundary) {
      cnt = ls * gs;
      slots = ls;
      j = 2 * j;
    } else {
      off = boundary;
      cnt -= ls * gs;
      slots -= ls;
      j = 2 * j + 1;
    }
  }
  if (slots == 1) return;
  const int token = perm[(int64_t)bh * n_q + pos];
  const T* x = Q + ((int64_t)bh * n_q + token) * D;
  const float* mu = node_mu + ((int64_t)bh * G + j) * D;
  const float* v = node_v + ((int64_t)bh * G + j) * D;
  float p = 0.f;
#pragma unroll
  for (int c = lane; c < D; c += 32) p = fmaf(to_f32(x[c]) - mu[c], v[c], p);
  p = warp_sum(p);
  if (lane == 0) {
    seg_key[(int64_t)bh * n_q + pos] = float_order_key(p);
    if (trace) trace[level * trace_level_stride + (int64_t)bh * n_q + token] = p;
  }
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

static int levels_of(int G) {
  int L = 0;
  while ((1 << L) < G) ++L;
  return L;
}

template <class T, int D>
static int run_pddp_t(const T* Q, int64_t BH, int n_q, int gs, int32_t* groups, float* trace,
                      const PddpWork& w, cudaStream_t st) {
  const int G = (n_q + gs - 1) / gs;
  const int L = levels_of(G);
  const int64_t total = BH * n_q;
  pddp_init_kernel<<<(unsigned)ceil_div(total, 256), 256, 0, st>>>(w.perm, n_q, total);
  TLSP_TRY(check_launch());
  cudaFuncSetAttribute(pddp_direction_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)direction_smem_bytes<D>());
  for (int level = 0; level < L; ++level) {
    const int nodes = 1 << level;
    const int64_t max_rows = ceil_div(n_q, nodes) + gs;
    int64_t cpn = std::min<int64_t>(ceil_div(max_rows, 256), w.partial_slots / (BH * nodes));
    if (cpn < 2) cpn = 1;
    if (cpn > 1) {
      dim3 grid((unsigned)cpn, (unsigned)nodes, (unsigned)BH);
      pddp_moments_kernel<T, D><<<grid, kMomThreads, 0, st>>>(Q, w.perm, n_q, gs, G, level,
                                                              (int)cpn, w.partials);
      TLSP_TRY(check_launch());
    }
    pddp_direction_kernel<T, D><<<dim3(nodes, (unsigned)BH), kMomThreads,
                                  direction_smem_bytes<D>(), st>>>(
        Q, w.perm, n_q, gs, G, level, (int)cpn, w.partials, w.node_mu, w.node_v);
    TLSP_TRY(check_launch());
    pddp_project_kernel<T, D><<<dim3((unsigned)ceil_div(n_q, 8), (unsigned)BH), 256, 0, st>>>(
        Q, w.perm, n_q, gs, G, level, w.node_mu, w.node_v, w.seg_key, trace, total);
    TLSP_TRY(check_launch());
    pddp_split_kernel<<<dim3(nodes, (unsigned)BH), kSelectThreads, 0, st>>>(
        w.perm, w.tmp, w.seg_key, n_q, gs, G, level);
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
