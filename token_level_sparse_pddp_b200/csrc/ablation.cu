// Ablation kernels: the pieces MC-Sparse replaces, run on the same library so
// the method can be taken apart one component at a time (the MC-Sparse
// review, section 3 and its ablation table: exact KV selection, token
// granularity, query grouping and residual compensation added one by one on
// top of block-sparse attention with mean-pooled scores).
//
//   raster groups        query groups of consecutive tokens (no PDDP);
//   block top-k          block-granular selection: keys in blocks of b
//                        consecutive tokens, a block scored by the sum of its
//                        keys' exact scores, the k / b best blocks expanded;
//   pooled block scores  the block-sparse baseline's approximate scoring:
//                        (mean of the group's query rows) . (mean of the
//                        block's key rows) / sqrt(d).
// Sparse attention over the expanded blocks is the library's own sparse pass.
#include "kernels.h"
#include "select.cuh"

namespace tlsp {

__global__ void raster_groups_kernel(int32_t* __restrict__ groups, int n_q, int64_t per_head,
                                     int64_t total) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int64_t q = i % per_head;
  groups[i] = q < n_q ? (int32_t)q : -1;
}

int launch_raster_groups(int32_t* groups, int64_t BH, int n_q, int gs, cudaStream_t st) {
  const int64_t G = (n_q + (int64_t)gs - 1) / gs;
  const int64_t total = BH * G * gs;
  if (total == 0) return TLSP_OK;
  raster_groups_kernel<<<(unsigned)ceil_div(total, 256), 256, 0, st>>>(groups, n_q, G * gs, total);
  return check_launch();
}

// One CTA per row of `in` ([rows, n_in] fp32): block scores bs[m] = sum of
// in[m * sum_width .. (m + 1) * sum_width) (in index order; sum_width = 1 takes
// the row as block scores already), the kb blocks of largest score (ties to the
// lower block) in ascending block order, expanded to the kb * b_expand keys
// m * b_expand + t. Block scores are staged in shared memory (and written to
// block_out when given).
__global__ void __launch_bounds__(kSelectThreads)
block_topk_kernel(const float* __restrict__ in, int n_in, int n_blocks, int sum_width, int kb,
                  int b_expand, int32_t* __restrict__ indices, float* __restrict__ block_out) {
  extern __shared__ __align__(128) uint8_t blk_smem[];
  uint32_t* bs = reinterpret_cast<uint32_t*>(blk_smem);
  int32_t* chosen = reinterpret_cast<int32_t*>(blk_smem + (size_t)((n_blocks + 3) & ~3) * 4);
  __shared__ SelectShared sh;
  const int64_t row = blockIdx.x;
  const float* src = in + row * (int64_t)n_in;
  for (int m = threadIdx.x; m < n_blocks; m += kSelectThreads) {
    float s = 0.f;
    for (int t = 0; t < sum_width; ++t) s += src[(int64_t)m * sum_width + t];
    bs[m] = __float_as_uint(s);
    if (block_out) block_out[row * n_blocks + m] = s;
  }
  __syncthreads();
  smem_select_ordered(
      bs, n_blocks, kb, [](uint32_t w) { return ~float_order_key(__uint_as_float(w)); }, sh,
      [&](uint32_t pos, int m) { chosen[pos] = m; }, [](uint32_t, int) {});
  __syncthreads();
  int32_t* out = indices + row * (int64_t)kb * b_expand;
  for (int t = threadIdx.x; t < kb * b_expand; t += kSelectThreads)
    out[t] = chosen[t / b_expand] * b_expand + t % b_expand;
}

size_t block_topk_smem(int n_blocks, int kb) {
  return (size_t)((n_blocks + 3) & ~3) * 4 + (size_t)kb * 4;
}
constexpr int kBlockSmemMax = 200 * 1024;

int launch_block_topk(const float* in, int64_t rows, int n_in, int n_blocks, int sum_width,
                      int kb, int b_expand, int32_t* indices, float* block_out, cudaStream_t st) {
  if (rows == 0) return TLSP_OK;
  const size_t smem = block_topk_smem(n_blocks, kb);
  if (smem > (size_t)kBlockSmemMax || rows > 0x7fffffffLL) return TLSP_ERR_UNSUPPORTED;
  TLSP_TRY(ensure_smem_limit((const void*)block_topk_kernel, kBlockSmemMax));
  block_topk_kernel<<<(unsigned)rows, kSelectThreads, smem, st>>>(in, n_in, n_blocks, sum_width,
                                                                  kb, b_expand, indices, block_out);
  return check_launch();
}

// Mean of the rows `rows(u)` of X for each unit u (one warp per unit; lane l
// takes channels l, l + 32, ...), in fp32, summed in row order.
//   K blocks: unit (bh, m) = key rows m*b .. m*b + b - 1 of head bh;
//   Q groups: unit (bh, g) = the group's member rows (-1 entries skipped).
template <class T>
__global__ void pool_rows_kernel(const T* __restrict__ X, int n_rows, int d, int units_per_head,
                                 int64_t total_units, const int32_t* __restrict__ groups, int gs,
                                 int b, float* __restrict__ out) {
  const int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (u >= total_units) return;
  const int64_t bh = u / units_per_head;
  const int m = (int)(u % units_per_head);
  const T* Xh = X + bh * (int64_t)n_rows * d;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int cnt = 0;
  const int len = groups ? gs : b;
  for (int t = 0; t < len; ++t) {
    int r;
    if (groups) {
      r = groups[(bh * units_per_head + m) * (int64_t)gs + t];
      if (r < 0 || r >= n_rows) continue;
    } else {
      r = m * b + t;
    }
    ++cnt;
    for (int q = 0; q < d / 32; ++q) acc[q] += to_f32(Xh[(int64_t)r * d + lane + 32 * q]);
  }
  const float inv = cnt > 0 ? 1.f / (float)cnt : 0.f;
  for (int q = 0; q < d / 32; ++q) out[u * d + lane + 32 * q] = acc[q] * inv;
}

// Pooled block scores: one CTA per (bh, g); sc[bh, g, m] = Qbar[bh, g] . Kbar[bh, m] * scale,
// each dot product by one thread in channel order.
__global__ void __launch_bounds__(256)
pooled_scores_kernel(const float* __restrict__ Qbar, const float* __restrict__ Kbar, int G,
                     int n_blocks, int d, float scale, float* __restrict__ sc) {
  __shared__ float qs[128];
  const int64_t bg = blockIdx.x;  // bh * G + g
  const int64_t bh = bg / G;
  for (int c = threadIdx.x; c < d; c += blockDim.x) qs[c] = Qbar[bg * d + c];
  __syncthreads();
  for (int m = threadIdx.x; m < n_blocks; m += blockDim.x) {
    const float* kb = Kbar + (bh * n_blocks + m) * d;
    float s = 0.f;
    for (int c = 0; c < d; ++c) s = fmaf(qs[c], kb[c], s);
    sc[bg * n_blocks + m] = s * scale;
  }
}

int launch_pooled_select(const AttnArgs& a, const int32_t* groups, int block, int32_t* indices,
                         float* block_scores, float* scratch, cudaStream_t st) {
  const int n_blocks = a.n_kv / block;
  const int kb = a.k / block;
  float* Kbar = scratch;
  float* Qbar = Kbar + a.BH * (int64_t)n_blocks * a.d;
  float* sc = block_scores ? block_scores : Qbar + a.BH * (int64_t)a.G * a.d;
  const int64_t k_units = a.BH * (int64_t)n_blocks, q_units = a.BH * (int64_t)a.G;
  if (a.bf16) {
    pool_rows_kernel<__nv_bfloat16><<<(unsigned)ceil_div(k_units * 32, 256), 256, 0, st>>>(
        (const __nv_bfloat16*)a.K, a.n_kv, a.d, n_blocks, k_units, nullptr, 0, block, Kbar);
    TLSP_TRY(check_launch());
    pool_rows_kernel<__nv_bfloat16><<<(unsigned)ceil_div(q_units * 32, 256), 256, 0, st>>>(
        (const __nv_bfloat16*)a.Q, a.n_q, a.d, a.G, q_units, groups, a.gs, 0, Qbar);
  } else {
    pool_rows_kernel<float><<<(unsigned)ceil_div(k_units * 32, 256), 256, 0, st>>>(
        (const float*)a.K, a.n_kv, a.d, n_blocks, k_units, nullptr, 0, block, Kbar);
    TLSP_TRY(check_launch());
    pool_rows_kernel<float><<<(unsigned)ceil_div(q_units * 32, 256), 256, 0, st>>>(
        (const float*)a.Q, a.n_q, a.d, a.G, q_units, groups, a.gs, 0, Qbar);
  }
  TLSP_TRY(check_launch());
  pooled_scores_kernel<<<(unsigned)q_units, 256, 0, st>>>(Qbar, Kbar, a.G, n_blocks, a.d,
                                                          1.f / sqrtf((float)a.d), sc);
  TLSP_TRY(check_launch());
  return launch_block_topk(sc, q_units, n_blocks, n_blocks, 1, kb, block, indices, nullptr, st);
}

size_t pooled_scratch_floats(const AttnArgs& a, int block) {
  const int64_t n_blocks = a.n_kv / block;
  return (size_t)(a.BH * n_blocks * a.d + a.BH * (int64_t)a.G * a.d + a.BH * (int64_t)a.G * n_blocks);
}

}  // namespace tlsp
