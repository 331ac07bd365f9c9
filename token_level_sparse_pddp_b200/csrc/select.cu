// Token-level KV selection (per-group top-k) and the single PDDP cut hook.
//
// MC-Sparse review, section 3: each query group keeps the individual KV
// tokens of highest exact score, not whole blocks. Ties go to the lower key
// index and the kept set is listed in ascending key order.
#include "kernels.h"
#include "select.cuh"

namespace tlsp {

// One CTA per score row: the k largest scores (ties: lower index) in
// ascending key order.
__global__ void __launch_bounds__(kSelectThreads)
topk_rows_kernel(const float* __restrict__ scores, int n_kv, int k, int32_t* __restrict__ indices) {
  __shared__ SelectShared sh;
  const int64_t row = blockIdx.x;
  const float* s = scores + row * (int64_t)n_kv;
  int32_t* out = indices + row * (int64_t)k;
  // largest score first == smallest complemented order key
  auto key = [&](int i) -> uint32_t { return ~float_order_key(__ldg(s + i)); };
  select_smallest_ordered(
      key, n_kv, k, sh, [&](uint32_t pos, int i) { out[pos] = i; }, [](uint32_t, int) {});
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
                cudaStream_t stream) {
  if (rows == 0) return TLSP_OK;
  topk_rows_kernel<<<(unsigned)rows, kSelectThreads, 0, stream>>>(scores, n_kv, k, indices);
  return check_launch();
}

int launch_split(const float* proj, const int32_t* members, int n, int n_left, int32_t* left,
                 int32_t* right, cudaStream_t stream) {
  split_kernel<<<1, kSelectThreads, 0, stream>>>(proj, members, n, n_left, left, right);
  return check_launch();
}

}  // namespace tlsp
