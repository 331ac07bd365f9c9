// Token-level KV selection (per-group top-k) and the single PDDP cut hook.
//
// MC-Sparse review, section 3: each query group keeps the individual KV
// tokens of highest exact score, not whole blocks. Ties go to the lower key
// index and the kept set is listed in ascending key order.
#include <algorithm>

#include "kernels.h"
#include "select.cuh"
#include "tc_ptx.cuh"

namespace tlsp {

// One CTA per score row: the k largest scores (ties: lower index) in
// ascending key order. Keys are read from global memory on every pass; used
// when a row does not fit in shared memory.
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

constexpr int kTopkSmemKeys = 52 * 1024;  // rows up to 52K keys are staged (208 KB)
constexpr uint32_t kBulkChunk = 32768;
constexpr uint64_t kTopkWaitNs = 1000000000ull;

__device__ __forceinline__ uint32_t topk_key(uint32_t w) {
  // largest score first == smallest complemented order key
  return ~float_order_key(__uint_as_float(w));
}

// Persistent variant: each CTA stages one score row at a time in shared
// memory (a bulk copy when rows are 16-byte aligned, else plain loads), so the
// row crosses HBM once and every pass of the selection reads shared memory.
// Dynamic shared memory: the row, rounded up to 4 words.
__global__ void __launch_bounds__(kSelectThreads, 1)
topk_rows_smem_kernel(const float* __restrict__ scores, int64_t rows, int n_kv, int k,
                      int32_t* __restrict__ indices, int* status) {
  extern __shared__ __align__(128) uint8_t topk_smem[];
  uint32_t* buf = reinterpret_cast<uint32_t*>(topk_smem);
  __shared__ SelectShared sh;
  __shared__ uint64_t bar;
  const int t = threadIdx.x;
  const bool bulk = (n_kv % 4) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15u) == 0;
  if (t == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  uint32_t phase = 0;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const float* s = scores + row * (int64_t)n_kv;
    if (bulk) {
      if (t == 0) {
        const uint32_t bytes = (uint32_t)n_kv * 4u;
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive_expect_tx(&bar, bytes);
        for (uint32_t off = 0; off < bytes; off += kBulkChunk)
          ptx::bulk_load(ptx::smem_u32(topk_smem) + off, reinterpret_cast<const uint8_t*>(s) + off,
                         min(kBulkChunk, bytes - off), &bar);
      }
      const bool ok = ptx::mbar_wait(&bar, phase, nullptr, kTopkWaitNs);
      phase ^= 1u;
      if (__syncthreads_or(!ok)) {
        if (t == 0) record_status(status, TLSP_ERR_TIMEOUT);
        return;
      }
    } else {
      for (int i = t; i < n_kv; i += kSelectThreads) buf[i] = __float_as_uint(__ldg(s + i));
      __syncthreads();
    }
    int32_t* out = indices + row * (int64_t)k;
    smem_select_ordered(
        buf, n_kv, k, [](uint32_t w) { return topk_key(w); }, sh,
        [&](uint32_t pos, int i) { out[pos] = i; }, [](uint32_t, int) {});
    __syncthreads();  // the row buffer is free for the next row
  }
}

size_t topk_smem_bytes(int n_kv) { return (size_t)((n_kv + 3) & ~3) * 4; }

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
  if (rows == 0) return TLSP_OK;
  if (n_kv <= kTopkSmemKeys) {
    const size_t smem = topk_smem_bytes(n_kv);
    cudaFuncSetAttribute(topk_rows_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)topk_smem_bytes(kTopkSmemKeys));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = std::min<int64_t>(rows, sms);
    topk_rows_smem_kernel<<<(unsigned)grid, kSelectThreads, smem, stream>>>(scores, rows, n_kv, k,
                                                                           indices, status);
    return check_launch();
  }
  topk_rows_kernel<<<(unsigned)rows, kSelectThreads, 0, stream>>>(scores, n_kv, k, indices);
  return check_launch();
}

int launch_split(const float* proj, const int32_t* members, int n, int n_left, int32_t* left,
                 int32_t* right, cudaStream_t stream) {
  split_kernel<<<1, kSelectThreads, 0, stream>>>(proj, members, n, n_left, left, right);
  return check_launch();
}

}  // namespace tlsp
