// Dense attention for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc or hand the library a workspace: code
// running while a CUDA graph is being captured, or inside a framework whose
// memory pool owns every allocation. tlsp_dense_attention_noalloc serves them
// with the scratch it needs (the per-query log partition of the dense pass
// and the device status word) taken from a fixed array that lives in this
// library's own device memory, reserved when the library is loaded and held
// by every GPU that loads it until the process exits.
#include <mutex>

#include "kernels.h"

namespace tlsp {
namespace {

constexpr size_t kStatusBytes = 256;
constexpr size_t kMaxLse = size_t(4) << 20;  // B*H*n_q <= 4,194,304 queries
constexpr size_t kScratchBytes = kStatusBytes + kMaxLse * sizeof(float);  // 16 MiB + 256 B

// Status word at offset 0, the log partitions after it. In host code this
// name is only a stand-in for the symbol, never a device address.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached.
int scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return TLSP_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return TLSP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      set_last_cuda_error(e);
      return TLSP_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TLSP_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace tlsp

using namespace tlsp;

extern "C" int tlsp_dense_attention_noalloc(const tlsp_dims* dims, const void* Q, const void* K,
                                            const void* V, void* O, void* stream) {
  TLSP_TRY(validate_dims(dims));
  if (!Q || !K || !V || !O) return TLSP_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return TLSP_ERR_INVALID_ARG;
  const size_t queries = (size_t)dims->batch * dims->heads * dims->n_q;
  if (queries > kMaxLse) return TLSP_ERR_UNSUPPORTED;  // beyond the fixed scratch
  void* scratch = nullptr;
  TLSP_TRY(scratch_on_current_device(&scratch));
  cudaStream_t st = (cudaStream_t)stream;
  // the status word must start at zero for this call (a memset, not an allocation)
  cudaError_t e = cudaMemsetAsync(scratch, 0, kStatusBytes, st);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return TLSP_ERR_CUDA;
  }
  AttnArgs a;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.BH = (int64_t)dims->batch * dims->heads;
  a.n_q = dims->n_q;
  a.n_kv = dims->n_kv;
  a.d = dims->head_dim;
  a.gs = 1;
  a.G = dims->n_q;
  a.k = 1;
  a.bf16 = dims->dtype == TLSP_BF16;
  a.status = static_cast<int*>(scratch);
  return dense_pass(a, O, reinterpret_cast<float*>(static_cast<char*>(scratch) + kStatusBytes), st);
}
