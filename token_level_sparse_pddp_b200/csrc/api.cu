// C ABI of libtlsp (declared in include/tlsp.h): argument validation,
// workspace layout and dispatch to the kernels.
#include <algorithm>
#include <cstdio>
#include <mutex>
#include <tuple>
#include <vector>

#include "kernels.h"

namespace tlsp {

std::atomic<int64_t> g_launch_count{0};
static thread_local int t_last_cuda_error = 0;
void set_last_cuda_error(cudaError_t e) { t_last_cuda_error = (int)e; }

// ----------------------------------------------------------------- per-device launch facts

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::mutex g_attr_mu;
std::vector<std::tuple<const void*, int, int>> g_attr_done;  // (kernel, device, bytes)

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}
}  // namespace

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

int ensure_smem_limit(const void* fn, int bytes) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_attr_mu);
  for (const auto& t : g_attr_done)
    if (std::get<0>(t) == fn && std::get<1>(t) == dev && std::get<2>(t) >= bytes) return TLSP_OK;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return TLSP_ERR_CUDA;
  }
  g_attr_done.emplace_back(fn, dev, bytes);
  return TLSP_OK;
}

// ----------------------------------------------------------------- workspace

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;  // status word at 0, debug flag at 64
constexpr int64_t kPddpPartialSlots = 640;
// The anchor step scores and selects (head, group) rows in batches of about
// this many score bytes: a batch's scores are still in L2 when the selection
// reads them, and the workspace holds one batch, not every row.
constexpr size_t kScoreBatchBytes = size_t(80) << 20;
constexpr int64_t kBatchRowQuantum = 148;  // whole waves of the score kernel on a B200

static size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Rows (head, group) per score batch: every row when they fit, else as many
// whole waves of kBatchRowQuantum rows as fit in kScoreBatchBytes (at least
// one row; at most 65535, the score launch's limit).
static int64_t score_batch_rows(const tlsp_dims& d, int gs) {
  const int64_t total = (int64_t)d.batch * d.heads * ((d.n_q + gs - 1) / gs);
  int64_t per = (int64_t)(kScoreBatchBytes / (sizeof(float) * (size_t)d.n_kv));
  if (per >= kBatchRowQuantum) per = per / kBatchRowQuantum * kBatchRowQuantum;
  per = std::max<int64_t>(1, std::min<int64_t>(per, 65535));
  return std::min(total, per);
}

struct Layout {
  size_t lse, scores, perm, tmp, seg_key, node_mu, node_v, partials, total;
};

static Layout layout_of(const tlsp_dims& d, int gs) {
  const size_t BH = (size_t)d.batch * d.heads;
  const size_t G = (size_t)((d.n_q + gs - 1) / gs);
  Layout L{};
  size_t off = kStatusBytes;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  L.lse = take(sizeof(float) * BH * d.n_q);
  L.scores = take(sizeof(float) * (size_t)score_batch_rows(d, gs) * d.n_kv);
  L.perm = take(sizeof(int32_t) * BH * d.n_q);
  L.tmp = take(sizeof(int32_t) * BH * d.n_q);
  L.seg_key = take(sizeof(uint32_t) * BH * d.n_q);
  L.node_mu = take(sizeof(float) * BH * G * d.head_dim);
  L.node_v = take(sizeof(float) * BH * G * d.head_dim);
  L.partials = take(sizeof(float) * (size_t)kPddpPartialSlots *
                    ((size_t)d.head_dim * d.head_dim + 2 * d.head_dim));
  L.total = off;
  return L;
}

template <class P>
static P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int validate_dims(const tlsp_dims* d) {
  if (!d) return TLSP_ERR_INVALID_ARG;
  if (d->batch < 1 || d->heads < 1 || d->n_q < 1 || d->n_kv < 1) return TLSP_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return TLSP_ERR_INVALID_ARG;
  if (d->dtype != TLSP_F32 && d->dtype != TLSP_BF16) return TLSP_ERR_INVALID_ARG;
  if ((int64_t)d->batch * d->heads > 65535) return TLSP_ERR_UNSUPPORTED;
  return TLSP_OK;
}

static int validate_grouping(const tlsp_dims* d, int32_t gs) {
  if (gs < 1) return TLSP_ERR_INVALID_ARG;
  const int64_t G = (d->n_q + (int64_t)gs - 1) / gs;
  if (G > 65535) return TLSP_ERR_UNSUPPORTED;
  return TLSP_OK;
}

static int check_ws(const tlsp_dims* d, int32_t gs, void* ws, size_t ws_bytes) {
  if (!ws || !aligned16(ws)) return TLSP_ERR_INVALID_ARG;
  if (ws_bytes < layout_of(*d, gs).total) return TLSP_ERR_WORKSPACE;
  return TLSP_OK;
}

static AttnArgs attn_args(const tlsp_dims* d, const void* Q, const void* K, const void* V,
                          int32_t gs, int32_t k, void* ws) {
  AttnArgs a;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.BH = (int64_t)d->batch * d->heads;
  a.n_q = d->n_q;
  a.n_kv = d->n_kv;
  a.d = d->head_dim;
  a.gs = gs;
  a.G = (d->n_q + gs - 1) / gs;
  a.k = k;
  a.bf16 = d->dtype == TLSP_BF16;
  a.status = at<int>(ws, 0);
  return a;
}

__global__ void bounded_wait_kernel(volatile int* flag, int* status, int64_t spin_limit) {
  for (int64_t i = 0; i < spin_limit; ++i) {
    if (*flag != 0) return;
    __nanosleep(32);
  }
  record_status(status, TLSP_ERR_TIMEOUT);
}

static int group_impl(const tlsp_dims* dims, const void* Q, int32_t gs, int32_t* groups,
                      float* proj, void* ws, size_t ws_bytes, void* stream) {
  TLSP_TRY(validate_dims(dims));
  TLSP_TRY(validate_grouping(dims, gs));
  if (!Q || !groups || !aligned16(Q)) return TLSP_ERR_INVALID_ARG;
  TLSP_TRY(check_ws(dims, gs, ws, ws_bytes));
  const Layout L = layout_of(*dims, gs);
  const int64_t BH = (int64_t)dims->batch * dims->heads;
  cudaStream_t st = (cudaStream_t)stream;
  if (proj) {
    const int levels = tlsp_num_levels(dims->n_q, gs);
    if (levels > 0) {
      cudaError_t e = cudaMemsetAsync(proj, 0, sizeof(float) * levels * BH * dims->n_q, st);
      if (e != cudaSuccess) {
        set_last_cuda_error(e);
        return TLSP_ERR_CUDA;
      }
    }
  }
  PddpWork w{at<int32_t>(ws, L.perm),    at<int32_t>(ws, L.tmp),   at<uint32_t>(ws, L.seg_key),
             at<float>(ws, L.node_mu),   at<float>(ws, L.node_v),  at<float>(ws, L.partials),
             kPddpPartialSlots,          at<int>(ws, 0)};
  return run_pddp(Q, dims->dtype == TLSP_BF16, dims->head_dim, BH, dims->n_q, gs, groups, proj, w,
                  st);
}

}  // namespace tlsp

using namespace tlsp;

extern "C" {

int32_t tlsp_num_groups(int32_t n_q, int32_t group_size) {
  if (n_q < 1 || group_size < 1) return -1;
  return (int32_t)(((int64_t)n_q + group_size - 1) / group_size);
}

int32_t tlsp_num_levels(int32_t n_q, int32_t group_size) {
  const int32_t G = tlsp_num_groups(n_q, group_size);
  if (G < 1) return -1;
  int32_t L = 0;
  while ((int64_t(1) << L) < G) ++L;
  return L;
}

size_t tlsp_workspace_bytes(const tlsp_dims* dims, int32_t group_size, int32_t k) {
  if (validate_dims(dims) != TLSP_OK || validate_grouping(dims, group_size) != TLSP_OK) return 0;
  if (k < 1 || k > dims->n_kv) return 0;
  return layout_of(*dims, group_size).total;
}

int tlsp_group_queries(const tlsp_dims* dims, const void* Q, int32_t group_size, int32_t* groups,
                       void* ws, size_t ws_bytes, void* stream) {
  return group_impl(dims, Q, group_size, groups, nullptr, ws, ws_bytes, stream);
}

int tlsp_group_queries_trace(const tlsp_dims* dims, const void* Q, int32_t group_size,
                             int32_t* groups, float* proj, void* ws, size_t ws_bytes,
                             void* stream) {
  if (!proj) return TLSP_ERR_INVALID_ARG;
  return group_impl(dims, Q, group_size, groups, proj, ws, ws_bytes, stream);
}

int tlsp_split_from_projections(const float* proj, const int32_t* members, int32_t n,
                                int32_t n_left, int32_t* left_out, int32_t* right_out,
                                void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (!proj || !members || n < 1 || n_left < 0 || n_left > n) return TLSP_ERR_INVALID_ARG;
  if ((n_left > 0 && !left_out) || (n_left < n && !right_out)) return TLSP_ERR_INVALID_ARG;
  return launch_split(proj, members, n, n_left, left_out, right_out, (cudaStream_t)stream);
}

int tlsp_anchor_attention(const tlsp_dims* dims, const void* Q, const void* K, const void* V,
                          const int32_t* groups, int32_t group_size, int32_t k, void* O,
                          int32_t* indices, float* R, float* scores, void* ws, size_t ws_bytes,
                          void* stream) {
  TLSP_TRY(validate_dims(dims));
  TLSP_TRY(validate_grouping(dims, group_size));
  if (k < 1 || k > dims->n_kv) return TLSP_ERR_INVALID_ARG;
  if (!Q || !K || !V || !groups || !O || !indices || !R) return TLSP_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(R))
    return TLSP_ERR_INVALID_ARG;
  TLSP_TRY(check_ws(dims, group_size, ws, ws_bytes));
  const Layout L = layout_of(*dims, group_size);
  cudaStream_t st = (cudaStream_t)stream;
  const AttnArgs a = attn_args(dims, Q, K, V, group_size, k, ws);
  float* lse = at<float>(ws, L.lse);
  TLSP_TRY(dense_pass(a, O, lse, st));
  // exact scores and the top-k selection, batch by batch of (head, group) rows
  const int64_t total = a.BH * a.G, per = score_batch_rows(*dims, group_size);
  for (int64_t r0 = 0; r0 < total; r0 += per) {
    const int64_t rows = std::min(per, total - r0);
    float* S = scores ? scores + r0 * a.n_kv : at<float>(ws, L.scores);
    TLSP_TRY(scores_pass(a, groups, lse, S, r0, rows, st));
    TLSP_TRY(launch_topk(S, rows, a.n_kv, k, indices + r0 * k, a.status, st));
  }
  return sparse_pass(a, groups, indices, O, R, nullptr, nullptr, st);
}

int tlsp_dense_attention(const tlsp_dims* dims, const void* Q, const void* K, const void* V,
                         void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  TLSP_TRY(validate_dims(dims));
  if (!Q || !K || !V || !O) return TLSP_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return TLSP_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return TLSP_ERR_INVALID_ARG;
  const size_t lse_bytes = sizeof(float) * (size_t)dims->batch * dims->heads * dims->n_q;
  if (ws_bytes < kStatusBytes + (lse ? 0 : lse_bytes)) return TLSP_ERR_WORKSPACE;
  const AttnArgs a = attn_args(dims, Q, K, V, 1, 1, ws);
  return dense_pass(a, O, lse ? lse : at<float>(ws, kStatusBytes), (cudaStream_t)stream);
}

int tlsp_reuse_attention(const tlsp_dims* dims, const void* Q, const void* K, const void* V,
                         const int32_t* groups, int32_t group_size, int32_t k,
                         const int32_t* indices, const float* R, void* O, void* ws,
                         size_t ws_bytes, void* stream) {
  TLSP_TRY(validate_dims(dims));
  TLSP_TRY(validate_grouping(dims, group_size));
  if (k < 1 || k > dims->n_kv) return TLSP_ERR_INVALID_ARG;
  if (!Q || !K || !V || !groups || !O || !indices || !R) return TLSP_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(R))
    return TLSP_ERR_INVALID_ARG;
  // the reuse step's only scratch is the status word
  if (!ws || !aligned16(ws)) return TLSP_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes) return TLSP_ERR_WORKSPACE;
  const AttnArgs a = attn_args(dims, Q, K, V, group_size, k, ws);
  return sparse_pass(a, groups, indices, nullptr, nullptr, R, O, (cudaStream_t)stream);
}

int tlsp_topk_from_scores(const float* scores, int32_t rows, int32_t n_kv, int32_t k,
                          int32_t* indices, void* ws, size_t ws_bytes, void* stream) {
  if (!scores || !indices || rows < 0 || n_kv < 1 || k < 1 || k > n_kv)
    return TLSP_ERR_INVALID_ARG;
  if (ws && (!aligned16(ws) || ws_bytes < kStatusBytes)) return TLSP_ERR_INVALID_ARG;
  int* status = ws ? at<int>(ws, 0) : nullptr;
  return launch_topk(scores, rows, n_kv, k, indices, status, (cudaStream_t)stream);
}

int tlsp_group_raster(const tlsp_dims* dims, int32_t group_size, int32_t* groups, void* stream) {
  TLSP_TRY(validate_dims(dims));
  TLSP_TRY(validate_grouping(dims, group_size));
  if (!groups) return TLSP_ERR_INVALID_ARG;
  return launch_raster_groups(groups, (int64_t)dims->batch * dims->heads, dims->n_q, group_size,
                              (cudaStream_t)stream);
}

int tlsp_block_topk_from_scores(const float* scores, int32_t rows, int32_t n_kv, int32_t k,
                                int32_t block, int32_t* indices, float* block_scores,
                                void* stream) {
  if (!scores || !indices || rows < 0 || n_kv < 1 || k < 1 || k > n_kv || block < 1)
    return TLSP_ERR_INVALID_ARG;
  if (n_kv % block != 0 || k % block != 0) return TLSP_ERR_UNSUPPORTED;
  return launch_block_topk(scores, rows, n_kv, n_kv / block, block, k / block, block, indices,
                           block_scores, (cudaStream_t)stream);
}

int tlsp_pooled_block_select(const tlsp_dims* dims, const void* Q, const void* K,
                             const int32_t* groups, int32_t group_size, int32_t k, int32_t block,
                             int32_t* indices, float* block_scores, void* ws, size_t ws_bytes,
                             void* stream) {
  TLSP_TRY(validate_dims(dims));
  TLSP_TRY(validate_grouping(dims, group_size));
  if (!Q || !K || !groups || !indices || k < 1 || k > dims->n_kv || block < 1)
    return TLSP_ERR_INVALID_ARG;
  if (dims->n_kv % block != 0 || k % block != 0) return TLSP_ERR_UNSUPPORTED;
  TLSP_TRY(check_ws(dims, group_size, ws, ws_bytes));
  const Layout L = layout_of(*dims, group_size);
  const AttnArgs a = attn_args(dims, Q, K, nullptr, group_size, k, ws);
  // Pooled rows and block scores go to the workspace's chunk-moment region
  // (grouping scratch, idle during selection).
  if (pooled_scratch_floats(a, block) * sizeof(float) > L.total - L.partials)
    return TLSP_ERR_WORKSPACE;
  return launch_pooled_select(a, groups, block, indices, block_scores, at<float>(ws, L.partials),
                              (cudaStream_t)stream);
}

int tlsp_get_device_status(const void* ws) {
  if (!ws) return TLSP_ERR_INVALID_ARG;
  int code = 0;
  cudaError_t e = cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return TLSP_ERR_CUDA;
  }
  return code;
}

int tlsp_reset_device_status(void* ws, void* stream) {
  if (!ws) return TLSP_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    set_last_cuda_error(e);
    return TLSP_ERR_CUDA;
  }
  return TLSP_OK;
}

int tlsp_debug_bounded_wait(void* ws, size_t ws_bytes, int64_t spin_limit, void* stream) {
  if (!ws || ws_bytes < kStatusBytes || spin_limit < 0) return TLSP_ERR_INVALID_ARG;
  bounded_wait_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(at<volatile int>(ws, 64), at<int>(ws, 0),
                                                         spin_limit);
  return check_launch();
}

const char* tlsp_status_string(int status) {
  switch (status) {
    case TLSP_OK: return "TLSP_OK";
    case TLSP_ERR_INVALID_ARG: return "TLSP_ERR_INVALID_ARG";
    case TLSP_ERR_UNSUPPORTED: return "TLSP_ERR_UNSUPPORTED";
    case TLSP_ERR_WORKSPACE: return "TLSP_ERR_WORKSPACE";
    case TLSP_ERR_CUDA: return "TLSP_ERR_CUDA";
    case TLSP_ERR_TIMEOUT: return "TLSP_ERR_TIMEOUT";
    case TLSP_ERR_DEVICE_ASSERT: return "TLSP_ERR_DEVICE_ASSERT";
    default: return "TLSP_UNKNOWN_STATUS";
  }
}

int tlsp_last_cuda_error(void) { return t_last_cuda_error; }

int64_t tlsp_launch_count(void) { return g_launch_count.load(); }

}  // extern "C"
