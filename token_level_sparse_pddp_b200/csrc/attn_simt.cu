// CUDA-core (SIMT) attention kernels: dense pass, exact group scores and
// gathered sparse pass with the residual epilogues. They compute in fp32 and
// serve fp32 inputs (where bf16 tensor-core products would miss a 1e-4
// tolerance) and any head_dim/group_size the tensor-core kernels do not take.
//
// MC-Sparse review, section 3: anchor step = dense output, exact per-group KV
// scores, top-k selection and R = O_full - O_sparse; reuse step = sparse
// attention over the cached selection + R.
//
// Pattern of the two attention loops: one warp per query row; for 32 keys at
// a time each lane forms one logit (lane-per-key dot product against the row
// staged in shared memory), the warp updates the running max / sum (online
// softmax), and the P V product is accumulated with each lane owning D/32
// output channels.
#include "kernels.h"

namespace tlsp {

constexpr int kSimtWarps = 4;

template <class T, int D>
__device__ __forceinline__ float dot_row(const float* __restrict__ q_s, const T* __restrict__ k) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < D; c += 8) {
    float kv[8];
    load8(k + c, kv);
#pragma unroll
    for (int e = 0; e < 8; ++e) s = fmaf(q_s[c + e], kv[e], s);
  }
  return s;
}

// Online-softmax attention of one query row (staged in q_s) over keys
// key_id(0..n-1). Returns o (lane-owned channels c = lane + 32*e), m and l.
template <class T, int D, class KeyId>
__device__ __forceinline__ void row_attention(const float* q_s, const T* __restrict__ K,
                                              const T* __restrict__ V, int n, KeyId key_id,
                                              float scale, float (&o)[D / 32], float& m,
                                              float& l) {
  const int lane = threadIdx.x & 31;
  m = -INFINITY;
  l = 0.f;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) o[e] = 0.f;
  for (int t0 = 0; t0 < n; t0 += 32) {
    const int t = t0 + lane;
    const int j = t < n ? key_id(t) : -1;
    float s = -INFINITY;
    if (j >= 0) s = dot_row<T, D>(q_s, K + (int64_t)j * D) * scale;
    const float m_new = fmaxf(m, warp_max(s));
    if (m_new == -INFINITY) continue;  // no valid key seen yet (warp-uniform)
    const float p = (j >= 0) ? expf(s - m_new) : 0.f;
    const float corr = expf(m - m_new);  // m = -inf before the first valid key -> 0
    l = l * corr + warp_sum(p);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) o[e] *= corr;
    const int cnt = min(32, n - t0);
    for (int u = 0; u < cnt; ++u) {
      const float pu = __shfl_sync(0xffffffffu, p, u);
      const int ju = __shfl_sync(0xffffffffu, j, u);
      if (ju < 0) continue;
      const T* v = V + (int64_t)ju * D;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) o[e] = fmaf(pu, to_f32(v[lane + 32 * e]), o[e]);
    }
    m = m_new;
  }
}

// Dense attention: O [bh, n_q, D] in T, LSE [bh, n_q] fp32.
template <class T, int D>
__global__ void __launch_bounds__(kSimtWarps * 32)
dense_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                  int n_q, int n_kv, float scale, T* __restrict__ O, float* __restrict__ LSE) {
  __shared__ __align__(16) float q_s[kSimtWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kSimtWarps + warp;
  const int64_t bh = blockIdx.y;
  if (i >= n_q) return;
  const T* q = Q + (bh * n_q + i) * D;
  for (int c = lane; c < D; c += 32) q_s[warp][c] = to_f32(q[c]);
  __syncwarp();
  float o[D / 32], m, l;
  row_attention<T, D>(q_s[warp], K + bh * n_kv * D, V + bh * n_kv * D, n_kv,
                      [](int t) { return t; }, scale, o, m, l);
  const float inv = 1.f / l;
  T* out = O + (bh * n_q + i) * D;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) out[lane + 32 * e] = from_f32<T>(o[e] * inv);
  if (lane == 0) LSE[bh * n_q + i] = m + logf(l);
}

// Exact group scores: S[bh, g, j] = sum_{i in g} exp(q_i . k_j * scale - LSE_i).
// One thread per key, the group's rows staged 32 at a time in shared memory.
template <class T, int D>
__global__ void __launch_bounds__(128)
scores_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const float* __restrict__ LSE,
                   const int32_t* __restrict__ groups, int n_q, int n_kv, int gs, int G,
                   int64_t row0, float scale, float* __restrict__ S, int* status) {
  __shared__ __align__(16) float q_s[32][D];
  __shared__ float lse_s[32];
  const int64_t grow = row0 + blockIdx.y;  // (head, group) row; S holds this launch's rows
  const int g = (int)(grow % G);
  const int64_t bh = grow / G;
  const int j = blockIdx.x * 128 + threadIdx.x;
  const int32_t* grp = groups + (bh * G + g) * (int64_t)gs;
  const T* kj = K + (bh * n_kv + min(j, n_kv - 1)) * D;
  float acc = 0.f;
  for (int r0 = 0; r0 < gs; r0 += 32) {
    const int nr = min(32, gs - r0);
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * D; e += 128) {
      const int r = e / D, c = e % D;
      int tok = r < nr ? grp[r0 + r] : -1;
      if (tok >= n_q) {
        record_status(status, TLSP_ERR_DEVICE_ASSERT);
        tok = -1;
      }
      q_s[r][c] = tok >= 0 ? to_f32(Q[(bh * n_q + tok) * D + c]) : 0.f;
      if (c == 0) lse_s[r] = tok >= 0 ? LSE[bh * n_q + tok] : INFINITY;  // padding: exp(-inf) = 0
    }
    __syncthreads();
    if (j < n_kv) {
      for (int r = 0; r < nr; ++r) {
        const float s = dot_row<T, D>(q_s[r], kj) * scale;
        acc += expf(s - lse_s[r]);
      }
    }
  }
  if (j < n_kv) S[(int64_t)blockIdx.y * n_kv + j] = acc;
}

// Gathered sparse attention over indices[bh, g, 0..k) with the residual
// epilogues: kAnchor writes R = O_full - O_sp (fp32), otherwise
// O = O_sp + R (in T).
template <class T, int D, bool kAnchor>
__global__ void __launch_bounds__(kSimtWarps * 32)
sparse_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                   const int32_t* __restrict__ groups, const int32_t* __restrict__ indices,
                   int n_q, int n_kv, int gs, int G, int k, float scale,
                   const T* __restrict__ O_full, float* __restrict__ R_out,
                   const float* __restrict__ R_in, T* __restrict__ O_out, int* status) {
  __shared__ __align__(16) float q_s[kSimtWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kSimtWarps + warp;
  const int g = blockIdx.y;
  const int64_t bh = blockIdx.z;
  if (r >= gs) return;
  const int tok = groups[(bh * G + g) * (int64_t)gs + r];
  // members of a group are token ids in [0, n_q); only the ragged tail of
  // the last group holds padding, and padding is -1
  const int members = g == G - 1 ? n_q - (G - 1) * gs : gs;
  if (r < members ? (tok < 0 || tok >= n_q) : tok != -1) {
    if (lane == 0) record_status(status, TLSP_ERR_DEVICE_ASSERT);
    return;
  }
  if (tok < 0) return;  // padding row of the ragged last group
  const T* q = Q + (bh * n_q + tok) * D;
  for (int c = lane; c < D; c += 32) q_s[warp][c] = to_f32(q[c]);
  __syncwarp();
  const int32_t* sel = indices + (bh * G + g) * (int64_t)k;
  float o[D / 32], m, l;
  row_attention<T, D>(
      q_s[warp], K + bh * n_kv * D, V + bh * n_kv * D, k,
      [&](int t) {
        const int j = sel[t];
        if ((unsigned)j >= (unsigned)n_kv) {
          record_status(status, TLSP_ERR_DEVICE_ASSERT);
          return -1;
        }
        return j;
      },
      scale, o, m, l);
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const int64_t row = (bh * n_q + tok) * D;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) {
    const int c = lane + 32 * e;
    const float osp = o[e] * inv;
    if (kAnchor)
      R_out[row + c] = to_f32(O_full[row + c]) - osp;
    else
      O_out[row + c] = from_f32<T>(osp + R_in[row + c]);
  }
}

// ----------------------------------------------------------------- launchers

template <class T, int D>
static int dense_t(const AttnArgs& a, void* O, float* LSE, cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(a.n_q, kSimtWarps), (unsigned)a.BH);
  dense_simt_kernel<T, D><<<grid, kSimtWarps * 32, 0, st>>>(
      (const T*)a.Q, (const T*)a.K, (const T*)a.V, a.n_q, a.n_kv, rsqrtf((float)D), (T*)O, LSE);
  return check_launch();
}

template <class T, int D>
static int scores_t(const AttnArgs& a, const int32_t* groups, const float* LSE, float* S,
                    int64_t row0, int64_t rows, cudaStream_t st) {
  if (rows <= 0) return TLSP_OK;
  if (rows > 65535) return TLSP_ERR_UNSUPPORTED;
  dim3 grid((unsigned)ceil_div(a.n_kv, 128), (unsigned)rows);
  scores_simt_kernel<T, D><<<grid, 128, 0, st>>>((const T*)a.Q, (const T*)a.K, LSE, groups, a.n_q,
                                                 a.n_kv, a.gs, a.G, row0, rsqrtf((float)D), S,
                                                 a.status);
  return check_launch();
}

template <class T, int D>
static int sparse_t(const AttnArgs& a, const int32_t* groups, const int32_t* indices,
                    const void* O_full, float* R_out, const float* R_in, void* O_out,
                    cudaStream_t st) {
  dim3 grid((unsigned)ceil_div(a.gs, kSimtWarps), (unsigned)a.G, (unsigned)a.BH);
  if (R_out)
    sparse_simt_kernel<T, D, true><<<grid, kSimtWarps * 32, 0, st>>>(
        (const T*)a.Q, (const T*)a.K, (const T*)a.V, groups, indices, a.n_q, a.n_kv, a.gs, a.G,
        a.k, rsqrtf((float)D), (const T*)O_full, R_out, nullptr, nullptr, a.status);
  else
    sparse_simt_kernel<T, D, false><<<grid, kSimtWarps * 32, 0, st>>>(
        (const T*)a.Q, (const T*)a.K, (const T*)a.V, groups, indices, a.n_q, a.n_kv, a.gs, a.G,
        a.k, rsqrtf((float)D), nullptr, nullptr, R_in, (T*)O_out, a.status);
  return check_launch();
}

#define TLSP_DISPATCH(fn, ...)                                                       \
  (a.bf16 ? (a.d == 128 ? fn<__nv_bfloat16, 128>(__VA_ARGS__)                        \
                        : fn<__nv_bfloat16, 64>(__VA_ARGS__))                        \
          : (a.d == 128 ? fn<float, 128>(__VA_ARGS__) : fn<float, 64>(__VA_ARGS__)))

int simt_dense(const AttnArgs& a, void* O, float* LSE, cudaStream_t st) {
  return TLSP_DISPATCH(dense_t, a, O, LSE, st);
}
int simt_scores(const AttnArgs& a, const int32_t* groups, const float* LSE, float* S,
                int64_t row0, int64_t rows, cudaStream_t st) {
  return TLSP_DISPATCH(scores_t, a, groups, LSE, S, row0, rows, st);
}
int simt_sparse(const AttnArgs& a, const int32_t* groups, const int32_t* indices,
                const void* O_full, float* R_out, const float* R_in, void* O_out,
                cudaStream_t st) {
  return TLSP_DISPATCH(sparse_t, a, groups, indices, O_full, R_out, R_in, O_out, st);
}

}  // namespace tlsp
