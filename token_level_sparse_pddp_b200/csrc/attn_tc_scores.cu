// Exact per-group KV scores on the sm_100a tensor cores (bf16, head_dim 128).
//
// MC-Sparse review, section 3: on the anchor step each query group selects
// its KV tokens from exact attention scores (not mean-pooled estimates). The
// score of key j for group g is the attention mass the group puts on it,
// S_g[j] = sum_{i in g} exp(q_i . k_j / sqrt(d) - LSE_i), with LSE_i the log
// partition of query i from the dense pass.
//
// One CTA per (head, group) for groups of at most 128 queries. The CTA keeps
// the group's Q rows in shared memory and streams all keys in chunks of 128
// with TMA box loads (four slots). The product is taken transposed,
// S^T = K_chunk Q_g^T (M = 128 keys on TMEM lanes, N = 128 queries on TMEM
// columns), so thread t (lane t) owns key j0 + t and sums its own lane:
// no cross-thread reduction and no atomics; the per-query LSE (in log2 units)
// is a shared-memory broadcast. S^T is double-buffered in TMEM so the next
// chunk's MMA runs while a chunk is summed.
// Warp roles (416 threads): warps 0-3 and 4-7 sum (lane t of both warps w
// and w + 4 is key j0 + 32 (w % 4) + t; warps 0-3 take the group's query
// columns 0-63 and warps 4-7 columns 64-127, so two warps per SM sub-partition
// hide each other's TMEM and SFU latency); warps 4-7 hand their partial sums
// to warps 0-3 through a double-buffered shared-memory slot, and warps 0-3
// store the total. Warps 8-11 gather Q_g with 16-byte cp.async (128-byte
// swizzle), then lane 0 of warp 8 issues the K loads; warp 12 allocates TMEM
// and lane 0 issues tcgen05.mma.
// Every wait is bounded (1 s); on expiry the kernel records TLSP_ERR_TIMEOUT
// and unwinds.
#include "kernels.h"
#include "tc_ptx.cuh"

namespace tlsp {
namespace {

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kThreads = 416;
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr int kKSlots = 4;
constexpr uint32_t kSmQ = 0, kSmK = kTileBytes;
constexpr uint32_t kSmBar = (1 + kKSlots) * kTileBytes;
constexpr uint32_t kSmLse = kSmBar + 256;
constexpr uint32_t kSmX = kSmLse + kTile * 4;  // partial sums, 2 x 128 floats
constexpr uint32_t kSmemBytes = kSmX + 2 * kTile * 4 + 1024;
constexpr uint32_t kTmCols = 256;
constexpr uint64_t kWaitNs = 1000000000ull;

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t s_full[2], s_empty[2];
  uint64_t x_full[2], x_empty[2];  // partial sums of warps 4-7 -> warps 0-3
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct ScoreParams {
  CUtensorMap tmK;  // [BH*n_kv, 128] bf16, box 64 x 128, 128-byte swizzle
  const __nv_bfloat16* __restrict__ Q;
  const int32_t* __restrict__ groups;
  const float* __restrict__ lse;
  float* __restrict__ S;
  int n_q, n_kv, gs, G;
  float scale_log2;
  int* status;
};

__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(c >> 3) * kHalfBytes + (uint32_t)r * 128u +
         ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void fail(Bars& b, int* status) {
  b.abort = 1;
  record_status(status, TLSP_ERR_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1)
    scores_tc_kernel(const __grid_constant__ ScoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  Bars& bars = *reinterpret_cast<Bars*>(smem + kSmBar);
  float* lse2_s = reinterpret_cast<float*>(smem + kSmLse);
  volatile int* abort_flag = &bars.abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = blockIdx.x / p.G;
  const int g = blockIdx.x % p.G;
  const int32_t* grp = p.groups + (bh * p.G + g) * (int64_t)p.gs;
  const int n_chunks = (p.n_kv + kTile - 1) / kTile;

  if (tid == 0) {
    ptx::mbar_init(&bars.q_full, 128);
    for (int s = 0; s < kKSlots; ++s) {
      ptx::mbar_init(&bars.k_full[s], 1);
      ptx::mbar_init(&bars.k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars.s_full[s], 1);
      ptx::mbar_init(&bars.s_empty[s], 256);
      ptx::mbar_init(&bars.x_full[s], 128);
      ptx::mbar_init(&bars.x_empty[s], 128);
    }
    ptx::mbar_init(&bars.drain, 1);
    bars.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 12) {
    ptx::tmem_alloc(&bars.tmem_base, kTmCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------ producers
    const int pt = tid - 256;
    const __nv_bfloat16* Qbh = p.Q + bh * (int64_t)p.n_q * kD;
    const int c = pt & 15;
#pragma unroll 1
    for (int b = 0; b < 16; b += 8) {
      int rows[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = (b + i) * 8 + (pt >> 4);
        int tok = r < p.gs ? __ldg(grp + r) : -1;
        if (tok >= p.n_q) {
          record_status(p.status, TLSP_ERR_DEVICE_ASSERT);
          tok = -1;
        }
        rows[i] = tok;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = (b + i) * 8 + (pt >> 4);
        const __nv_bfloat16* s = Qbh + (rows[i] >= 0 ? (int64_t)rows[i] * kD + c * 8 : 0);
        ptx::cp_async16(base + kSmQ + swz(r, c), s, rows[i] >= 0 ? 16u : 0u);
      }
    }
    ptx::cp_async_arrive_noinc(&bars.q_full);
    if (warp == 8 && lane == 0) {
      const int kv_row = (int)(bh * p.n_kv);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n_chunks; ++j) {
        const int s = j % kKSlots, u = j / kKSlots;
        if (u > 0 && !ptx::mbar_wait(&bars.k_empty[s], (u - 1) & 1, abort_flag, kWaitNs)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars.k_full[s], kTileBytes);
        const uint32_t dst = base + kSmK + s * kTileBytes;
        ptx::tma_load_2d(dst, &p.tmK, 0, kv_row + j * kTile, &bars.k_full[s]);
        ptx::tma_load_2d(dst + kHalfBytes, &p.tmK, 64, kv_row + j * kTile, &bars.k_full[s]);
        issued = j + 1;
      }
      if (!ok) {
        fail(bars, p.status);
        for (int j = max(0, issued - kKSlots); j < issued; ++j)
          ptx::mbar_wait(&bars.k_full[j % kKSlots], (j / kKSlots) & 1, nullptr, kWaitNs);
      }
    }
    ptx::cp_async_wait_all();
  } else if (warp == 12) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16(kTile, kTile, false);
      bool ok = ptx::mbar_wait(&bars.q_full, 0, abort_flag, kWaitNs);
      for (int j = 0; j < n_chunks && ok; ++j) {
        const int s = j & 1, ks = j % kKSlots;
        if (j >= 2) ok = ptx::mbar_wait(&bars.s_empty[s], ((j >> 1) - 1) & 1, abort_flag, kWaitNs);
        ok = ok && ptx::mbar_wait(&bars.k_full[ks], (j / kKSlots) & 1, abort_flag, kWaitNs);
        if (!ok) break;
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_after();
        const uint32_t kb = base + kSmK + ks * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kHalfBytes + (uint32_t)(kk & 3) * 32u;
          // D[key][query] = K[key] . Q[query]: A = K chunk, B = Q_g, both K-major
          ptx::mma_ss(tmem + s * kTile, ptx::sw128_desc(kb + off, 16, 1024),
                      ptx::sw128_desc(base + kSmQ + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        ptx::tc_commit(&bars.s_full[s]);
        ptx::tc_commit(&bars.k_empty[ks]);
      }
      if (!ok) fail(bars, p.status);
      ptx::tc_commit(&bars.drain);
      ptx::mbar_wait(&bars.drain, 0, nullptr, kWaitNs);  // even after an abort
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ sums
    const int r = tid & 127, half = warp >> 2;  // key lane r, query columns 64*half ..
    float* xs = reinterpret_cast<float*>(smem + kSmX);
    if (half == 0) {
      // log2-unit LSE of the group's queries; padding rows contribute exp2(-inf) = 0
      const int tok = r < p.gs ? grp[r] : -1;
      lse2_s[r] = (tok >= 0 && tok < p.n_q) ? p.lse[bh * p.n_q + tok] * 1.4426950408889634f
                                             : INFINITY;
    }
    asm volatile("bar.sync 2, 256;" ::: "memory");
    float lse2[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) lse2[e] = lse2_s[64 * half + e];
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16) + 64 * half;
    float* out = p.S + (bh * p.G + g) * (int64_t)p.n_kv;
    for (int j = 0; j < n_chunks; ++j) {
      const int s = j & 1;
      if (!ptx::mbar_wait(&bars.s_full[s], (j >> 1) & 1, abort_flag, kWaitNs)) {
        fail(bars, p.status);
        break;
      }
      ptx::tc_fence_after();
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t c0[32], c1[32];
      ptx::tmem_ld32(tl + s * kTile, c0);
      ptx::tmem_ld32(tl + s * kTile + 32, c1);
      ptx::tmem_ld_wait(c0);
      ptx::reg_barrier(c1);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars.s_empty[s]);  // S is in registers: the MMA may overwrite it
#pragma unroll
      for (int e = 0; e < 32; ++e)
        acc[e & 3] += ptx::ex2(fmaf(__uint_as_float(c0[e]), p.scale_log2, -lse2[e]));
#pragma unroll
      for (int e = 0; e < 32; ++e)
        acc[e & 3] += ptx::ex2(fmaf(__uint_as_float(c1[e]), p.scale_log2, -lse2[32 + e]));
      const float part = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      if (half == 1) {
        // slot s is free once warps 0-3 have read it for chunk j - 2
        if (j >= 2 && !ptx::mbar_wait(&bars.x_empty[s], ((j >> 1) - 1) & 1, abort_flag, kWaitNs)) {
          fail(bars, p.status);
          break;
        }
        xs[s * kTile + r] = part;
        ptx::mbar_arrive(&bars.x_full[s]);
      } else {
        if (!ptx::mbar_wait(&bars.x_full[s], (j >> 1) & 1, abort_flag, kWaitNs)) {
          fail(bars, p.status);
          break;
        }
        const float total = part + xs[s * kTile + r];
        ptx::mbar_arrive(&bars.x_empty[s]);
        const int key = j * kTile + r;
        if (key < p.n_kv) out[key] = total;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmCols);
  }
}

}  // namespace

bool tc_scores_supported(const AttnArgs& a) { return a.bf16 && a.d == kD && a.gs <= kTile; }

int tc_scores(const AttnArgs& a, const int32_t* groups, const float* lse, float* S,
              cudaStream_t st) {
  ScoreParams p{};
  if ((uint64_t)a.BH * (uint64_t)a.n_kv >= 0x7fffffffull) return TLSP_ERR_UNSUPPORTED;
  TLSP_TRY(make_tmap_bf16_rows(&p.tmK, a.K, (uint64_t)a.BH * a.n_kv, kD, 64, kTile));
  p.Q = (const __nv_bfloat16*)a.Q;
  p.groups = groups;
  p.lse = lse;
  p.S = S;
  p.n_q = a.n_q;
  p.n_kv = a.n_kv;
  p.gs = a.gs;
  p.G = a.G;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
  p.status = a.status;
  const int64_t ctas = a.BH * a.G;
  if (ctas > 0x7fffffffLL) return TLSP_ERR_UNSUPPORTED;
  cudaFuncSetAttribute(scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kSmemBytes);
  scores_tc_kernel<<<(unsigned)ctas, kThreads, kSmemBytes, st>>>(p);
  return check_launch();
}

}  // namespace tlsp
