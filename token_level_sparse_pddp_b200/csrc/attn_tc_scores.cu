// Exact per-group KV scores on the sm_100a tensor cores (bf16, head_dim 128).
//
// MC-Sparse review, section 3: on the anchor step each query group selects
// its KV tokens from exact attention scores (not mean-pooled estimates). The
// score of key j for group g is the attention mass the group puts on it,
// S_g[j] = sum_{i in g} exp(q_i . k_j / sqrt(d) - LSE_i), with LSE_i the log
// partition of query i from the dense pass.
//
// One CTA per (head, group) row for groups of at most 128 queries; a launch
// covers a contiguous range of rows (the anchor step goes through them in
// batches whose scores stay in L2 for the selection that follows). The CTA keeps
// the group's Q rows in shared memory and streams all keys in chunks of 128
// with TMA box loads (four slots). The product is taken transposed,
// S^T = K_chunk Q_g^T (M = 128 keys on TMEM lanes, N = 128 queries on TMEM
// columns), so thread t (lane t) owns key j0 + t and sums its own lane:
// no cross-thread reduction and no atomics; the per-query LSE (in log2 units)
// is a shared-memory broadcast. A quarter of the exponentials are computed on
// the FMA pipe (a polynomial, on packed fp32 pairs) instead of the
// special-function unit, which the pass otherwise saturates. S^T is double-buffered in TMEM so the next
// chunk's MMA runs while a chunk is summed.
// Warp roles (416 threads): warps 0-3 sum the even chunks (TMEM buffer 0)
// and warps 4-7 the odd ones (buffer 1), each lane over all 128 query
// columns of its key, so the two warps of an SM sub-partition work on
// different chunks and one's TMEM loads overlap the other's exp2; each
// warpgroup stores its chunk's sums itself. Warps 8-11 gather Q_g with
// 16-byte cp.async (128-byte swizzle), then lane 0 of warp 8 issues the K
// loads; warp 12 allocates TMEM and lane 0 issues tcgen05.mma.
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
constexpr uint32_t kSmemBytes = kSmLse + kTile * 4 + 1024;
constexpr uint32_t kTmCols = 256;
constexpr uint64_t kWaitNs = 1000000000ull;

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t s_full[2], s_empty[2];
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
  float* __restrict__ S;  // rows row0 .. row0 + gridDim.x - 1, from S[0]
  int64_t row0;           // first (head, group) row of this launch
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
  const int64_t grow = p.row0 + blockIdx.x;
  const int64_t bh = grow / p.G;
  const int g = (int)(grow % p.G);
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
      ptx::mbar_init(&bars.s_empty[s], 128);
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
    // warpgroup h = warp / 4 takes the chunks j = h, h + 2, ... (TMEM buffer h);
    // lane r of warp w is key j * 128 + 32 (w % 4) + r and sums all 128 columns
    const int r = tid & 127, h = warp >> 2;
    if (h == 0) {
      // minus the log2-unit LSE of the group's queries; padding rows contribute
      // exp2(-inf) = 0 (or at most 2.4e-38 on the FMA-pipe path)
      const int tok = r < p.gs ? grp[r] : -1;
      lse2_s[r] = (tok >= 0 && tok < p.n_q) ? -(p.lse[bh * p.n_q + tok] * 1.4426950408889634f)
                                             : -INFINITY;
    }
    asm volatile("bar.sync 2, 256;" ::: "memory");
    const float4* l4 = reinterpret_cast<const float4*>(lse2_s);
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16) + h * kTile;
    float* out = p.S + (int64_t)blockIdx.x * p.n_kv;
    for (int j = h; j < n_chunks; j += 2) {
      if (!ptx::mbar_wait(&bars.s_full[h], (j >> 1) & 1, abort_flag, kWaitNs)) {
        fail(bars, p.status);
        break;
      }
      ptx::tc_fence_after();
      uint64_t acc01 = 0ull, acc23 = 0ull;  // packed fp32 pairs
      const uint64_t sc2 = ptx::f2_pack(p.scale_log2, p.scale_log2);
      // columns 32q .. 32q + 31 of this lane against the queries' LSE
      auto sum32 = [&](const uint32_t (&c)[32], int q) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 l = l4[(32 * q + e) >> 2];
          const uint64_t x01 = ptx::f2_fma(ptx::f2_pack(__uint_as_float(c[e]), __uint_as_float(c[e + 1])),
                                           sc2, ptx::f2_pack(l.x, l.y));
          const uint64_t x23 = ptx::f2_fma(ptx::f2_pack(__uint_as_float(c[e + 2]), __uint_as_float(c[e + 3])),
                                           sc2, ptx::f2_pack(l.z, l.w));
          float a, b;
          ptx::f2_unpack(x01, a, b);
          acc01 = ptx::f2_add(acc01, ptx::f2_pack(ptx::ex2(a), ptx::ex2(b)));
          // every other group of four: its second pair on the FMA pipe, so a
          // quarter of the exponentials leave the special-function unit
          if (((e >> 2) % 2) == 2 - 1) {
            acc23 = ptx::f2_add(acc23, ptx::exp2_poly2(x23));
          } else {
            float cc, d;
            ptx::f2_unpack(x23, cc, d);
            acc23 = ptx::f2_add(acc23, ptx::f2_pack(ptx::ex2(cc), ptx::ex2(d)));
          }
        }
      };
      // each quarter's TMEM load is in flight while the one before it is summed
      uint32_t c0[32], c1[32];
      ptx::tmem_ld32(tl, c0);
      ptx::tmem_ld_wait(c0);
      ptx::tmem_ld32(tl + 32, c1);
      sum32(c0, 0);
      ptx::tmem_ld_wait(c1);
      ptx::tmem_ld32(tl + 64, c0);
      sum32(c1, 1);
      ptx::tmem_ld_wait(c0);
      ptx::tmem_ld32(tl + 96, c1);
      sum32(c0, 2);
      ptx::tmem_ld_wait(c1);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars.s_empty[h]);  // S is in registers: the MMA may overwrite it
      sum32(c1, 3);
      const int key = j * kTile + r;
      float a0, a1, a2, a3;
      ptx::f2_unpack(acc01, a0, a1);
      ptx::f2_unpack(acc23, a2, a3);
      if (key < p.n_kv) out[key] = (a0 + a1) + (a2 + a3);
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

int tc_scores(const AttnArgs& a, const int32_t* groups, const float* lse, float* S, int64_t row0,
              int64_t rows, cudaStream_t st) {
  ScoreParams p{};
  if ((uint64_t)a.BH * (uint64_t)a.n_kv >= 0x7fffffffull) return TLSP_ERR_UNSUPPORTED;
  TLSP_TRY(make_tmap_bf16_rows(&p.tmK, a.K, (uint64_t)a.BH * a.n_kv, kD, 64, kTile));
  p.Q = (const __nv_bfloat16*)a.Q;
  p.groups = groups;
  p.lse = lse;
  p.S = S;
  p.row0 = row0;
  p.n_q = a.n_q;
  p.n_kv = a.n_kv;
  p.gs = a.gs;
  p.G = a.G;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
  p.status = a.status;
  if (rows <= 0) return TLSP_OK;
  if (rows > 0x7fffffffLL) return TLSP_ERR_UNSUPPORTED;
  TLSP_TRY(ensure_smem_limit((const void*)scores_tc_kernel, (int)kSmemBytes));
  scores_tc_kernel<<<(unsigned)rows, kThreads, kSmemBytes, st>>>(p);
  return check_launch();
}

}  // namespace tlsp
