// Dense attention of the anchor step on the sm_100a tensor cores (bf16,
// head_dim 128): O_full and the per-query log partition that the exact
// group scores are taken against.
//
// MC-Sparse review, section 3: the anchor step runs full attention once,
// O_full = softmax(Q K^T / sqrt(d)) V, and keeps each query's log partition
// LSE_i = log sum_j exp(q_i . k_j / sqrt(d)).
//
// One CTA per block of 128 consecutive queries. Warp roles (192 threads,
// one CTA per SM):
//   warps 0-3  softmax + epilogue: thread t owns query row t = TMEM lane t;
//   warp 4     lane 0 loads the Q tile and the K and V tiles of each chunk
//              of 128 keys with TMA box loads (128-byte swizzle, the tcgen05
//              canonical layout; three K and two V slots);
//   warp 5     allocates TMEM; lane 0 issues the tcgen05.mma instructions.
// Per chunk j: S_j = Q K_j^T (M=N=K=128, fp32 in TMEM), online softmax with
// exp2 on the SFU (S read from TMEM 64 columns at a time, the second half
// loading while the first is processed), P_j (bf16) written back to TMEM,
// and O += P_j V_j with A read from TMEM and V as an MN-major B operand.
// TMEM columns: S double buffer [0,256), O [256,384), P double buffer
// [384,512), so QK_{j+1} runs while chunk j's softmax does.
// The softmax keeps a reference max per row (the first chunk's: the max of
// its first 32 columns) and computes each chunk in one pass against it; only
// when the chunk's P sum exceeds 2^8 (no key can exceed the reference by more
// than 2^8 otherwise) is the chunk's true max taken, the reference raised to
// it, O rescaled in TMEM and the chunk recomputed (by the whole warp: its TMEM
// accesses are warp-collective; rows that do not need it keep their
// reference, or raise it by less than 2^8). Between raises the stale
// reference is used for numerator and denominator alike, which cancels
// exactly in O / l.
// Every wait is bounded (1 s); on expiry the kernel records
// TLSP_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace tlsp {
namespace {

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kThreads = 192;
constexpr int kLoadWarp = 4, kMmaWarp = 5;
constexpr uint32_t kTileBytes = kTile * kD * 2;  // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-column half: 128 rows x 128 B
constexpr int kKSlots = 3, kVSlots = 2;
constexpr uint32_t kSmQ = 0;
constexpr uint32_t kSmK = kTileBytes;
constexpr uint32_t kSmV = (1 + kKSlots) * kTileBytes;
constexpr uint32_t kSmBar = (1 + kKSlots + kVSlots) * kTileBytes;
constexpr uint32_t kSmemBytes = kSmBar + 256 + 1024;  // + slack to align the base
constexpr uint32_t kTmCols = 512;
constexpr uint32_t kTmS = 0, kTmO = 256, kTmP = 384;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr float kRescaleLog2 = 8.f;

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKSlots], k_empty[kKSlots], v_full[kVSlots], v_empty[kVSlots];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_final, drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct DenseParams {
  CUtensorMap tmQ, tmK, tmV;  // [BH*n, 128] bf16 row maps, box 64 x 128, 128-byte swizzle
  int n_q, n_kv, q_tiles;
  float scale_log2;
  __nv_bfloat16* __restrict__ O;
  float* __restrict__ lse;  // [BH, n_q] natural-log partition
  int* status;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void fail(Bars& b, int* status) {
  b.abort = 1;
  record_status(status, TLSP_ERR_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_dense_tc_kernel(const __grid_constant__ DenseParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  Bars& bars = *reinterpret_cast<Bars*>(smem + kSmBar);
  volatile int* abort_flag = &bars.abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = blockIdx.x / p.q_tiles;
  const int t = blockIdx.x % p.q_tiles;
  const int n_chunks = (p.n_kv + kTile - 1) / kTile;

  if (tid == 0) {
    ptx::mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kKSlots; ++s) {
      ptx::mbar_init(&bars.k_full[s], 1);
      ptx::mbar_init(&bars.k_empty[s], 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      ptx::mbar_init(&bars.v_full[s], 1);
      ptx::mbar_init(&bars.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars.s_full[s], 1);
      ptx::mbar_init(&bars.p_full[s], 128);
    }
    ptx::mbar_init(&bars.o_done, 1);
    ptx::mbar_init(&bars.o_final, 1);
    ptx::mbar_init(&bars.drain, 1);
    bars.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(&bars.tmem_base, kTmCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int q_row = (int)(bh * p.n_q) + t * kTile, kv_row = (int)(bh * p.n_kv);
      ptx::mbar_arrive_expect_tx(&bars.q_full, kTileBytes);
      ptx::tma_load_2d(base + kSmQ, &p.tmQ, 0, q_row, &bars.q_full);
      ptx::tma_load_2d(base + kSmQ + kHalfBytes, &p.tmQ, 64, q_row, &bars.q_full);
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int j = 0; j < n_chunks; ++j) {
        const int ks = j % kKSlots, ku = j / kKSlots, vs = j % kVSlots, vu = j / kVSlots;
        const int y = kv_row + j * kTile;
        if (ku > 0 && !ptx::mbar_wait(&bars.k_empty[ks], (ku - 1) & 1, abort_flag, kWaitNs)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars.k_full[ks], kTileBytes);
        ptx::tma_load_2d(base + kSmK + ks * kTileBytes, &p.tmK, 0, y, &bars.k_full[ks]);
        ptx::tma_load_2d(base + kSmK + ks * kTileBytes + kHalfBytes, &p.tmK, 64, y,
                         &bars.k_full[ks]);
        issued_k = j + 1;
        if (vu > 0 && !ptx::mbar_wait(&bars.v_empty[vs], (vu - 1) & 1, abort_flag, kWaitNs)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars.v_full[vs], kTileBytes);
        ptx::tma_load_2d(base + kSmV + vs * kTileBytes, &p.tmV, 0, y, &bars.v_full[vs]);
        ptx::tma_load_2d(base + kSmV + vs * kTileBytes + kHalfBytes, &p.tmV, 64, y,
                         &bars.v_full[vs]);
        issued_v = j + 1;
      }
      if (!ok) {
        fail(bars, p.status);
        // loads already issued land before the CTA's shared memory goes away
        for (int j = max(0, issued_k - kKSlots); j < issued_k; ++j)
          ptx::mbar_wait(&bars.k_full[j % kKSlots], (j / kKSlots) & 1, nullptr, kWaitNs);
        for (int j = max(0, issued_v - kVSlots); j < issued_v; ++j)
          ptx::mbar_wait(&bars.v_full[j % kVSlots], (j / kVSlots) & 1, nullptr, kWaitNs);
        ptx::mbar_wait(&bars.q_full, 0, nullptr, kWaitNs);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_qk = ptx::idesc_bf16(kTile, kTile, false);
      constexpr uint32_t id_pv = ptx::idesc_bf16(kTile, kD, true);
      bool ok = ptx::mbar_wait(&bars.q_full, 0, abort_flag, kWaitNs);
      auto issue_qk = [&](int j) {
        const int s = j & 1, ks = j % kKSlots;
        ok = ok && ptx::mbar_wait(&bars.k_full[ks], (j / kKSlots) & 1, abort_flag, kWaitNs);
        if (!ok) return;
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_after();
        const uint32_t kb = base + kSmK + ks * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kHalfBytes + (uint32_t)(kk & 3) * 32u;
          ptx::mma_ss(tmem + kTmS + s * kTile, ptx::sw128_desc(base + kSmQ + off, 16, 1024),
                      ptx::sw128_desc(kb + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
        }
        ptx::tc_commit(&bars.s_full[s]);
        ptx::tc_commit(&bars.k_empty[ks]);
      };
      issue_qk(0);
      if (n_chunks > 1) issue_qk(1);
      for (int j = 0; j < n_chunks && ok; ++j) {
        const int s = j & 1, vs = j % kVSlots;
        ok = ptx::mbar_wait(&bars.p_full[s], (j >> 1) & 1, abort_flag, kWaitNs) &&
             ptx::mbar_wait(&bars.v_full[vs], (j / kVSlots) & 1, abort_flag, kWaitNs);
        if (!ok) break;
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_after();
        const uint32_t vb = base + kSmV + vs * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          ptx::mma_ts(tmem + kTmO, tmem + kTmP + s * 64 + kk * 8,
                      ptx::sw128_desc(vb + kk * 2048, kHalfBytes, 1024), id_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::tc_commit(&bars.v_empty[vs]);
        ptx::tc_commit(j == n_chunks - 1 ? &bars.o_final : &bars.o_done);
        if (j + 2 < n_chunks) issue_qk(j + 2);
      }
      if (!ok) fail(bars, p.status);
      // all issued MMAs must land before TMEM is released
      ptx::tc_commit(&bars.drain);
      ptx::mbar_wait(&bars.drain, 0, nullptr, kWaitNs);  // even after an abort
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax
    const int r = tid;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const int tok = t * kTile + r < p.n_q ? t * kTile + r : -1;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_chunks; ++j) {
      const int s = j & 1;
      if (!ptx::mbar_wait(&bars.s_full[s], (j >> 1) & 1, abort_flag, kWaitNs)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const int valid_n = min(kTile, p.n_kv - j * kTile);
      const uint32_t s_col = tl + kTmS + s * kTile, p_col = tl + kTmP + s * 64;
      // One pass over the chunk in 32-column blocks (the next block's TMEM load
      // in flight while a block is processed): P = 2^(s * scale - m_ref) with
      // the current reference max, packed to bf16 pairs. Returns the sum of P.
      auto p_pass = [&](float m_ref) {
        const float neg_m = -m_ref;
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
        auto block = [&](const uint32_t (&cur)[32], int b) {
          uint32_t pk[16];
          if (32 * b + 32 <= valid_n) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float p0 = ptx::ex2(fmaf(__uint_as_float(cur[2 * e]), p.scale_log2, neg_m));
              const float p1 = ptx::ex2(fmaf(__uint_as_float(cur[2 * e + 1]), p.scale_log2, neg_m));
              sm[e & 3] += p0 + p1;
              pk[e] = pack_bf16(p0, p1);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c0 = 32 * b + 2 * e;
              const float p0 =
                  c0 < valid_n ? ptx::ex2(fmaf(__uint_as_float(cur[2 * e]), p.scale_log2, neg_m)) : 0.f;
              const float p1 =
                  c0 + 1 < valid_n ? ptx::ex2(fmaf(__uint_as_float(cur[2 * e + 1]), p.scale_log2, neg_m))
                                   : 0.f;
              sm[e & 3] += p0 + p1;
              pk[e] = pack_bf16(p0, p1);
            }
          }
          ptx::tmem_st16(p_col + 16 * b, pk);
        };
        uint32_t ra[32], rb[32];
        ptx::tmem_ld32(s_col, ra);
        ptx::tmem_ld32(s_col + 32, rb);
        ptx::tmem_ld_wait(ra);
        ptx::reg_barrier(rb);
        block(ra, 0);
        ptx::tmem_ld32(s_col + 64, ra);
        block(rb, 1);
        ptx::tmem_ld32(s_col + 96, rb);
        ptx::tmem_ld_wait(ra);
        ptx::reg_barrier(rb);
        block(ra, 2);
        block(rb, 3);
        return (sm[0] + sm[1]) + (sm[2] + sm[3]);
      };
      // The chunk's max over the valid columns (a pass over S in TMEM, by the
      // whole warp: `cols` columns).
      auto max_pass = [&](int cols) {
        float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
        for (int b = 0; b < cols / 32; ++b) {
          uint32_t c[32];
          ptx::tmem_ld32(s_col + 32 * b, c);
          ptx::tmem_ld_wait(c);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (32 * b + e < valid_n) pm[e & 3] = fmaxf(pm[e & 3], __uint_as_float(c[e]));
        }
        return fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
      };
      // first chunk: the max of its first 32 columns becomes the reference
      if (j == 0) m_run = max_pass(32) * p.scale_log2;
      // Speculative: usually the reference still holds. No key of the chunk
      // exceeds it by more than 2^8 unless the chunk's P sum does, so the sum
      // decides; only then is the true max taken. The rescale below is made of
      // warp-collective TMEM accesses, so the warp takes it together when any
      // of its rows needs it.
      float sum = p_pass(m_run);
      // (rows past n_q hold whatever the Q box read there; they never vote, so
      // a head's result does not depend on the rows that follow it)
      if (__any_sync(0xffffffffu, tok >= 0 && !(sum <= 256.f))) {
        // rows of the warp that do not need it keep their reference (factor 1),
        // or raise it by less than 2^8
        const float m_tile = fmaxf(max_pass(kTile) * p.scale_log2, m_run);
        if (j > 0) {
          // raise the reference max: O *= 2^(m_run - m_tile) once PV(j-1) has landed
          const float f = ptx::ex2(m_run - m_tile);
          if (!ptx::mbar_wait(&bars.o_done, (j - 1) & 1, abort_flag, kWaitNs)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            ptx::tmem_ld32(tl + kTmO + q * 32, o);
            ptx::tmem_ld_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            ptx::tmem_st32(tl + kTmO + q * 32, o);
          }
          l_run *= f;
        }
        m_run = m_tile;
        ptx::tmem_st_wait();
        sum = p_pass(m_run);
      }
      l_run += sum;
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars.p_full[s]);
    }
    if (ok && !ptx::mbar_wait(&bars.o_final, 0, abort_flag, kWaitNs)) ok = false;
    if (!ok) {
      fail(bars, p.status);
    } else {
      ptx::tc_fence_after();
      const float inv = 1.f / l_run;
      if (tok >= 0)  // log partition in natural units: (m + log2 l) ln 2
        p.lse[bh * p.n_q + tok] = (m_run + __log2f(l_run)) * 0.6931471805599453f;
      const int64_t row = (bh * p.n_q + (tok >= 0 ? tok : 0)) * kD;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        ptx::tmem_ld32(tl + kTmO + q * 32, o);  // every lane: the load is warp-collective
        ptx::tmem_ld_wait(o);
        if (tok < 0) continue;
        uint4* dst = reinterpret_cast<uint4*>(p.O + row + q * 32);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t* w = o + 8 * c;
          dst[c] = make_uint4(
              pack_bf16(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv),
              pack_bf16(__uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv),
              pack_bf16(__uint_as_float(w[4]) * inv, __uint_as_float(w[5]) * inv),
              pack_bf16(__uint_as_float(w[6]) * inv, __uint_as_float(w[7]) * inv));
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmCols);
  }
}

}  // namespace

int tc_dense(const AttnArgs& a, void* O, float* lse, cudaStream_t st) {
  DenseParams p{};
  if ((uint64_t)a.BH * (uint64_t)std::max(a.n_q, a.n_kv) >= 0x7fffffffull)
    return TLSP_ERR_UNSUPPORTED;
  TLSP_TRY(make_tmap_bf16_rows(&p.tmQ, a.Q, (uint64_t)a.BH * a.n_q, kD, 64, kTile));
  TLSP_TRY(make_tmap_bf16_rows(&p.tmK, a.K, (uint64_t)a.BH * a.n_kv, kD, 64, kTile));
  TLSP_TRY(make_tmap_bf16_rows(&p.tmV, a.V, (uint64_t)a.BH * a.n_kv, kD, 64, kTile));
  p.n_q = a.n_q;
  p.n_kv = a.n_kv;
  p.q_tiles = (a.n_q + kTile - 1) / kTile;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
  p.O = (__nv_bfloat16*)O;
  p.lse = lse;
  p.status = a.status;
  const int64_t tiles = a.BH * p.q_tiles;
  if (tiles > 0x7fffffffLL) return TLSP_ERR_UNSUPPORTED;
  TLSP_TRY(ensure_smem_limit((const void*)attn_dense_tc_kernel, (int)kSmemBytes));
  attn_dense_tc_kernel<<<(unsigned)tiles, kThreads, kSmemBytes, st>>>(p);
  return check_launch();
}

}  // namespace tlsp
