// Sparse attention on the sm_100a tensor cores (bf16, head_dim 128): the
// gathered pass of anchor and reuse steps, with the dense-sparse residual
// fused into the epilogue (the dense pass is in attn_tc_dense.cu).
//
// MC-Sparse review, section 3: the anchor step runs dense attention (its
// output and the exact scores), each query group attends only to its own
// selected KV tokens (token level, beyond block boundaries), the anchor step
// stores R = O_full - O_sparse and the reuse steps return O_sparse + R
// (additive correction for the discarded tail).
//
// One CTA per 128-query tile of a group (g_s <= 128 is one tile; padding
// rows are zero and never written back). Warp roles (416 threads, one CTA
// per SM):
//   warps 0-3  softmax + epilogue: thread t owns query row t = TMEM lane t;
//   warps 4-11 producers: together they load the tile's selection into
//              shared memory and gather its Q rows, then warps 4-7 gather the
//              K rows and warps 8-11 the V rows of each chunk of 128 selected
//              keys, with 16-byte cp.async (eight issuing warps: the gather
//              rate grows with the warps that issue), into 128-byte swizzled
//              shared memory (the tcgen05 canonical layout);
//   warp 12    allocates TMEM; lane 0 issues the tcgen05.mma instructions.
// Per chunk j: S_j = Q K_j^T (M=N=K=128, fp32 in TMEM), online softmax with
// exp2 on the SFU (S read from TMEM 64 columns at a time, the second half
// loading while the first is processed), P_j (bf16) written back to TMEM,
// and O += P_j V_j with A
// read from TMEM and V as an MN-major B operand. TMEM columns: S double
// buffer [0,256), O [256,384), P double buffer [384,512). K has three
// shared-memory slots and V two, so loads run ahead of the math.
// The softmax keeps a reference max per row and computes each chunk in one
// pass against it (the first chunk's reference is the max of its first 32
// columns); only when the chunk's P sum exceeds 2^8 (no key can exceed the
// reference by more than 2^8 otherwise) is the chunk's true max taken, the
// reference raised to it, O rescaled in TMEM and the chunk recomputed (by the
// whole warp: its TMEM accesses are warp-collective).
// Between raises the stale reference is used for numerator and denominator
// alike, which cancels exactly in O / l.
// The scale-and-subtract and the row sums run on packed fp32 pairs.
// Epilogue operands (R rows for the reuse step, O_full rows for the anchor
// step) are copied by the producers into the two K slots that the last chunk
// does not use, once those slots' last QK^T has completed, so the epilogue
// reads them from shared memory instead of waiting on L2 per row; the output
// rows go back through the free V slots, a whole row per warp store.
// Every wait is bounded (1 s); on expiry the kernel records
// TLSP_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
// Index checks: a selection entry outside [0, n_kv), a group entry outside
// [0, n_q) before the ragged tail of the last group, or one other than -1
// inside it, is recorded as TLSP_ERR_DEVICE_ASSERT (that key is read as a
// zero row, that query row is skipped); such a tile's output is unspecified.
#include <climits>
#include <type_traits>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace tlsp {
namespace {

enum Mode { kAnchor = 1, kReuse = 2 };

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kThreads = 416;
constexpr uint32_t kTileBytes = kTile * kD * 2;  // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-column half: 128 rows x 128 B
constexpr int kKSlots = 3, kVSlots = 2;
constexpr uint32_t kSmQ = 0;
constexpr uint32_t kSmK = kTileBytes;                  // kKSlots slots
constexpr uint32_t kSmV = (1 + kKSlots) * kTileBytes;  // kVSlots slots
constexpr uint32_t kSmBar = (1 + kKSlots + kVSlots) * kTileBytes;
constexpr uint32_t kSmIdx = kSmBar + 256;  // the tile's selection, when it fits
constexpr int kIdxCap = 8192;
constexpr uint32_t kSmemBytes = kSmIdx + kIdxCap * 4 + 1024;  // + slack to align the base
constexpr uint32_t kTmCols = 512;
constexpr uint32_t kTmS = 0, kTmO = 256, kTmP = 384;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr float kRescaleLog2 = 8.f;

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKSlots], k_empty[kKSlots], v_full[kVSlots], v_empty[kVSlots];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_final, drain, r_full;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct AttnParams {
  const __nv_bfloat16* __restrict__ Q;
  const __nv_bfloat16* __restrict__ K;
  const __nv_bfloat16* __restrict__ V;
  const int32_t* __restrict__ groups;
  const int32_t* __restrict__ indices;
  int n_q, n_kv, gs, G, k, tiles_per_group;
  float scale_log2;
  const __nv_bfloat16* __restrict__ O_full;  // anchor: the dense output as stored
  float* __restrict__ R_out;                 // anchor
  const float* __restrict__ R_in;            // reuse
  __nv_bfloat16* __restrict__ O_out;         // reuse
  int wave;                                  // CTAs resident at once (one per SM)
  int* status;
};

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

// Members of group g: every group holds gs tokens except the last, which
// holds n_q - (G-1)*gs followed by -1 padding.
__device__ __forceinline__ int members_of(const AttnParams& p, int g) {
  return g == p.G - 1 ? p.n_q - (p.G - 1) * p.gs : p.gs;
}

// Token of row gr of a group, or -1 for a padding row. A member entry
// outside [0, n_q), or a padding entry other than -1, is recorded.
__device__ __forceinline__ int group_token(const int32_t* grp, int gr, int members,
                                           const AttnParams& p) {
  if (gr >= p.gs) return -1;
  const int tok = __ldg(grp + gr);
  const bool ok = gr < members ? (tok >= 0 && tok < p.n_q) : tok == -1;
  if (!ok) {
    record_status(p.status, TLSP_ERR_DEVICE_ASSERT);
    return -1;
  }
  return tok;
}

// Sparse tiles: pulls into L2 what the prologue and epilogue of tile nb read
// from HBM: its selection, its query rows and the rows its epilogue reads
// (R for the reuse step, O_full for the anchor step). Called by the 128
// producer threads (pt) once their gathers are issued, for the tile one wave
// ahead, which is the one most likely to start next on some SM; L2 is shared,
// so it helps wherever that tile runs. Every address lies inside its array.
template <int kMode>
__device__ void warm_tile_l2(const AttnParams& p, int64_t nb, int pt) {
  const int tiles_per_head = p.G * p.tiles_per_group;
  const int64_t bh = nb / tiles_per_head;
  const int rem = (int)(nb % tiles_per_head);
  const int g = rem / p.tiles_per_group, t = rem % p.tiles_per_group;
  const int32_t* grp = p.groups + (bh * p.G + g) * (int64_t)p.gs;
  const int32_t* sel = p.indices + (bh * p.G + g) * (int64_t)p.k;
  for (int q = pt * 32; q < p.k; q += 128 * 32) prefetch_l2(sel + q);
  if (pt == 0) prefetch_l2(sel + p.k - 1);
  const int gr = t * kTile + pt;
  if (gr >= p.gs) return;
  const int tok = __ldg(grp + gr);
  if (tok < 0 || tok >= p.n_q) return;
  const int64_t row = (bh * p.n_q + tok) * kD;
  prefetch_l2(p.Q + row);
  prefetch_l2(p.Q + row + 64);
  if (kMode == kReuse) {
#pragma unroll
    for (int l = 0; l < 4; ++l) prefetch_l2(p.R_in + row + 32 * l);
  } else {
    prefetch_l2(p.O_full + row);
    prefetch_l2(p.O_full + row + 64);
  }
}

// Row r (0..127) of a [128 x 128] bf16 tile, 16-byte chunk c (0..15), in
// the 128-byte-swizzled layout: two 64-column halves of 128 rows x 128 B,
// chunk index XOR (row mod 8) inside each 1024-byte atom.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(c >> 3) * kHalfBytes + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// Gathers a [128 x 128] bf16 tile whose row r is global row rows(r) (or
// zeros for rows(r) < 0) with NT threads; thread pt copies 16-byte chunk
// c = pt % 16 of rows it * (NT / 16) + pt / 16, so a warp instruction moves
// two whole 256-byte rows (a thread per 16 bytes of a row: measured twice as
// fast as a thread per row, whose instructions touch 32 rows each).
template <int NT>
__device__ __forceinline__ void gather_rows(uint32_t dst, const __nv_bfloat16* src,
                                            const int (&rows)[2048 / NT], int pt) {
  const int c = pt & 15;
#pragma unroll
  for (int it = 0; it < 2048 / NT; ++it) {
    const int r = it * (NT / 16) + (pt >> 4);
    const int row = rows[it];
    const __nv_bfloat16* s = src + (row >= 0 ? (int64_t)row * kD + c * 8 : 0);
    ptx::cp_async16(dst + swz(r, c), s, row >= 0 ? 16u : 0u);
  }
}

// Marks positions past k in chunk_rows (no stored entry has this value).
constexpr int kPastK = INT_MIN;

// Global rows of chunk j of the selection for a producer thread of NT: read
// from shared memory at sel_smem when the selection was staged there
// (kStaged; an explicit shared load), else from global memory at sel.
// Positions past k are padding (-1); a selected entry outside [0, n_kv) is
// recorded and read as a zero row.
template <int NT, bool kStaged>
__device__ __forceinline__ void chunk_rows(const int32_t* sel, uint32_t sel_smem, int j, int k,
                                           int n_kv, int pt, int (&rows)[2048 / NT],
                                           int* status) {
#pragma unroll
  for (int it = 0; it < 2048 / NT; ++it) {
    const int q = j * kTile + it * (NT / 16) + (pt >> 4);
    int v = kPastK;
    if (q < k) {
      if (kStaged)
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(sel_smem + 4u * (uint32_t)q));
      else
        v = __ldg(sel + q);
    }
    rows[it] = v;
  }
#pragma unroll
  for (int it = 0; it < 2048 / NT; ++it) {
    if ((unsigned)rows[it] >= (unsigned)n_kv) {  // padding past k, or a bad entry
      if (rows[it] != kPastK) record_status(status, TLSP_ERR_DEVICE_ASSERT);
      rows[it] = -1;
    }
  }
}

// The two K slots that the last of n_chunks chunks does not use (ascending):
// they hold the epilogue's operand rows.
__device__ __forceinline__ void epi_slots(int n_chunks, int& a, int& b) {
  const int last = (n_chunks - 1) % kKSlots;
  a = last == 0 ? 1 : 0;
  b = last == 2 ? 1 : 2;
}

// The last chunk before the final one that used K slot s, or -1.
__device__ __forceinline__ int last_use(int s, int n_chunks) {
  const int m = n_chunks - 2;
  if (m < s) return -1;
  return m - (m - s) % kKSlots;
}

// Shared-memory address of 16-byte chunk c of epilogue row r: reuse rows are
// R's 512 bytes (rows 0-63 in slot a, 64-127 in slot b), anchor rows are
// O_full's 256 bytes (all in slot a). Chunk c sits at position c ^ (r mod 8)
// of its row, so eight consecutive rows reading the same c hit eight
// different 16-byte bank groups.
template <int kMode>
__device__ __forceinline__ uint32_t epi_addr(uint32_t slot_a, uint32_t slot_b, int r, int c) {
  const uint32_t sw = (uint32_t)(c ^ (r & 7)) << 4;
  if (kMode == kReuse) return (r < 64 ? slot_a : slot_b) + (uint32_t)(r & 63) * 512u + sw;
  return slot_a + (uint32_t)r * 256u + sw;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void fail(Bars& b, int* status) {
  b.abort = 1;
  record_status(status, TLSP_ERR_TIMEOUT);
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  Bars& bars = *reinterpret_cast<Bars*>(smem + kSmBar);
  volatile int* abort_flag = &bars.abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // tile -> (head, group, 128-row part of the group)
  const int tiles_per_head = p.G * p.tiles_per_group;
  const int64_t bh = blockIdx.x / tiles_per_head;
  const int rem = blockIdx.x % tiles_per_head;
  const int g = rem / p.tiles_per_group;
  const int t = rem % p.tiles_per_group;
  const int members = members_of(p, g);
  const int32_t* grp = p.groups + (bh * p.G + g) * (int64_t)p.gs;
  const int32_t* sel = p.indices + (bh * p.G + g) * (int64_t)p.k;
  const int n_keys = p.k;
  const int n_chunks = (n_keys + kTile - 1) / kTile;

  if (tid == 0) {
    ptx::mbar_init(&bars.q_full, 256);
    for (int s = 0; s < kKSlots; ++s) {
      ptx::mbar_init(&bars.k_full[s], 128);
      ptx::mbar_init(&bars.k_empty[s], 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      ptx::mbar_init(&bars.v_full[s], 128);
      ptx::mbar_init(&bars.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&bars.s_full[s], 1);
      ptx::mbar_init(&bars.p_full[s], 128);
    }
    ptx::mbar_init(&bars.o_done, 1);
    ptx::mbar_init(&bars.o_final, 1);
    ptx::mbar_init(&bars.drain, 1);
    ptx::mbar_init(&bars.r_full, 256);
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

  if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ producers
    const int pt = tid - 128;
    // The tile's selection goes to shared memory once (4-byte cp.async by all
    // 128 producers, its own commit group), so no chunk waits on an index load.
    const bool idx_smem = p.k <= kIdxCap;
    if (idx_smem) {
      for (int q = pt; q < p.k; q += 256)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(base + kSmIdx + 4u * q),
                     "l"(sel + q)
                     : "memory");
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    {
      // all 256 gather Q; then warps 4-7 stream K chunks and warps 8-11 V chunks
      const __nv_bfloat16* Qbh = p.Q + bh * (int64_t)p.n_q * kD;
      {
        int rows[8];
#pragma unroll
        for (int it = 0; it < 8; ++it)
          rows[it] = group_token(grp, t * kTile + it * 16 + (pt >> 4), members, p);
        gather_rows<256>(base + kSmQ, Qbh, rows, pt);
        ptx::cp_async_arrive_noinc(&bars.q_full);
      }
      if (idx_smem) {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        asm volatile("bar.sync 1, 256;" ::: "memory");
      }
      {
      const bool is_k = warp < 8;
      const int qt = pt & 127;
      const __nv_bfloat16* src = (is_k ? p.K : p.V) + bh * (int64_t)p.n_kv * kD;
      const int nslots = is_k ? kKSlots : kVSlots;
      const uint32_t slot0 = base + (is_k ? kSmK : kSmV);
      uint64_t* full = is_k ? bars.k_full : bars.v_full;
      uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
      // the chunk loop, with the selection read from shared memory (staged)
      // or from global memory, chosen once
      auto stream = [&](auto staged) {
        constexpr bool kStaged = decltype(staged)::value;
        int rows[16];
        chunk_rows<128, kStaged>(sel, base + kSmIdx, 0, p.k, p.n_kv, qt, rows, p.status);
        for (int j = 0; j < n_chunks; ++j) {
          const int s = j % nslots, u = j / nslots;
          if (u > 0 && !ptx::mbar_wait(&empty[s], (u - 1) & 1, abort_flag, kWaitNs)) {
            fail(bars, p.status);
            break;
          }
          gather_rows<128>(slot0 + s * kTileBytes, src, rows, qt);
          ptx::cp_async_arrive_noinc(&full[s]);
          if (j + 1 < n_chunks)
            chunk_rows<128, kStaged>(sel, base + kSmIdx, j + 1, p.k, p.n_kv, qt, rows, p.status);
        }
      };
      if (idx_smem)
        stream(std::true_type{});
      else
        stream(std::false_type{});
      }
      if (pt < 128 && p.wave > 0 && (int64_t)blockIdx.x + p.wave < (int64_t)gridDim.x)
        warm_tile_l2<kMode>(p, (int64_t)blockIdx.x + p.wave, pt);
      // Epilogue operand rows into the two K slots the last chunk does not
      // use, once their last QK^T has completed (by then every earlier phase
      // of those slots' barriers has completed too, for K and V producers
      // alike, so the parity waits are unambiguous). A warp instruction moves
      // one whole R row (reuse) or two O_full rows (anchor).
      {
        int sa, sb;
        epi_slots(n_chunks, sa, sb);
        bool ok = true;
        for (int i = 0; i < 2 && ok; ++i) {
          const int s = i ? sb : sa, jl = last_use(s, n_chunks);
          if (jl >= 0 && !ptx::mbar_wait(&bars.k_empty[s], (jl / kKSlots) & 1, abort_flag, kWaitNs))
            ok = false;
        }
        if (!ok) {
          fail(bars, p.status);
        } else {
          const uint32_t slot_a = base + kSmK + sa * kTileBytes, slot_b = base + kSmK + sb * kTileBytes;
          constexpr int kChunks = kMode == kReuse ? 32 : 16;  // 16-byte chunks per row
          constexpr int kRowsPerPass = 256 / kChunks;
#pragma unroll 4
          for (int it = 0; it < kTile / kRowsPerPass; ++it) {
            const int r = it * kRowsPerPass + pt / kChunks, c = pt % kChunks;
            const int gr = t * kTile + r;
            int tok = gr < members ? __ldg(grp + gr) : -1;
            if (tok >= p.n_q) tok = -1;
            if (tok < 0) continue;
            const int64_t row = (bh * p.n_q + tok) * kD;
            const void* src = kMode == kReuse ? (const void*)(p.R_in + row + c * 4)
                                              : (const void*)(p.O_full + row + c * 8);
            ptx::cp_async16(epi_addr<kMode>(slot_a, slot_b, r, c), src, 16u);
          }
          ptx::cp_async_arrive_noinc(&bars.r_full);
        }
      }
      ptx::cp_async_wait_all();
    }
  } else if (warp == 12) {
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
    // (the producers' Q gather validates the group entries and records bad
    // ones; here a bad entry, or anything in the ragged tail, is skipped)
    const int gr = t * kTile + r;
    int tok = gr < members ? grp[gr] : -1;
    if (tok >= p.n_q) tok = -1;
    if (tok >= 0) {  // the row the epilogue reads, towards L2 while the tile computes
      const int64_t row = (bh * p.n_q + tok) * kD;
      if (kMode == kReuse) {
#pragma unroll
        for (int l = 0; l < 4; ++l) prefetch_l2(p.R_in + row + 32 * l);
      } else {
        prefetch_l2(p.O_full + row);
        prefetch_l2(p.O_full + row + 64);
      }
    }
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_chunks; ++j) {
      const int s = j & 1;
      if (!ptx::mbar_wait(&bars.s_full[s], (j >> 1) & 1, abort_flag, kWaitNs)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const int valid_n = min(kTile, n_keys - j * kTile);
      const uint32_t s_col = tl + kTmS + s * kTile, p_col = tl + kTmP + s * 64;
      // One pass over the chunk in 32-column blocks (the next block's TMEM load
      // in flight while a block is processed): P = 2^(s * scale - m_ref) with
      // the current reference max (the scale-and-subtract and the sums on
      // packed fp32 pairs), packed to bf16 pairs. Returns the sum of P.
      auto p_pass = [&](float m_ref) {
        const float neg_m = -m_ref;
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
        const uint64_t sc2 = ptx::f2_pack(p.scale_log2, p.scale_log2), nm2 = ptx::f2_pack(neg_m, neg_m);
        auto block = [&](const uint32_t (&cur)[32], int b) {
          uint32_t pk[16];
          if (32 * b + 32 <= valid_n) {
            uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const uint64_t x = ptx::f2_fma(
                  ptx::f2_pack(__uint_as_float(cur[2 * e]), __uint_as_float(cur[2 * e + 1])), sc2, nm2);
              float x0, x1;
              ptx::f2_unpack(x, x0, x1);
              const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
              acc[e & 1] = ptx::f2_add(acc[e & 1], ptx::f2_pack(p0, p1));
              pk[e] = pack_bf16(p0, p1);
            }
            float a0, a1, a2, a3;
            ptx::f2_unpack(acc[0], a0, a1);
            ptx::f2_unpack(acc[1], a2, a3);
            sm[b & 3] += (a0 + a1) + (a2 + a3);
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
      if (__any_sync(0xffffffffu, !(sum <= 256.f))) {
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
    // Epilogue: O / l from TMEM, 32 columns at a time, with the operand row
    // (R for the reuse step, O_full for the anchor step) from shared memory.
    const bool has_row = tok >= 0;
    int sa, sb;
    epi_slots(n_chunks, sa, sb);
    const uint32_t slot_a = base + kSmK + sa * kTileBytes, slot_b = base + kSmK + sb * kTileBytes;
    if (ok && !ptx::mbar_wait(&bars.o_final, 0, abort_flag, kWaitNs)) ok = false;
    if (ok && !ptx::mbar_wait(&bars.r_full, 0, abort_flag, kWaitNs)) ok = false;
    ok = __all_sync(0xffffffffu, ok);  // the epilogue's TMEM loads and shuffles are warp-collective
    if (!ok) {
      fail(bars, p.status);
    } else {
      ptx::tc_fence_after();
      const float inv = 1.f / l_run;
      // Each thread writes its output row (bf16 O for the reuse step, fp32 R
      // for the anchor step) into the free V slots, chunk c of row r at
      // position c ^ (r mod 8); each warp then stores its own 32 rows with
      // whole-row warp instructions, so a store touches 2 (or 1) rows instead
      // of 32.
      const uint32_t ostage = base + kSmV;
      constexpr uint32_t kRowBytes = kMode == kReuse ? 256u : 512u;
      const uint32_t orow = ostage + (uint32_t)r * kRowBytes;
      auto ost = [&](int c) { return orow + ((uint32_t)(c ^ (r & 7)) << 4); };
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        ptx::tmem_ld32(tl + kTmO + q * 32, o);
        ptx::tmem_ld_wait(o);
        if (!has_row) continue;  // (no warp-collective instruction follows in this iteration)
        if (kMode == kAnchor) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 u = ptx::ld_shared_v4(epi_addr<kMode>(slot_a, slot_b, r, 4 * q + c));
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int e = 8 * c + 4 * h;
              ptx::st_shared_v4(
                  ost(8 * q + 2 * c + h),
                  __float_as_uint(__uint_as_float(w[2 * h] << 16) - __uint_as_float(o[e]) * inv),
                  __float_as_uint(__uint_as_float(w[2 * h] & 0xffff0000u) -
                                  __uint_as_float(o[e + 1]) * inv),
                  __float_as_uint(__uint_as_float(w[2 * h + 1] << 16) -
                                  __uint_as_float(o[e + 2]) * inv),
                  __float_as_uint(__uint_as_float(w[2 * h + 1] & 0xffff0000u) -
                                  __uint_as_float(o[e + 3]) * inv));
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 u0 = ptx::ld_shared_v4(epi_addr<kMode>(slot_a, slot_b, r, 8 * q + 2 * c));
            const uint4 u1 = ptx::ld_shared_v4(epi_addr<kMode>(slot_a, slot_b, r, 8 * q + 2 * c + 1));
            ptx::st_shared_v4(
                ost(4 * q + c),
                pack_bf16(__uint_as_float(o[8 * c]) * inv + __uint_as_float(u0.x),
                          __uint_as_float(o[8 * c + 1]) * inv + __uint_as_float(u0.y)),
                pack_bf16(__uint_as_float(o[8 * c + 2]) * inv + __uint_as_float(u0.z),
                          __uint_as_float(o[8 * c + 3]) * inv + __uint_as_float(u0.w)),
                pack_bf16(__uint_as_float(o[8 * c + 4]) * inv + __uint_as_float(u1.x),
                          __uint_as_float(o[8 * c + 5]) * inv + __uint_as_float(u1.y)),
                pack_bf16(__uint_as_float(o[8 * c + 6]) * inv + __uint_as_float(u1.z),
                          __uint_as_float(o[8 * c + 7]) * inv + __uint_as_float(u1.w)));
          }
        }
      }
      __syncwarp();
      // whole-row stores: lane l takes chunk l % kPer of row (l / kPer) of
      // each group of 32 / kPer rows
      constexpr int kPer = (int)(kRowBytes / 16);  // 16-byte chunks per row
      constexpr int kRowsPer = 32 / kPer;
#pragma unroll 4
      for (int i = 0; i < 32 / kRowsPer; ++i) {
        const int rl = i * kRowsPer + lane / kPer, c = lane % kPer;
        const int rr = warp * 32 + rl;
        const int tok_rr = __shfl_sync(0xffffffffu, tok, rl);
        if (tok_rr < 0) continue;
        const uint4 v = ptx::ld_shared_v4(ostage + (uint32_t)rr * kRowBytes +
                                          ((uint32_t)(c ^ (rr & 7)) << 4));
        const int64_t grow = (bh * p.n_q + tok_rr) * kD;
        if (kMode == kAnchor)
          reinterpret_cast<uint4*>(p.R_out + grow)[c] = v;
        else
          reinterpret_cast<uint4*>(p.O_out + grow)[c] = v;
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

template <int kMode>
int launch(const AttnParams& p, int64_t tiles, cudaStream_t st) {
  TLSP_TRY(ensure_smem_limit((const void*)attn_tc_kernel<kMode>, (int)kSmemBytes));
  attn_tc_kernel<kMode><<<(unsigned)tiles, kThreads, kSmemBytes, st>>>(p);
  return check_launch();
}

AttnParams base_params(const AttnArgs& a) {
  AttnParams p{};
  p.Q = (const __nv_bfloat16*)a.Q;
  p.K = (const __nv_bfloat16*)a.K;
  p.V = (const __nv_bfloat16*)a.V;
  p.n_q = a.n_q;
  p.n_kv = a.n_kv;
  p.gs = a.gs;
  p.G = a.G;
  p.k = a.k;
  p.tiles_per_group = (a.gs + kTile - 1) / kTile;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
  p.status = a.status;
  p.wave = device_sm_count();
  return p;
}

}  // namespace

bool tc_attention_supported(const AttnArgs& a) { return a.bf16 && a.d == kD; }

int tc_sparse(const AttnArgs& a, const int32_t* groups, const int32_t* indices,
              const void* O_full, float* R_out, const float* R_in, void* O_out,
              cudaStream_t st) {
  AttnParams p = base_params(a);
  p.groups = groups;
  p.indices = indices;
  p.O_full = (const __nv_bfloat16*)O_full;
  p.R_out = R_out;
  p.R_in = R_in;
  p.O_out = (__nv_bfloat16*)O_out;
  const int64_t tiles = a.BH * a.G * p.tiles_per_group;
  if (tiles > 0x7fffffffLL) return TLSP_ERR_UNSUPPORTED;
  if (R_out) return launch<kAnchor>(p, tiles, st);
  return launch<kReuse>(p, tiles, st);
}

}  // namespace tlsp
