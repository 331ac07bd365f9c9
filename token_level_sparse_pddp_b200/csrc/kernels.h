// Internal interface between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace tlsp {

// ---- api.cu: shape checks shared by the entry points
int validate_dims(const tlsp_dims* d);

// ---- pddp.cu: tile-aligned query grouping
struct PddpWork {
  int32_t* perm;      // [BH, n_q] token ids, node segments contiguous
  int32_t* tmp;       // [BH, n_q] partition scratch
  uint32_t* seg_key;  // [BH, n_q] order keys of the projections, by position
  float* node_mu;     // [BH, G, d]
  float* node_v;      // [BH, G, d]
  float* partials;    // [partial_slots, d*d + 2d] chunk moments
  int64_t partial_slots;
  int* status;        // device status word (timed-out waits)
};
int run_pddp(const void* Q, bool bf16, int d, int64_t BH, int n_q, int gs, int32_t* groups,
             float* trace, const PddpWork& w, cudaStream_t st);

// ---- select.cu: top-k and the single PDDP cut
int launch_topk(const float* scores, int64_t rows, int n_kv, int k, int32_t* indices,
                int* status, cudaStream_t stream);
int launch_split(const float* proj, const int32_t* members, int n, int n_left, int32_t* left,
                 int32_t* right, cudaStream_t stream);

// ---- ablation.cu: the components MC-Sparse replaces
int launch_raster_groups(int32_t* groups, int64_t BH, int n_q, int gs, cudaStream_t st);
int launch_block_topk(const float* in, int64_t rows, int n_in, int n_blocks, int sum_width,
                      int kb, int b_expand, int32_t* indices, float* block_out, cudaStream_t st);

// ---- attention kernels
struct AttnArgs {
  const void *Q, *K, *V;
  int64_t BH;
  int n_q, n_kv, d, gs, G, k;
  bool bf16;
  int* status;
};
int simt_dense(const AttnArgs& a, void* O, float* LSE, cudaStream_t st);
int launch_pooled_select(const AttnArgs& a, const int32_t* groups, int block, int32_t* indices,
                         float* block_scores, float* scratch, cudaStream_t st);
size_t pooled_scratch_floats(const AttnArgs& a, int block);
// scores of the (head, group) rows row0 .. row0 + rows - 1 into S[0 .. rows * n_kv)
int simt_scores(const AttnArgs& a, const int32_t* groups, const float* LSE, float* S,
                int64_t row0, int64_t rows, cudaStream_t st);
int simt_sparse(const AttnArgs& a, const int32_t* groups, const int32_t* indices,
                const void* O_full, float* R_out, const float* R_in, void* O_out,
                cudaStream_t st);

// tmap.cu: 2-D bf16 row-major tensor map [rows, cols], 128-byte swizzle
int make_tmap_bf16_rows(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols,
                        uint32_t box_cols, uint32_t box_rows);

// attn_tc.cu: tensor-core gathered sparse pass (bf16, d = 128)
bool tc_attention_supported(const AttnArgs& a);
int tc_sparse(const AttnArgs& a, const int32_t* groups, const int32_t* indices,
              const void* O_full, float* R_out, const float* R_in, void* O_out,
              cudaStream_t st);
// attn_tc_dense.cu: tensor-core dense pass (same support condition)
int tc_dense(const AttnArgs& a, void* O, float* lse, cudaStream_t st);

// attn_tc_scores.cu: exact group scores on the tensor cores (bf16, d = 128, g_s <= 128)
bool tc_scores_supported(const AttnArgs& a);
int tc_scores(const AttnArgs& a, const int32_t* groups, const float* lse, float* S, int64_t row0,
              int64_t rows, cudaStream_t st);

// Exact group scores of the (head, group) rows row0 .. row0 + rows - 1 (row
// = head * G + group) into S[0 .. rows * n_kv).
inline int scores_pass(const AttnArgs& a, const int32_t* groups, const float* lse, float* S,
                       int64_t row0, int64_t rows, cudaStream_t st) {
  if (tc_scores_supported(a)) return tc_scores(a, groups, lse, S, row0, rows, st);
  return simt_scores(a, groups, lse, S, row0, rows, st);
}

// Sparse pass with the residual epilogue on the best kernel for the shape.
inline int sparse_pass(const AttnArgs& a, const int32_t* groups, const int32_t* indices,
                       const void* O_full, float* R_out, const float* R_in, void* O_out,
                       cudaStream_t st) {
  if (tc_attention_supported(a)) return tc_sparse(a, groups, indices, O_full, R_out, R_in, O_out, st);
  return simt_sparse(a, groups, indices, O_full, R_out, R_in, O_out, st);
}

// Dense pass (O and the log partition per query) on the best kernel.
inline int dense_pass(const AttnArgs& a, void* O, float* lse, cudaStream_t st) {
  if (tc_attention_supported(a)) return tc_dense(a, O, lse, st);
  return simt_dense(a, O, lse, st);
}

}  // namespace tlsp
