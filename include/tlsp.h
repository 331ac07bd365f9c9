/*
 * tlsp.h — C ABI of libtlsp: token-level sparse attention with PDDP query
 * grouping (MC-Sparse) on NVIDIA B200 (sm_100a).
 *
 * The method is the one the review "MC-Sparse: Deconstructing and Closing the
 * Dense-Sparse Attention Gap in Diffusion Transformers" describes in section 3
 * ("Method & Key Results"):
 *   - queries of each head are split into equal-size, tile-aligned groups by
 *     fast principal direction divisive partitioning (PDDP);
 *   - on an anchor denoising step a dense attention pass gives the dense
 *     output and exact per-group KV scores, each group keeps its top-k KV
 *     tokens (token level, not blocks), and the dense-sparse residual
 *     R = O_full - O_sparse is stored;
 *   - on the reuse steps that follow, only sparse attention over the cached
 *     selection runs and R is added back as an additive correction.
 *
 * Conventions shared by every call below
 *   - All tensor pointers are DEVICE memory owned by the caller. The library
 *     allocates and frees nothing on these paths; scratch comes from the
 *     caller's workspace `ws` (size from tlsp_workspace_bytes()).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and performs no host synchronisation.
 *   - Arguments are validated on the host before anything is enqueued; on a
 *     validation error nothing is launched and the error code is returned.
 *     A failed launch returns TLSP_ERR_CUDA (query tlsp_last_cuda_error()).
 *   - Errors found on the device (a bounded wait that ran out, an index out of
 *     range) are recorded in a status word at the start of `ws`; read it with
 *     tlsp_get_device_status() after synchronising the stream. The workspace
 *     must be zero-filled once before first use (or reset with
 *     tlsp_reset_device_status()).
 *   - Q, K, V are never modified. Layouts are row-major with the head
 *     dimension contiguous: Q, O [B, H, n_q, d]; K, V [B, H, n_kv, d]; tokens
 *     of the (frame, height, width) grid flattened as n = (t*Hg + y)*Wg + x.
 *   - Data pointers must be 16-byte aligned.
 *   - Softmax scale is 1/sqrt(d); attention is bidirectional with no mask.
 */
#ifndef TLSP_H_
#define TLSP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TLSP_OK = 0,
  TLSP_ERR_INVALID_ARG = -1,   /* null pointer, bad shape, misaligned pointer, k > n_kv ... */
  TLSP_ERR_UNSUPPORTED = -2,   /* valid request this build has no kernel for */
  TLSP_ERR_WORKSPACE = -3,     /* ws_bytes smaller than the call needs */
  TLSP_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed */
  TLSP_ERR_TIMEOUT = -5,       /* device: a bounded wait ran out (kernel returned early) */
  TLSP_ERR_DEVICE_ASSERT = -6  /* device: an internal check failed (e.g. index out of range) */
} tlsp_status;

typedef enum { TLSP_F32 = 0, TLSP_BF16 = 1 } tlsp_dtype;

typedef struct {
  int32_t batch;     /* B >= 1 */
  int32_t heads;     /* H >= 1 */
  int32_t n_q;       /* query tokens per head, >= 1 */
  int32_t n_kv;      /* key/value tokens per head, >= 1 (may differ from n_q) */
  int32_t head_dim;  /* d: 64 or 128 */
  tlsp_dtype dtype;  /* element type of Q, K, V and O */
} tlsp_dims;

/* Number of query groups per head: G = ceil(n_q / group_size). Every group
 * holds group_size queries except the last, which holds n_q - (G-1)*group_size
 * (reading of "equal-size" groups when group_size does not divide n_q).
 * Returns -1 for non-positive arguments. */
int32_t tlsp_num_groups(int32_t n_q, int32_t group_size);

/* Number of PDDP bisection levels: ceil(log2(G)) (0 when G == 1). */
int32_t tlsp_num_levels(int32_t n_q, int32_t group_size);

/* Workspace bytes sufficient for every call below with these dims,
 * group_size and k (the maximum over calls). 0 on invalid arguments. The
 * anchor call scores and selects the (head, group) rows in batches of at
 * most about 80 MB of fp32 scores; the workspace holds one batch (not the
 * B*H*G*n_kv matrix), so a NULL `scores` argument is always allowed. */
size_t tlsp_workspace_bytes(const tlsp_dims* dims, int32_t group_size, int32_t k);

/* Tile-aligned query grouping by fast PDDP (review section 3: queries that
 * look alike share a group; groups have equal size, aligned to the GPU tile,
 * and are formed by principal direction divisive partitioning).
 *   Q       [B, H, n_q, d] in dims->dtype (the anchor step's queries).
 *   groups  out, int32 [B, H, G*group_size]: group g occupies
 *           [g*group_size, (g+1)*group_size); token ids ascending inside a
 *           group; the last group's unused tail is -1.
 * Per (b, h) the root node holds all n_q tokens and G leaf slots. A node
 * with s > 1 slots is centred, its leading principal direction is found by
 * 16 power iterations from the normalised ones vector (sign: largest
 * component positive; a node with no spread uses e_0), every token is
 * projected on it, and the floor(s/2)*group_size tokens of lowest projection
 * (ties: lower token id) go left with floor(s/2) slots, the rest right.
 * Leaves are numbered left to right. Arithmetic is fp32. */
int tlsp_group_queries(const tlsp_dims* dims, const void* Q, int32_t group_size, int32_t* groups,
                       void* ws, size_t ws_bytes, void* stream);

/* As tlsp_group_queries, and also writes the projections the cuts were made
 * on: proj [L, B, H, n_q] fp32 with L = tlsp_num_levels(); proj[l][b][h][t]
 * is token t's projection at level l if t's node was split at level l, else 0.
 * Cutting every node on these values reproduces `groups` exactly. */
int tlsp_group_queries_trace(const tlsp_dims* dims, const void* Q, int32_t group_size,
                             int32_t* groups, float* proj, void* ws, size_t ws_bytes,
                             void* stream);

/* One PDDP cut on caller-supplied projections (parity hook).
 *   proj     [*] fp32, indexed by token id (entries of `members` only are read).
 *   members  [n] int32 token ids in ascending order.
 *   n_left   0 <= n_left <= n.
 *   left_out [n_left], right_out [n - n_left]: the n_left members of lowest
 *            (projection, token id) and the rest, each ascending by token id.
 * -0 and +0 compare equal (the tie then falls to the token id). */
int tlsp_split_from_projections(const float* proj, const int32_t* members, int32_t n,
                                int32_t n_left, int32_t* left_out, int32_t* right_out,
                                void* ws, size_t ws_bytes, void* stream);

/* Anchor step (review section 3: exact KV selection on the anchor step and
 * the residual R = O_full - O_sparse).
 *   Q, K, V   inputs in dims->dtype.
 *   groups    [B, H, G*group_size] from tlsp_group_queries (this step's Q).
 *   k         KV tokens kept per group, 1 <= k <= n_kv.
 *   O         out [B, H, n_q, d] in dims->dtype: dense attention output
 *             O_full, in token order.
 *   indices   out int32 [B, H, G, k]: per group the k keys with the largest
 *             exact score S_g[j] = sum_{i in g} softmax_j(q_i . k_j / sqrt(d))
 *             (ties: lower key index), listed ascending.
 *   R         out fp32 [B, H, n_q, d], token order: O_full as stored in O
 *             minus the sparse output over `indices` (softmax renormalised
 *             over the selection).
 *   scores    optional out fp32 [B, H, G, n_kv]: the exact group scores the
 *             selection was made on (NULL: kept in the workspace). Selecting
 *             the top k of these values with the rule above reproduces
 *             `indices` exactly. */
int tlsp_anchor_attention(const tlsp_dims* dims, const void* Q, const void* K, const void* V,
                          const int32_t* groups, int32_t group_size, int32_t k, void* O,
                          int32_t* indices, float* R, float* scores, void* ws, size_t ws_bytes,
                          void* stream);

/* Dense attention alone (the dense pass of the anchor step; also the
 * baseline a reuse step is compared with).
 *   O    out [B, H, n_q, d] in dims->dtype: softmax(q_i . k_j / sqrt(d)) V.
 *   lse  optional out fp32 [B, H, n_q]: log sum_j exp(q_i . k_j / sqrt(d))
 *        (NULL: kept in the workspace, which must then hold at least
 *        256 + 4*B*H*n_q bytes; with lse given, 256 bytes suffice). */
int tlsp_dense_attention(const tlsp_dims* dims, const void* Q, const void* K, const void* V,
                         void* O, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Dense attention that allocates nothing (no counterpart in the paper: it is
 * a convenience of this library). For callers that may not allocate device
 * memory or pass a workspace, e.g. code running during CUDA graph capture or
 * under a framework whose pool owns all allocations. Same result as
 * tlsp_dense_attention with lse = NULL.
 *   Q, K, V, O   as for tlsp_dense_attention; O is written.
 * Its scratch (the per-query log partition and a status word) is a fixed
 * array in the library's device memory, 16 MiB + 256 B, held by every GPU
 * that loads the library until exit. Limit: B*H*n_q <= 4194304, larger
 * requests return TLSP_ERR_UNSUPPORTED with nothing launched. The first call
 * on each device looks the array's address up (with that device current);
 * make that first call before any stream capture. Every call shares the
 * array and it keeps the last call's contents: calls that overlap on one GPU
 * (for instance issued on different streams) race on it. The status word is
 * cleared at the start of each call; device-side errors recorded there are
 * not reported. */
int tlsp_dense_attention_noalloc(const tlsp_dims* dims, const void* Q, const void* K,
                                 const void* V, void* O, void* stream);

/* Reuse step (review section 3: reuse of the anchor's exact selections and
 * the residual as an additive correction).
 *   Q, K, V   this step's inputs; groups, indices and R from the last anchor.
 *   O         out [B, H, n_q, d] in dims->dtype, token order:
 *             O_i = sparse attention of q_i over indices[g(i)] + R_i.
 *   ws        only its status word is used: 16-byte aligned and at least
 *             256 bytes (a full tlsp_workspace_bytes() workspace also works).
 * groups, indices and R are caller-kept state, checked on the device: a
 * selection entry outside [0, n_kv), a group member outside [0, n_q), or a
 * padding entry of the last group's ragged tail other than -1, records
 * TLSP_ERR_DEVICE_ASSERT in the status word; the output of the tiles
 * involved is then unspecified (the others are unaffected). */
int tlsp_reuse_attention(const tlsp_dims* dims, const void* Q, const void* K, const void* V,
                         const int32_t* groups, int32_t group_size, int32_t k,
                         const int32_t* indices, const float* R, void* O, void* ws,
                         size_t ws_bytes, void* stream);

/* Top-k selection on caller-supplied scores (parity hook; the same kernel
 * the anchor step uses).
 *   scores   fp32 [rows, n_kv]; indices out int32 [rows, k], ascending, the k
 *            largest per row with ties to the lower index; -0 equals +0.
 *   ws       optional (NULL allowed): when given, 16-byte aligned and at least
 *            256 bytes, a timed-out wait inside the kernel is recorded in its
 *            status word; ws_bytes is its size. */
int tlsp_topk_from_scores(const float* scores, int32_t rows, int32_t n_kv, int32_t k,
                          int32_t* indices, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Ablation: the components MC-Sparse replaces (review section 3 and its
 * ablation table, which adds exact KV selection, token granularity, query
 * grouping and residual compensation one by one on top of block-sparse
 * attention with mean-pooled scores). Sparse attention over any selection is
 * tlsp_reuse_attention (with R = 0 for no residual compensation).
 * ------------------------------------------------------------------------- */

/* Raster query groups (no PDDP): group g holds tokens g*group_size ..
 * g*group_size + group_size - 1 in ascending order, -1 past n_q.
 *   groups  out int32 [B, H, G*group_size]. */
int tlsp_group_raster(const tlsp_dims* dims, int32_t group_size, int32_t* groups, void* stream);

/* Block-granular selection from per-key scores: keys in blocks of `block`
 * consecutive tokens; a block's score is the fp32 sum of its keys' scores in
 * key order; the k / block blocks of largest score (ties to the lower block)
 * are taken and expanded to their keys, ascending.
 *   scores        fp32 [rows, n_kv] (for example the exact group scores of
 *                 the anchor step); indices out int32 [rows, k];
 *   block_scores  optional out fp32 [rows, n_kv / block] (NULL: not written).
 * Requires block | n_kv and block | k (else TLSP_ERR_UNSUPPORTED) and
 * n_kv / block + k / block <= 51200. */
int tlsp_block_topk_from_scores(const float* scores, int32_t rows, int32_t n_kv, int32_t k,
                                int32_t block, int32_t* indices, float* block_scores,
                                void* stream);

/* Block-sparse baseline selection (approximate, mean-pooled scoring): for
 * each group g and key block m, score = mean(Q rows of g) . mean(K rows of m)
 * / sqrt(d) in fp32; the k / block best blocks (ties to the lower block) are
 * expanded to their keys, ascending.
 *   groups        int32 [B, H, G*group_size] (any grouping, e.g. raster);
 *   indices       out int32 [B, H, G, k];
 *   block_scores  optional out fp32 [B, H, G, n_kv / block];
 *   ws            as for tlsp_anchor_attention (the pooled rows and block
 *                 scores use its grouping scratch; TLSP_ERR_WORKSPACE if they
 *                 do not fit).
 * Requires block | n_kv and block | k (else TLSP_ERR_UNSUPPORTED). */
int tlsp_pooled_block_select(const tlsp_dims* dims, const void* Q, const void* K,
                             const int32_t* groups, int32_t group_size, int32_t k, int32_t block,
                             int32_t* indices, float* block_scores, void* ws, size_t ws_bytes,
                             void* stream);

/* Device status recorded in `ws` (TLSP_OK, TLSP_ERR_TIMEOUT or
 * TLSP_ERR_DEVICE_ASSERT). Synchronises with the device (blocking copy of the
 * status word): call it after the stream that used `ws` has finished. */
int tlsp_get_device_status(const void* ws);

/* Clears the status word at the start of `ws` (asynchronous on `stream`). */
int tlsp_reset_device_status(void* ws, void* stream);

/* Test hook for the error path: launches one thread that waits on a flag in
 * `ws` which nothing sets, for at most `spin_limit` polls, then records
 * TLSP_ERR_TIMEOUT and returns. It never hangs: the wait is bounded. */
int tlsp_debug_bounded_wait(void* ws, size_t ws_bytes, int64_t spin_limit, void* stream);

/* Human-readable name of a status code. */
const char* tlsp_status_string(int status);

/* The cudaError_t of the last TLSP_ERR_CUDA returned on this thread (0 if none). */
int tlsp_last_cuda_error(void);

/* Number of kernels this library has launched in this process (counted on
 * the host at each launch); used to report launches inside a timed region. */
int64_t tlsp_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* TLSP_H_ */
