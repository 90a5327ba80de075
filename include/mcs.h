/*
 * mcs.h -- C ABI of the MC-Sparse (Meta-Cached Sparse Attention) hot path on
 * NVIDIA B200 (sm_100a).
 *
 * The method (aiqbench.com, "MC-Sparse: Deconstructing and Closing the
 * Dense-Sparse Attention Gap in Diffusion Transformers", abstract; cctest.ai,
 * "MC-Sparse Narrows the Dense-Sparse Attention Gap in Diffusion
 * Transformers", design choices): a metadata pass computes exact dense
 * attention probabilities, organises similar queries into tile-aligned
 * groups, selects individual KV tokens per group from those probabilities and
 * caches the residual between dense and sparse outputs; later denoising steps
 * reuse the groups, indices and residual.
 *
 * Conventions for every entry point
 *   - Q, K, V, O: bf16, layout [B, H, N, d], contiguous (d fastest), in
 *     device memory, 16-byte aligned.  d is 64 or 128.
 *   - scale: softmax scale applied to Q.K (usually 1/sqrt(d)).
 *   - All device buffers are owned by the caller.  The library allocates no
 *     device memory and keeps no per-call state.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are detected on the host before any
 *     launch and returned synchronously; nothing is launched then.
 *   - A launch failure returns MCS_ERR_CUDA.  Errors the device detects (a
 *     bounded wait that ran out) are recorded in a per-device status word
 *     that mcs_last_device_status() reads; kernels never trap.
 *   - Query groups: perm[b,h,:] is a permutation of 0..N-1; group g of head
 *     (b,h) is the queries perm[b,h,g*G .. min((g+1)*G, N)-1]; the last group
 *     may be partial.  n_groups = ceil(N / G).
 *   - KV indices: kv_idx[b,h,g,0..k'-1] with k' = min(k, N): unique,
 *     strictly ascending, in [0, N).
 *   - Residual: float32 [B, H, N, d] in the original token order.
 */
#ifndef MCS_H_
#define MCS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MCS_ABI_VERSION 2

typedef struct CUstream_st *mcs_stream_t; /* same type as cudaStream_t */

typedef enum {
  MCS_OK = 0,
  MCS_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer   */
  MCS_ERR_UNSUPPORTED = 2,  /* d or G outside the supported set            */
  MCS_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required  */
  MCS_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed        */
  MCS_ERR_TIMEOUT = 5,      /* a bounded device wait ran out               */
  MCS_ERR_BAD_META = 6,     /* metadata failed validation                  */
  MCS_ERR_TOO_LARGE = 7     /* shape exceeds a fixed, compiled-in capacity */
} mcs_status;

/* Cached metadata of one plan ("query groups, KV indices ... and residuals",
 * aiqbench.com abstract).  All pointers are caller-owned device memory.
 *
 * pair_idx / pair_len (optional, both or neither) are derived from kv_idx:
 * for each pair p of adjacent groups (2p, 2p+1), the union of their kept
 * keys, ordered [keys only 2p keeps | keys both keep | keys only 2p+1
 * keeps], each segment ascending; pair_len[b,h,p] is the union's size u, so
 * group 2p's keys are positions [0, k) and group 2p+1's are [u - k, u).  When
 * the head has an odd number of groups the last pair is group 2p alone
 * (u = k).  Adjacent groups hold similar queries (cctest.ai "Hardware-aware
 * query organization") and keep mostly the same keys, so the reused step
 * gathers each shared key once per pair.  n_pairs = ceil(n_groups / 2). */
typedef struct {
  int32_t B, H, N, d, G, k, n_groups; /* k is stored clamped: k = min(k, N) */
  int32_t *perm;                      /* [B,H,N]                           */
  int32_t *kv_idx;                    /* [B,H,n_groups,k]                  */
  float *residual;                    /* [B,H,N,d]                         */
  int32_t *pair_idx;                  /* [B,H,n_pairs,2k] or NULL          */
  int32_t *pair_len;                  /* [B,H,n_pairs]    or NULL          */
} mcs_meta;

/* Library ABI version (MCS_ABI_VERSION of the build). */
int mcs_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *mcs_status_string(mcs_status s);

/* Fill in the scalar fields of `meta` (B, H, N, d, G, k clamped to N,
 * n_groups) and check them.  Pointers are left untouched. */
mcs_status mcs_meta_init(mcs_meta *meta, int B, int H, int N, int d, int G, int k);

/* Bytes of workspace mcs_plan and its stages need for this shape; 0 when the
 * shape is invalid.  The workspace must be 256-byte aligned device memory. */
size_t mcs_plan_workspace_size(int B, int H, int N, int d, int G, int k);

/*
 * mcs_plan -- the metadata pass: steps a1..a5 of the hot path.
 *   a1 grouping: per (b,h), centre Q, take the top principal direction of its
 *      covariance, sort the projections ascending (stable) -> perm.
 *   a2 exact probabilities: row max and sum of exp over all N keys, and the
 *      dense output (fp32, split-precision P.V).
 *   a3 group scores: colsum[g, j] = sum_{i in g} P_ij.
 *   a4 selection: per group the k' largest scores, ties to the lower index,
 *      stored ascending -> kv_idx.
 *   a5 residual: R = O_dense - O_sparse, O_sparse renormalised over the kept
 *      keys -> residual.
 * Sources: aiqbench.com abstract ("KV indices selected using exact attention
 * probabilities", "residuals between dense and sparse attention outputs");
 * cnshai.top "output-aware sparse attention / KV cache", section "MC-Sparse:
 * three failure modes, one fix"; cctest.ai design choices.
 *
 * meta: scalar fields are set by this call; meta->perm, ->kv_idx and
 *   ->residual must point to caller buffers of the sizes given above; when
 *   meta->pair_idx and ->pair_len are set, the pair union lists are built
 *   into them as well (as mcs_meta_pairs does), else into the workspace.
 * O_dense: optional bf16 [B,H,N,d] output of the dense attention of this step
 *   (what a plan step of the denoising loop produces); may be NULL.
 * workspace: >= mcs_plan_workspace_size(...) bytes of device memory.
 */
mcs_status mcs_plan(const void *Q, const void *K, const void *V, int B, int H, int N, int d,
                    int G, int k, float scale, mcs_meta *meta, void *O_dense, void *workspace,
                    size_t workspace_bytes, mcs_stream_t stream);

/*
 * Where mcs_plan_stats and mcs_plan_scores leave their results inside the
 * workspace, as byte offsets from its start (any pointer argument may be
 * NULL).  All float32, row-major:
 *   row_m   [B,H,N]          m_i, a reference near max_j s_ij log2(e) (s_ij =
 *                            scale Q_i.K_j): the softmax raises it only when
 *                            a later key exceeds it by more than 32, so
 *                            max_j s_ij log2(e) - 32 <= m_i <= max_j s_ij log2(e)
 *   row_l   [B,H,N]          l_i = sum_j 2^(s_ij log2(e) - m_i)
 *   O32     [B,H,N,d]        the dense output of the statistics pass
 *   colsum  [B,H,n_groups,N] sum over group g's queries of P_ij
 * m_i + log2(l_i) is the row's log2 normaliser whatever m_i is, and
 * P_ij = 2^(s_ij log2(e) - m_i) / l_i are the exact probabilities of
 * aiqbench.com's abstract; colsum holds the group sums the selection ranks.
 * For inspection and tests; valid after the stage that writes them.
 * INVALID_ARG for a shape mcs_plan_workspace_size rejects.
 */
mcs_status mcs_plan_workspace_offsets(int B, int H, int N, int d, int G, int k, size_t *row_m,
                                      size_t *row_l, size_t *O32, size_t *colsum);

/*
 * The plan's steps one by one.  mcs_plan is exactly mcs_plan_group,
 * mcs_plan_stats, mcs_plan_scores, mcs_plan_topk and mcs_plan_residual in this
 * order on one workspace (>= mcs_plan_workspace_size(B,H,N,d,G,k) bytes).
 * The later steps read what the earlier ones left in the workspace, so they
 * must run in this order, on the same workspace and the same shape; any
 * grouping perm (a permutation per head) and any valid selection may be fed
 * in between.
 */

/* a1: perm int32 [B,H,N]. */
mcs_status mcs_plan_group(const void *Q, int B, int H, int N, int d, int32_t *perm,
                          void *workspace, size_t workspace_bytes, mcs_stream_t stream);

/* a2: exact softmax row statistics over all N keys and the dense output in
 * fp32 (split-precision P.V) into the workspace; O_dense (bf16, optional, may
 * be NULL) receives the same dense output rounded to bf16. */
mcs_status mcs_plan_stats(const void *Q, const void *K, const void *V, int B, int H, int N, int d,
                          int G, int k, float scale, void *O_dense, void *workspace,
                          size_t workspace_bytes, mcs_stream_t stream);

/* a3: group probability sums colsum[b,h,g,j] = sum_{i in group g} P_ij into
 * the workspace, for the grouping `perm`.  Needs mcs_plan_stats first. */
mcs_status mcs_plan_scores(const void *Q, const void *K, const int32_t *perm, int B, int H,
                           int N, int d, int G, int k, float scale, void *workspace,
                           size_t workspace_bytes, mcs_stream_t stream);

/* a4: per group the min(k,N) largest scores, ties to the lower key index,
 * ascending -> kv_idx int32 [B,H,ceil(N/G),min(k,N)].  Needs mcs_plan_scores. */
mcs_status mcs_plan_topk(int B, int H, int N, int d, int G, int k, int32_t *kv_idx,
                         void *workspace, size_t workspace_bytes, mcs_stream_t stream);

/* a4 on caller-supplied scores: the selection mcs_plan_topk applies to the
 * group probability sums (cctest.ai "Individual KV selection"), for any
 * score matrix.  scores: float32 [rows, N] row-major on the device, meant to
 * be >= 0 and finite (the sign bit is ignored, so -x ranks as x; NaN ranks
 * above +inf).  kv_idx: int32 [rows, min(k,N)] on the device, caller-owned:
 * per row the min(k,N) largest scores, ties to the lower index, ascending.
 * rows == 0 is a no-op.  INVALID_ARG for null pointers, rows < 0, N < 1 or
 * k < 1; CUDA for a launch failure.  Asynchronous on `stream`. */
mcs_status mcs_select_topk(const float *scores, int rows, int N, int k, int32_t *kv_idx,
                           mcs_stream_t stream);

/* a5: residual float32 [B,H,N,d] = dense output (from mcs_plan_stats, same
 * Q, K, V) minus the output renormalised over each group's kept keys.  Runs
 * over pairs of groups; their union lists are built in the workspace. */
mcs_status mcs_plan_residual(const void *Q, const void *K, const void *V, const int32_t *perm,
                             const int32_t *kv_idx, int B, int H, int N, int d, int G, int k,
                             float scale, float *residual, void *workspace,
                             size_t workspace_bytes, mcs_stream_t stream);

/*
 * mcs_meta_pairs -- build meta->pair_idx and meta->pair_len (layout above)
 * from meta->kv_idx, e.g. for metadata made or loaded outside mcs_plan.
 * kv_idx must hold ascending unique lists (as mcs_plan writes them); other
 * input gives wrong lists but no out-of-bounds access.  Asynchronous.
 * INVALID_ARG for a null pointer or inconsistent sizes.
 */
mcs_status mcs_meta_pairs(const mcs_meta *meta, mcs_stream_t stream);

/*
 * mcs_sparse_step -- step a6, the reused denoising step: for every group g,
 *   O_i = sum_{j in S_g} softmax_j(scale Q_i.K_j) V_j + R_i   (i in g)
 * on the current step's Q, K, V with the cached groups, indices and residual
 * (aiqbench.com abstract: metadata "reused across subsequent denoising
 * steps"; cnshai.top section "MC-Sparse: three failure modes, one fix").
 * O: bf16 [B,H,N,d], original token order.  Needs no workspace.  With
 * meta->pair_idx / ->pair_len set it runs over pairs of groups sharing one
 * gathered key list (the same result up to fp32 summation order); without
 * them, one group at a time.  A pair_len outside [k, 2k] or an index outside
 * [0, N) is never read past or gathered: it records MCS_ERR_BAD_META in the
 * device status word.
 */
mcs_status mcs_sparse_step(const void *Q, const void *K, const void *V, const mcs_meta *meta,
                           float scale, void *O, mcs_stream_t stream);

/*
 * mcs_residual_compact -- the cached residual stored compactly: bf16 copy
 * residual_bf16[i] = round-to-nearest-even(residual[i]) of n float32 values
 * (e.g. n = B*H*N*d for meta->residual).  Both pointers 16-byte aligned
 * device memory (INVALID_ARG otherwise); n = 0 is a no-op.  Asynchronous.
 * The bf16 copy holds each value to 2^-9 relative; it halves what the reused
 * step reads per row and what a cached plan keeps per token.
 */
mcs_status mcs_residual_compact(const float *residual, size_t n, void *residual_bf16, mcs_stream_t stream);

/*
 * mcs_sparse_step_compact -- mcs_sparse_step with the residual read from a
 * bf16 copy (mcs_residual_compact, bf16 [B,H,N,d]) instead of
 * meta->residual, which is not read and may be NULL.  Needs the pair lists
 * (meta->pair_idx / ->pair_len; INVALID_ARG without them).  The result equals
 * mcs_sparse_step's on a residual whose values are the bf16 copy's.
 * Asynchronous; needs no workspace.
 */
mcs_status mcs_sparse_step_compact(const void *Q, const void *K, const void *V, const mcs_meta *meta,
                                   const void *residual_bf16, float scale, void *O, mcs_stream_t stream);

/*
 * mcs_dense -- step a7, dense attention O = softmax(scale Q K^T) V, the
 * comparison baseline the pages measure against ("relative to dense
 * attention", aiqbench.com abstract).  O: bf16 [B,H,N,d].
 */
mcs_status mcs_dense(const void *Q, const void *K, const void *V, int B, int H, int N, int d,
                     float scale, void *O, mcs_stream_t stream);

/* Bytes of workspace mcs_validate_meta needs (one byte per token). */
size_t mcs_validate_workspace_size(int B, int H, int N);

/*
 * Check cached metadata on the device: perm is a permutation per head,
 * kv_idx entries are in [0, N) and strictly ascending per group, the
 * residual is finite, and (when present) every pair_len lies in [k, 2k]
 * (exactly k for a lone last group) with its list's entries in [0, N).
 * Synchronous: waits for `stream`.  Returns MCS_OK or MCS_ERR_BAD_META;
 * *first_bad (may be NULL) receives a code of the first failed check:
 * 1 perm, 2 kv_idx range, 3 kv_idx order, 4 residual, 5 pair lists.
 * Never traps.
 */
mcs_status mcs_validate_meta(const mcs_meta *meta, void *workspace, size_t workspace_bytes,
                             int *first_bad, mcs_stream_t stream);

/*
 * mcs_validate_meta_noalloc -- the same checks as mcs_validate_meta, for
 * callers that cannot hand over a device workspace.  The pages describe no
 * such call; it exists for users of this library whose code may not call
 * cudaMalloc at the point of the check: runtimes that forbid device
 * allocation after start-up (a serving process that reserves all memory at
 * launch), and plugins that only receive raw pointers from a host framework
 * that owns all device memory and its allocator.
 *
 * Scratch: a fixed array compiled into the library, one per device that
 * loads it, held until the process exits: 256 bytes + one bit per token,
 * MCS_NOALLOC_MAX_TOKENS tokens (B*H*N) at most; larger shapes return
 * MCS_ERR_TOO_LARGE before anything is launched.  Nothing is allocated.
 * The first call on a device looks up that device's address of the array
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * Every call clears the scratch it uses, so a call never sees an earlier
 * call's contents, but calls that overlap on the GPU (two streams, or two
 * host threads on one device) share the array and race.  Synchronous, like
 * mcs_validate_meta; returns MCS_OK, MCS_ERR_BAD_META (with *first_bad) or
 * an argument / CUDA error.
 */
#define MCS_NOALLOC_MAX_TOKENS (1u << 23)
mcs_status mcs_validate_meta_noalloc(const mcs_meta *meta, int *first_bad, mcs_stream_t stream);

/*
 * Ablation tools -- the selection rules MC-Sparse replaces, for controlled
 * comparisons of its three failure modes (aiqbench.com abstract:
 * "constraints imposed by token grouping, inaccurate interaction selection,
 * and the attention contributions lost"; cnshai.top post, section "MC-Sparse:
 * three failure modes, one fix").  Their key lists feed mcs_plan_residual and
 * mcs_sparse_step like any other selection.  Not on the hot path.
 */

/* Bytes of workspace mcs_select_blocks needs; 0 for invalid sizes. */
size_t mcs_select_blocks_workspace_size(int rows, int N, int block, int k_blocks);

/* Block-granular selection: per row of `scores` (float32 [rows, N], >= 0,
 * e.g. the group probability sums), the keys are cut into aligned blocks of
 * `block` keys (a ragged last block is not a candidate), a block scores the
 * sum of its keys' scores, the k_blocks highest blocks are kept (ties to the
 * lower block index) and their keys written ascending to kv_idx (int32
 * [rows, k_blocks * block]).  1 <= k_blocks <= N / block, else INVALID_ARG.
 * workspace: >= mcs_select_blocks_workspace_size(...) bytes, 256-byte
 * aligned.  Asynchronous. */
mcs_status mcs_select_blocks(const float *scores, int rows, int N, int block, int k_blocks, int32_t *kv_idx,
                             void *workspace, size_t workspace_bytes, mcs_stream_t stream);

/* Pooled-query scores: for each group g of the grouping `perm` (int32
 * [B,H,N]), its queries averaged into one query qbar_g, and scores[b,h,g,j] =
 * softmax_j(scale qbar_g . K_j) (float32 [B,H,ceil(N/G),N]): a heuristic in
 * place of the exact summed probabilities; select with mcs_select_topk.  Same
 * Q/K conventions as mcs_plan; G in {64, 128}.  Asynchronous. */
mcs_status mcs_pooled_scores(const void *Q, const void *K, const int32_t *perm, int B, int H, int N, int d, int G,
                             float scale, float *scores, mcs_stream_t stream);

/* Block-granular selection as block indices: as mcs_select_blocks, but the
 * kept blocks' indices b (keys [b*block, (b+1)*block)) are written ascending
 * to blk_idx (int32 [rows, k_blocks]) instead of their keys.  Same workspace
 * (mcs_select_blocks_workspace_size) and errors.  Asynchronous. */
mcs_status mcs_select_block_indices(const float *scores, int rows, int N, int block, int k_blocks,
                                    int32_t *blk_idx, void *workspace, size_t workspace_bytes,
                                    mcs_stream_t stream);

/* Union lists of group pairs (the pair_idx / pair_len layout above) from any
 * ascending unique per-group lists `lists` (int32 [B,H,n_groups,k]): keys as
 * kv_idx, or block indices for mcs_sparse_step_blocks.  pair_idx int32
 * [B,H,ceil(n_groups/2),2k], pair_len int32 [B,H,ceil(n_groups/2)].
 * Unsorted input gives wrong lists but no out-of-bounds access.
 * INVALID_ARG for a null pointer or k < 1; UNSUPPORTED for B*H > 65535.
 * Asynchronous. */
mcs_status mcs_union_pairs(const int32_t *lists, int B, int H, int n_groups, int k, int32_t *pair_idx,
                           int32_t *pair_len, mcs_stream_t stream);

/*
 * mcs_sparse_step_blocks -- the reused step over a block-granular selection,
 * the coarse-block pattern that MC-Sparse's individual KV selection replaces
 * (cctest.ai article, "Individual KV selection"; cnshai.top post, section
 * "MC-Sparse: three failure modes, one fix": dropping whole blocks evicts
 * wanted tokens).  For every group g with kept blocks S_g:
 *   O_i = sum_{j in keys of S_g} softmax_j(scale Q_i.K_j) V_j (+ R_i)   (i in g)
 * Each 64-key tile is one contiguous TMA box per 64 columns instead of a row
 * gather; everything else is the pair kernel of mcs_sparse_step.
 * perm: int32 [B,H,N] grouping (as mcs_plan writes it).
 * pair_idx / pair_len: union lists of the groups' ascending block indices
 *   (mcs_union_pairs over int32 [B,H,n_groups,k_blocks]).
 * residual: float32 [B,H,N,d] added in the epilogue, or NULL for none.
 * block in {64, 128} (UNSUPPORTED otherwise), 1 <= k_blocks <= N / block
 * (INVALID_ARG otherwise).  O: bf16 [B,H,N,d].  A block index outside
 * [0, N / block) or a pair_len outside [k_blocks, 2 k_blocks] is never read
 * past: it records MCS_ERR_BAD_META in the device status word.
 * Given the expanded keys of the same blocks as kv_idx, mcs_sparse_step
 * (with pair lists) visits the same tiles in the same order and writes the
 * same bits.  Asynchronous; needs no workspace.
 */
mcs_status mcs_sparse_step_blocks(const void *Q, const void *K, const void *V, int B, int H, int N, int d, int G,
                                  int block, int k_blocks, const int32_t *perm, const int32_t *pair_idx,
                                  const int32_t *pair_len, const float *residual, float scale, void *O,
                                  mcs_stream_t stream);

/* Synchronise `stream`, then read and clear this device's status word.
 * Returns MCS_OK, or MCS_ERR_TIMEOUT if a kernel's bounded wait ran out
 * since the last read. */
mcs_status mcs_last_device_status(mcs_stream_t stream);

/* Self-test of the bounded device wait: launches one kernel that waits on an
 * mbarrier nothing ever arrives on; after `limit_ns` (0 = 1 ms) it gives up,
 * records MCS_ERR_TIMEOUT in the status word and returns normally, leaving
 * the context usable.  Asynchronous; read the outcome with
 * mcs_last_device_status(). */
mcs_status mcs_selftest_wait_timeout(uint64_t limit_ns, mcs_stream_t stream);

/* Upper bound, in nanoseconds, on any single wait inside the kernels
 * (default 4e9).  A kernel whose wait runs out records MCS_ERR_TIMEOUT and
 * returns cleanly.  0 restores the default. */
void mcs_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* MCS_H_ */
