/*
 * hisa.h -- C ABI of the two-level (block -> token) sparse-attention indexer
 * and of the sparse attention that consumes its output, for NVIDIA B200
 * (sm_100a).
 *
 * The method (sources cited by short key):
 *   [IP] "北大HISA稀疏注意力机制：长文本处理效率提升3倍" (intelliparadigm.com):
 *        section 1.2.1 "块级粗过滤" (coarse block filtering), section 1.2.2
 *        "块内精筛选" (fine token selection), section 3.2 (block sizes 64/128/256).
 *   [QB] QbitAI article on HISA (m.digipub.cc, KPSAJS2O0511DSSR): sections
 *        "塊級粗過濾", "塊內精挑字符" and "HISA的關鍵優勢在於" (cost
 *        O(L^2/B + L*m*B); output format and attention unchanged).
 *
 *   1. cut each sequence's indexer keys into blocks of B tokens and mean-pool
 *      every block into one block key;
 *   2. score each query against the block keys it can see with the
 *      indexer's score (below);
 *   3. keep m blocks: block 0, the query's own block c = floor(p/B), and the
 *      m-2 best of blocks 1..c-1 (all visible blocks when c+1 <= m);
 *   4. score the query against the tokens t <= p of those blocks;
 *   5. keep the k best tokens (ties: lower index first);
 *   6. softmax attention of every head over just those tokens.
 *
 * Conventions shared by every call
 *   - Tensors are dense, row-major, in DEVICE memory, owned by the caller
 *     (hisa_forward_host alone takes its inputs and outputs in host memory).
 *     The library allocates nothing; calls that need scratch take a caller
 *     workspace whose size the matching *_workspace_size call reports.
 *   - bf16 tensors are passed as void* (__nv_bfloat16 elements).  Base
 *     pointers must be 16-byte aligned.
 *   - Shapes (b = batch, H = n_heads, Hk = n_kv_heads, d = d_head):
 *       q_idx  [b][n_q][d_idx]  bf16     k_idx   [b][n_kv][d_idx] bf16
 *         ([b][n_q][Hi][d_idx] with an Hi-head indexer, idx_weights
 *          [b][n_q][Hi] fp32)
 *       block_keys [b][ceil(n_kv/B)][d_idx] fp32
 *       block_idx  [b][n_q][m]  int32    token_idx [b][n_q][k] int32
 *       q [b][n_q][H][d] bf16   k, v [b][n_kv][Hk][d] bf16
 *       o [b][n_q][H][d] bf16   lse [b][n_q][H] fp32 (natural log)
 *     Query i of a sequence sits at position p_i = n_kv - n_q + i
 *     (prefill: n_q = n_kv; decode: n_q = 1, p = n_kv - 1).
 *   - The indexer's score of a key kv (a block key in step 2, a token's
 *     k_idx row in step 4) is the original indexer's own score function
 *     ([IP] 1.2.1 item 2, 1.3 item 4 "Score Function Consistency"):
 *       n_idx_heads = 0:   q . kv                         (one head);
 *       n_idx_heads = Hi:  sum_j w_j * max(0, q_j . kv)   (Hi heads q_j with
 *                          the query's head weights w_j = idx_weights, the
 *                          multi-head indexer form of DeepSeek-V3.2).
 *     idx_weights must be NULL when n_idx_heads is 0 and non-NULL otherwise.
 *     With many queries per sequence both forms are scored on the tensor
 *     cores (the Hi-head form for Hi in {1, 2, 4, 8, 16}); other Hi and
 *     decode run on CUDA-core scorers.  Integer inputs and integer weights
 *     keep every score exact while |scores| * B < 2^24.
 *   - Index lists are ascending with -1 padding at the tail.  Ties in a
 *     selection go to the lower block / token index.
 *   - Every call validates its arguments on the host before launching
 *     anything (HISA_ERR_INVALID_ARG / HISA_ERR_UNSUPPORTED /
 *     HISA_ERR_WORKSPACE) and then only enqueues work on `stream`; results
 *     are ready when the stream reaches them (hisa_forward_host returns with
 *     its results in host memory).  A launch failure returns
 *     HISA_ERR_CUDA; hisa_last_cuda_error() gives the cudaError_t value.
 *   - Index lists given as INPUT are checked on the device: an entry that is
 *     out of range (below -1, beyond the query's own block / position, or not
 *     greater than every in-range entry before it) is skipped, never
 *     dereferenced, and bit 0 of *dev_status is set (atomicOr).  No kernel
 *     traps or waits unboundedly: a wait that runs out (1 s) sets bit 1 of
 *     *dev_status and the results of that call are not valid.
 *   - Supported sizes: d_idx in {64, 128, 256}; n_idx_heads in [0, 16];
 *     d_head in {64, 128}; B a
 *     power of two in [1, 4096]; m >= 2; k >= 1; n_heads a multiple of
 *     n_kv_heads; n_kv < 2^31.  Integer-valued indexer inputs (|x| <= 4)
 *     make every block mean and score exact in fp32, so selections are exact.
 */
#ifndef HISA_H
#define HISA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum hisa_status {
  HISA_OK = 0,
  HISA_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misaligned pointer */
  HISA_ERR_UNSUPPORTED = 2, /* valid request outside the sizes listed above */
  HISA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
  HISA_ERR_CUDA = 4         /* a CUDA call failed; see hisa_last_cuda_error() */
} hisa_status_t;

/* Problem description.  scale <= 0 selects 1/sqrt(d_head).  flags must be 0.
 * n_idx_heads: 0 for a one-head dot-product indexer, Hi in [1, 16] for the
 * Hi-head weighted form (see the conventions above). */
typedef struct hisa_params {
  int32_t batch;      /* b: independent sequences of equal length */
  int32_t d_idx;      /* indexer head dimension */
  int64_t n_q;        /* queries per sequence: the last n_q positions */
  int64_t n_kv;       /* keys per sequence */
  int32_t block;      /* B: tokens per block */
  int32_t top_m;      /* m: blocks kept per query (forced blocks included) */
  int32_t top_k;      /* k: tokens kept per query */
  int32_t n_heads;    /* H: attention query heads */
  int32_t n_kv_heads; /* Hk: attention key/value heads (H % Hk == 0) */
  int32_t d_head;     /* d: attention head dimension */
  float scale;        /* softmax scale tau */
  int32_t flags;      /* reserved, 0 */
  int32_t n_idx_heads; /* Hi: indexer query heads (0: one head, plain dot product) */
} hisa_params_t;

/* Step 1 -- [IP] 1.2.1 item 1; [QB] "塊級粗過濾" bullet 1.
 * block_keys[s][j][:] = mean of k_idx[s][t][:] over the tokens t of block j
 * (B of them, fewer in a final partial block), fp32, for blocks
 * j in [blk_begin, blk_end) of every sequence; blk_end < 0 means the last
 * block.  Other rows of block_keys are left untouched, so a decode loop can
 * refresh only the newest block. */
hisa_status_t hisa_block_pool(const hisa_params_t* params, const void* k_idx, int64_t blk_begin,
                              int64_t blk_end, float* block_keys, cudaStream_t stream);

/* Steps 2-3 -- [IP] 1.2.1 items 2-3; [QB] "塊級粗過濾" bullets 2-3 and the
 * forced first/last block remark of "塊內精挑字符".
 * block_idx[s][i][0..m): the min(m, c+1) kept blocks, ascending, -1 padded.
 * block_scores (nullable) [b][n_q][m] fp32: the indexer score of each kept block
 * (NaN for padding).  dev_status (nullable): see conventions.  Workspace:
 * hisa_block_topm_workspace_size bytes.  With many queries per sequence the
 * scores come from a tcgen05 tensor-core kernel that splits each fp32 block
 * key into three bf16 terms (fp32-faithful; exact on integer inputs), with
 * few queries from a CUDA-core kernel. */
hisa_status_t hisa_block_topm_workspace_size(const hisa_params_t* params, size_t* bytes);
hisa_status_t hisa_block_topm(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                              const float* block_keys, int32_t* block_idx, float* block_scores, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Steps 4-5 -- [IP] 1.2.2 items 1-2; [QB] "塊內精挑字符".
 * token_idx[s][i][0..k): the min(k, candidates) best tokens t <= p_i of the
 * blocks in block_idx[s][i], ascending, -1 padded (a token whose score is a
 * NaN of negative sign with one of the largest payloads -- no arithmetic
 * produces one -- counts as no candidate).  token_scores (nullable)
 * [b][n_q][k] fp32: their indexer scores (NaN for padding).  dev_status
 * (nullable) int32 on the device, see conventions.  Any workspace of at least
 * the reported minimum works; more lets more queries run per launch. */
hisa_status_t hisa_token_topk_workspace_size(const hisa_params_t* params, size_t* min_bytes,
                                             size_t* preferred_bytes);
hisa_status_t hisa_token_topk(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                              const void* k_idx, const int32_t* block_idx, int32_t* token_idx, float* token_scores,
                              int32_t* dev_status, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Step 6 -- [QB] "HISA的關鍵優勢在於" (the downstream attention is unchanged).
 * For every query i and head h (kv head g = h / (H / Hk)):
 *   o[s][i][h]   = sum_t softmax_t(scale * q[s][i][h] . k[s][t][g]) v[s][t][g]
 *   lse[s][i][h] = ln sum_t exp(scale * q[s][i][h] . k[s][t][g])
 * over the entries t of token_idx[s][i] (-1 skipped).  bf16 inputs, fp32
 * accumulation, bf16 output.  An empty list gives o = 0, lse = -inf.
 * lse and dev_status are nullable.  Workspace may be NULL (then every
 * query/head is one work item of a gather kernel); with
 * hisa_sparse_attn_workspace_size bytes the token list is split across CTAs
 * when there are few queries (decode), and with many queries per sequence and
 * d = 128 the query-tile kernel runs (tiles of 128 queries x 128 keys on the
 * tensor cores, each query's tokens as a bit mask over the key tile; its
 * workspace holds the masks and an fp16 copy of V scaled per KV head by a
 * power of two, and its weights are rounded to fp16: every output stays
 * within 2^-11 * max|v| of the exact weighted sum).  hisa_sparse_attn_kernel
 * tells which kernel a workspace size selects. */
hisa_status_t hisa_sparse_attn_workspace_size(const hisa_params_t* params, size_t* bytes);
hisa_status_t sparse_attn_fwd(const hisa_params_t* params, const void* q, const void* k, const void* v,
                              const int32_t* token_idx, void* o, float* lse, int32_t* dev_status, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/* Which step-6 kernel sparse_attn_fwd runs for these parameters and a workspace of
 * workspace_bytes (0: none): *kind = 1 for the query-tile kernel (many queries per sequence, head
 * dimension 128: tiles of 128 queries against tiles of 128 keys on the tensor cores, the kept
 * tokens as bit masks; it needs the full hisa_sparse_attn_workspace_size), 0 for the gather
 * kernels (each query's kept K/V rows gathered on their own).  No counterpart on the pages: it
 * tells a caller or a benchmark which kernel, and so which roofline, applies. */
hisa_status_t hisa_sparse_attn_kernel(const hisa_params_t* params, size_t workspace_bytes, int32_t* kind);

/* Steps 1-6 in one call.  block_idx_out and token_idx_out (nullable) receive
 * the intermediate selections.  Workspace: hisa_forward_workspace_size. */
hisa_status_t hisa_forward_workspace_size(const hisa_params_t* params, size_t* bytes);
hisa_status_t hisa_forward(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                           const void* k_idx, const void* q, const void* k, const void* v, void* o, float* lse,
                           int32_t* block_idx_out, int32_t* token_idx_out, int32_t* dev_status, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream);

/* Steps 1-6 with the inputs and outputs in HOST memory: q_idx, idx_weights,
 * k_idx, q, k, v are read from the host and o, lse (nullable) written back
 * there, in the layouts above.  Pinned host memory (cudaHostAlloc /
 * cudaHostRegister) lets the copies run asynchronously; pageable memory works
 * but the copies then stall the calling thread.  The device copies of the
 * inputs and outputs live in the caller's device workspace
 * (hisa_forward_host_workspace_size bytes, 16-byte aligned).
 *
 * The copies overlap the work: the indexer inputs go first (on stream) and
 * the indexer runs while copy_stream brings in Q, K and V in query chunks of
 * each sequence (a chunk of queries [i0, i1) needs the K/V rows up to its last
 * position only); attention of a chunk starts as soon as its rows have
 * arrived, and its O/LSE rows go back on copy_stream while the next chunk
 * runs.  With a copy_stream, chunks alternate between stream and a second
 * compute stream the call creates (each with its own part of the workspace),
 * so that a chunk starts on the SMs the previous chunk's last wave leaves
 * idle.  The selections equal hisa_forward's on the same inputs, and so do o
 * and lse bit for bit, except for a chunk or group with so few queries that
 * its token lists are split across CTAs differently (then they differ by the
 * rounding of the split merge), and when a head's V values reach 2^15 (the
 * fp16 scale of V then follows the chunk's rows, not all of them).
 * copy_stream (nullable, or equal to stream) runs the copies; without one
 * everything is serialised on stream.  The call
 * is synchronous: it returns when o and lse are in host memory (it
 * synchronises stream), so it cannot be captured in a CUDA graph.  Returns
 * HISA_ERR_INVALID_ARG when a host argument is device memory. */
hisa_status_t hisa_forward_host_workspace_size(const hisa_params_t* params, size_t* bytes);
hisa_status_t hisa_forward_host(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                                const void* k_idx, const void* q, const void* k, const void* v, void* o, float* lse,
                                int32_t* dev_status, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                                cudaStream_t copy_stream);

/* Steps 1-6 with caller-owned block keys that persist between calls (decode
 * serving, [QB] "HISA的關鍵優勢在於": the KV cache is unchanged, so the pooled
 * block keys of the cache can be kept).  block_keys [b][ceil(n_kv/B)][d_idx]
 * fp32 is read for every block and first rewritten for blocks
 * [refresh_begin, ceil(n_kv/B)): 0 pools everything (e.g. after a prefill),
 * (n_kv - 1) / B refreshes only the block the newest token entered.  Results
 * equal hisa_forward's.  Workspace: hisa_forward_workspace_size bytes. */
hisa_status_t hisa_forward_cached(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                                  const void* k_idx, float* block_keys, int64_t refresh_begin, const void* q,
                                  const void* k, const void* v, void* o, float* lse, int32_t* block_idx_out,
                                  int32_t* token_idx_out, int32_t* dev_status, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/* The flat token indexer the two-level one replaces ([IP] 1.1 item 1; [QB]
 * "兩步消除上下文索引瓶頸"): token_idx[s][i] = the min(k, p_i+1) best tokens
 * t <= p_i of the whole sequence.  Same output format as hisa_token_topk;
 * used as the speed comparator and for the degeneration check.  It runs the
 * token stage's own kernels over windows of consecutive blocks (8192
 * candidate tokens, or k rounded up to blocks, a window) and keeps a running
 * top-k per query, selected again with each window's keys, so no query's
 * whole row of candidates is ever held at once.  Workspace per query row
 * processed at once: the window's keys plus four k-entry arrays; min_bytes holds one row,
 * preferred_bytes all rows (up to 8 GiB), and any size in between is used in
 * chunks of rows.  Errors: HISA_ERR_WORKSPACE when workspace_bytes is below
 * min_bytes or the pointer is not 16-byte aligned; HISA_ERR_UNSUPPORTED for
 * more than 50000 blocks or k of 32768 or more. */
hisa_status_t hisa_flat_topk_workspace_size(const hisa_params_t* params, size_t* min_bytes,
                                            size_t* preferred_bytes);
hisa_status_t hisa_flat_topk(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                             const void* k_idx, int32_t* token_idx, float* token_scores, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/* The token stage (steps 4-5) for callers that cannot allocate device memory.
 * The pages have no counterpart of this call; it exists for users of the
 * library, not for the method.  Same arguments, results and device checks as
 * hisa_token_topk, minus the workspace: some callers only hand a library the
 * buffers they already own (an inference engine that plans all device memory
 * up front and gives plugins no allocator, a latency-critical loop that must
 * not call the synchronizing cudaMalloc, a binding that cannot manage a
 * scratch buffer's lifetime).  The scratch is a file-scope device array of
 * 16 MiB that every GPU loading this part of the library holds until exit;
 * queries run in chunks that fit it, and a request whose single query needs
 * more than 16 MiB of candidate keys (top_m * block * 4 bytes) returns
 * HISA_ERR_UNSUPPORTED.  Nothing is allocated by the call.  The first call on
 * each device looks up the array's device address; make that first call
 * before any stream capture.  The address is looked up again after the
 * device's context is replaced (cudaDeviceReset), which a later call detects
 * by the context's id.  All calls share the array: calls that overlap
 * on the GPU (other streams or host threads) race, so serialize them. */
hisa_status_t hisa_token_topk_noalloc(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                                      const void* k_idx, const int32_t* block_idx, int32_t* token_idx,
                                      float* token_scores, int32_t* dev_status, cudaStream_t stream);

/* ---- Decode with the context split across ranks (context parallelism) ----
 * Rank r owns tokens [t0, t0 + n_loc) of every sequence, t0 = first_block * B
 * (whole blocks; the last rank may end on a partial block), and runs the path
 * on its slice with `local` parameters (n_kv = n_loc, n_q = 1).  The pages
 * describe one device; splitting rests on two facts about the method: the
 * selections of steps 3 and 5 ([IP] 1.2.1 item 3, 1.2.2 item 2; [QB]
 * "塊級粗過濾", "塊內精挑字符") are the best entries under a total order
 * (score descending, index ascending), so the global best r are among the
 * union of every rank's best r; and attention over disjoint token sets merges
 * by log-sum-exp ([QB] "HISA的關鍵優勢在於": the attention itself is unchanged).
 * A step: hisa_block_candidates -> all-gather -> hisa_topk_merge (k = m) ->
 * hisa_remap_ids (global -> local blocks) -> hisa_token_topk (local) ->
 * hisa_remap_ids (local -> global tokens) -> all-gather -> hisa_topk_merge
 * (k) -> hisa_remap_ids (global -> local tokens) -> sparse_attn_fwd (local)
 * -> all-gather -> hisa_lse_merge.  All device pointers, asynchronous. */

/* Scratch for hisa_block_candidates: n_q * batch * ceil(n_kv / B) floats of `local`. */
hisa_status_t hisa_block_candidates_workspace_size(const hisa_params_t* local, size_t* bytes);
/* This rank's block candidates for step 3: its best top_m - 2 blocks among the
 * global blocks 1 .. c - 1 (c = (n_kv_global - 1) / B, the query's own block)
 * by the block score of step 2, plus the forced blocks 0 and c if it owns
 * them (score +inf).  Written as cand_scores / cand_ids [batch][top_m]
 * (global block ids), ascending by id, padded with (NaN, -1).  local.n_q must
 * be 1 (HISA_ERR_UNSUPPORTED otherwise); block_keys are this rank's pooled
 * keys [batch][ceil(n_loc / B)][d_idx]. */
hisa_status_t hisa_block_candidates(const hisa_params_t* local, int64_t n_kv_global, int64_t first_block,
                                    const void* q_idx, const float* idx_weights, const float* block_keys,
                                    float* cand_scores, int32_t* cand_ids, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream);
/* The best k (score descending, id ascending) of each row's candidates, given
 * as n_parts parts of [rows][n_per] each (the rank-major all-gather layout
 * [n_parts][rows][n_per]; entries with id -1 are empty).  Ties are resolved by
 * position, so the candidates must arrive in ascending id order within a row.
 * out_ids [rows][k]: ascending ids, -1 padded; out_scores (nullable) aligned,
 * NaN padded.  n_parts * n_per <= 2^24. */
hisa_status_t hisa_topk_merge(const float* scores, const int32_t* ids, int32_t n_parts, int64_t rows, int32_t n_per,
                              int32_t k, int32_t* out_ids, float* out_scores, cudaStream_t stream);
/* Index renumbering between global and shard-local ids (no counterpart on the
 * pages; argument marshalling between the steps above): for each row of
 * in [rows][cols], the entries with lo <= id < hi, in order, shifted by delta,
 * then -1.  in and out may be the same array. */
hisa_status_t hisa_remap_ids(const int32_t* in, int64_t rows, int32_t cols, int64_t lo, int64_t hi, int64_t delta,
                             int32_t* out, cudaStream_t stream);
/* Attention over disjoint token sets merged: o_parts [n_parts][rows][d] bf16
 * and lse_parts [n_parts][rows] (natural log, -inf for an empty set) ->
 * o [rows][d] bf16, lse [rows] (nullable). */
hisa_status_t hisa_lse_merge(const void* o_parts, const float* lse_parts, int32_t n_parts, int64_t rows, int32_t d,
                             void* o, float* lse, cudaStream_t stream);

/* Measurement helper, not a step of the method (the pages have no
 * counterpart): n_gathers copies of row h(e) (row_bytes each; h a hash of the
 * gather number e and seed, uniform over [0, n_rows)) into shared memory with
 * 16-byte cp.async, the copy pattern of sparse_attn_fwd's gathers without any
 * of its arithmetic or index reads, so that timing it gives that kernel a
 * measured ceiling for rows the L2 serves.  rows: device, [n_rows][row_bytes],
 * 16-byte aligned, n_rows < 2^31; row_bytes 32, 64, 128 or 256; sink: one device word the kernel adds a
 * copied word to, so the copies cannot be optimised away; ctas_per_sm: CTAs
 * of 4 warps launched per SM, 1..3 (64 KB of shared memory each), 0 = 3.
 * Returns HISA_ERR_INVALID_ARG for bad arguments; asynchronous on stream. */
hisa_status_t hisa_gather_probe(const void* rows, int64_t n_rows, int32_t row_bytes, int64_t n_gathers,
                                uint32_t seed, uint32_t* sink, int32_t ctas_per_sm, cudaStream_t stream);

/* Static text for a status code. */
const char* hisa_status_string(hisa_status_t status);
/* cudaError_t value of the last failed CUDA call on this host thread (0 if none). */
int32_t hisa_last_cuda_error(void);
/* Library version string. */
const char* hisa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HISA_H */
