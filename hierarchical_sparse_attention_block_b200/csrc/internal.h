// Launchers shared between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hisa.h"

namespace hisa {

// Validated problem shape (see hisa_params_t in hisa.h).
struct Shape {
  int batch;
  int64_t n_q, n_kv;
  int d_idx, B, m, k, H, Hkv, d;
  float scale;      // softmax scale, already resolved
  int64_t n_blk;    // ceil(n_kv / B)
  int64_t n_query;  // batch * n_q
  int HI = 0;                    // indexer heads: 0 = one head scored by a dot product
  const float* w_idx = nullptr;  // [n_query][HI] head weights when HI >= 1
};

// Shape of a request (the validation every call shares; see hisa.h).  need_attn: the attention
// fields matter.  with_weights then checks idx_weights against n_idx_heads and keeps it.
hisa_status_t make_shape(const hisa_params_t* p, bool need_indexer, bool need_attn, Shape* s);
hisa_status_t set_idx_weights(Shape* s, const float* idx_weights);

// Step 1: block means for blocks [b0, b1) of every sequence.
cudaError_t launch_block_pool(const Shape& s, const void* k_idx, int64_t b0, int64_t b1, float* block_keys,
                              cudaStream_t st);

// Step 2 (CUDA cores): scores[q][j] = q_idx[q] . block_keys[j] for j <= own block.
cudaError_t launch_block_score(const Shape& s, const void* q_idx, const float* block_keys, float* scores,
                               cudaStream_t st);

// Step 2 on the tensor cores (prefill): same output as launch_block_score.
// Returns cudaErrorNotSupported when the shape is outside the kernel's range.
// status (nullable): bit 1 is set if a bounded wait timed out.
cudaError_t launch_block_score_tc(const Shape& s, const void* q_idx, const float* block_keys, float* scores,
                                  int32_t* status, cudaStream_t st);
size_t block_score_tc_scratch_bytes(const Shape& s);
bool block_score_tc_eligible(const Shape& s);

// Step 3: block_idx from scores.
cudaError_t launch_block_topm(const Shape& s, const float* scores, int32_t* block_idx, float* block_scores,
                              cudaStream_t st);

// Steps 4-5 over queries [q0, q0 + nq) (global query ids).  `slots` is the
// number of block slots per query: m with a block list; for the flat indexer
// (block_idx == nullptr) a window of consecutive blocks, slot r being block
// blk_lo + r.  keys: [nq][slots * B].
cudaError_t launch_token_score(const Shape& s, const void* q_idx, const void* k_idx, const int32_t* block_idx,
                               int slots, uint32_t* keys, int32_t* status, int64_t q0, int64_t nq, cudaStream_t st,
                               int blk_lo = 0);
// Tensor-core version of launch_token_score for prefill (same key layout).
bool token_score_tc_eligible(const Shape& s, int slots);
cudaError_t launch_token_score_tc(const Shape& s, const void* q_idx, const void* k_idx, const int32_t* block_idx,
                                  int slots, uint32_t* keys, int32_t* status, int64_t q0, int64_t nq, cudaStream_t st,
                                  int blk_lo = 0);
// Writes row q (global query id) of the result at token_idx[q * k] (token_scores likewise).
cudaError_t launch_token_select(const Shape& s, const uint32_t* keys, const int32_t* block_idx, int slots,
                                int32_t* token_idx, float* token_scores, int64_t q0, int64_t nq, cudaStream_t st,
                                int blk_lo = 0);
// The flat indexer's streaming top-k for one window after the first: per row r (rows of it), the
// best k of the running list (run_ids / run_scores [rows][k], tokens below the window) and the
// window's n keys (keys [rows][n], tokens tok0 ..), by (score desc, token asc), ascending.
// out_scores may be null.
cudaError_t launch_flat_select(const uint32_t* keys, int n, const int32_t* run_ids, const float* run_scores, int k,
                               int64_t tok0, int64_t rows, int32_t* out_ids, float* out_scores, cudaStream_t st);

// Step 6.  The kernel is picked from the shape and the workspace: the query-tile kernel when it
// applies and `ws` holds its masks, else the gather kernels, with the token lists split across CTAs
// (few queries) when `ws` holds the partial states.  attn_workspace_bytes: what lets every path run.
int attn_pick_splits(const Shape& s);
size_t attn_partial_bytes(const Shape& s, int splits);
size_t attn_workspace_bytes(const Shape& s);
cudaError_t launch_sparse_attn(const Shape& s, const void* q, const void* k, const void* v, const int32_t* token_idx,
                               void* o, float* lse, int32_t* status, void* ws, size_t ws_bytes, cudaStream_t st);
// Step 6 for many queries per sequence: tiles of 128 queries x 128 keys on the tensor cores with
// the selections as bit masks (ws: sparse_attn_qtile_bytes of device memory for the masks and an
// fp16 copy of V).
bool sparse_attn_qtile_eligible(const Shape& s);
size_t sparse_attn_qtile_bytes(const Shape& s);
cudaError_t launch_sparse_attn_qtile(const Shape& s, const void* q, const void* k, const void* v,
                                     const int32_t* token_idx, void* o, float* lse, int32_t* status, void* ws,
                                     cudaStream_t st);
// Merge of the per-split (max, sum, output) states into O and the LSE.
cudaError_t launch_attn_merge(const Shape& s, const float* partial, void* o, float* lse, int splits, cudaStream_t st);
// Step 6 on the tensor cores (tcgen05, TMA gather), head dimension 128; cudaErrorNotSupported
// when the shape is outside its range.
bool sparse_attn_tc_eligible(const Shape& s);
cudaError_t launch_sparse_attn_tc(const Shape& s, const void* q, const void* k, const void* v,
                                  const int32_t* token_idx, void* o, float* lse, int32_t* status, int splits,
                                  float* partial, cudaStream_t st);

// Context-parallel decode (see the hisa_block_candidates family in hisa.h).
cudaError_t launch_block_candidates(const Shape& s, const float* scores, int64_t first, int64_t c, int r,
                                    float* cand_scores, int32_t* cand_ids, cudaStream_t st);
cudaError_t launch_topk_merge(const float* scores, const int32_t* ids, int n_parts, int64_t rows, int n_per, int k,
                              int32_t* out_ids, float* out_scores, cudaStream_t st);
cudaError_t launch_remap_ids(const int32_t* in, int64_t rows, int cols, int64_t lo, int64_t hi, int64_t delta,
                             int32_t* out, cudaStream_t st);
cudaError_t launch_lse_merge(const void* o_parts, const float* lse_parts, int G, int64_t rows, int d, void* o,
                             float* lse, cudaStream_t st);

// Measurement helper: gathers of hashed rows into shared memory (see hisa_gather_probe).
bool gather_probe_row_bytes_ok(int row_bytes);
cudaError_t launch_gather_probe(const void* rows, int64_t n_rows, int row_bytes, int64_t n_gathers, uint32_t seed,
                                uint32_t* sink, int ctas_per_sm, cudaStream_t st);

// cudaError_t value behind the last HISA_ERR_CUDA on this host thread.
extern thread_local int32_t g_last_cuda_error;

// Raises a kernel's dynamic shared-memory limit to `bytes` (once per device and kernel) when
// `bytes` plus the kernel's static shared memory exceed the default 48 KiB.
cudaError_t ensure_smem(const void* func, int bytes, int static_bytes = 0);

}  // namespace hisa
