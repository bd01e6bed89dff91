// Decode with the context split across ranks: the pieces that let each rank
// run the path on its own slice of the KV cache and exchange only small
// candidate lists.
//
// A rank owns tokens [t0, t0 + n_loc) of every sequence (t0 a multiple of the
// block size B), so it owns whole blocks [t0 / B, (t0 + n_loc) / B).  The
// selection rule of steps 3 and 5 ("北大HISA稀疏注意力机制" section 1.2.1 item 3
// and section 1.2.2 item 2: the best scores, ties to the lower index, the
// first and the query's own block always kept) is a total order, so the
// global best r are among the union of every rank's best r; and softmax
// attention over a union of disjoint token sets is the log-sum-exp merge of
// the per-set results.  The kernels here:
//   * block_candidates_kernel: this rank's best top_m - 2 blocks among blocks
//     1 .. c - 1 plus the forced blocks 0 and c it owns (score +inf), as
//     (score, global block id) pairs in ascending id order;
//   * topk_merge_kernel: the best k of (score, id) candidates that arrive in
//     ascending id order (the rank-major all-gather of per-rank lists that are
//     each ascending), written as ascending ids, -1 padded;
//   * remap_ids_kernel: ids inside [lo, hi) shifted by delta, compacted in
//     order, -1 padded (global <-> shard-local numbering);
//   * lse_merge_kernel: O = sum_g exp(lse_g - L) O_g / sum_g exp(lse_g - L),
//     LSE = L + ln sum_g exp(lse_g - L).
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace hisa {
namespace {

constexpr int kCandThreads = 256;

// One CTA per query row.  scores: [rows][n_blk_loc] from the block scorer (every local block).
__global__ void __launch_bounds__(kCandThreads)
    block_candidates_kernel(const float* __restrict__ scores, int64_t n_blk_loc, int64_t first, int64_t c, int r,
                            float* __restrict__ cand_scores, int32_t* __restrict__ cand_ids) {
  __shared__ SelectShared<kCandThreads> sm;
  const int64_t row = blockIdx.x;
  const float* sc = scores + row * n_blk_loc;
  const int width = r + 2;
  float* os = cand_scores + row * width;
  int32_t* oi = cand_ids + row * width;
  const uint32_t kForced = score_key(INFINITY);
  auto key = [&](int j) -> uint32_t {
    const int64_t g = first + j;
    if (g == 0 || g == c) return kForced;
    return (g >= 1 && g < c) ? score_key(sc[j]) : 0u;
  };
  const int n = (int)n_blk_loc;
  const int nv = count_nonzero<kCandThreads>(key, n, sm);
  int n_forced = 0;
  if (first <= 0 && 0 < first + n_blk_loc) ++n_forced;
  if (c > 0 && first <= c && c < first + n_blk_loc) ++n_forced;
  const int K = min(r + n_forced, nv);
  int emitted = 0;
  if (K > 0) {
    const SelectResult sel = (K == nv) ? select_all_nonzero() : radix_select<kCandThreads>(key, n, K, sm);
    emitted = emit_selected<kCandThreads>(key, n, sel, sm, [&](int j, int rank) {
      const int64_t g = first + j;
      os[rank] = (g == 0 || g == c) ? INFINITY : sc[j];
      oi[rank] = (int32_t)g;
    });
  }
  for (int i = emitted + threadIdx.x; i < width; i += kCandThreads) {
    os[i] = __int_as_float(0x7FC00000);
    oi[i] = -1;
  }
}

// Candidates of row `row`: part g's entries [g][row][0 .. n_per), taken part after part.
template <int NT>
__global__ void __launch_bounds__(NT)
    topk_merge_kernel(const float* __restrict__ scores, const int32_t* __restrict__ ids, int n_parts, int64_t rows,
                      int n_per, int k, int32_t* __restrict__ out_ids, float* __restrict__ out_scores) {
  __shared__ SelectShared<NT> sm;
  const int64_t row = blockIdx.x;
  const int n_cand = n_parts * n_per;
  auto at = [&](int j) -> int64_t { return ((int64_t)(j / n_per) * rows + row) * n_per + j % n_per; };
  auto key = [&](int j) -> uint32_t {
    const int64_t a = at(j);
    return ids[a] >= 0 ? score_key(scores[a]) : 0u;
  };
  const int nv = count_nonzero<NT>(key, n_cand, sm);
  const int K = min(k, nv);
  int32_t* oi = out_ids + row * (int64_t)k;
  float* os = out_scores ? out_scores + row * (int64_t)k : nullptr;
  if (K > 0) {
    const SelectResult sel = (K == nv) ? select_all_nonzero() : radix_select<NT>(key, n_cand, K, sm);
    emit_selected<NT>(key, n_cand, sel, sm, [&](int j, int rank) {
      const int64_t a = at(j);
      oi[rank] = ids[a];
      if (os) os[rank] = scores[a];
    });
  }
  for (int i = K + threadIdx.x; i < k; i += NT) {
    oi[i] = -1;
    if (os) os[i] = __int_as_float(0x7FC00000);
  }
}

// One warp per row.  `in` and `out` may be the same array: a chunk is read before anything at
// or after it is written.
__global__ void __launch_bounds__(256) remap_ids_kernel(const int32_t* in, int64_t rows, int cols, int64_t lo,
                                                        int64_t hi, int64_t delta, int32_t* out) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int32_t* a = in + row * cols;
  int32_t* b = out + row * cols;
  int n = 0;
  for (int c0 = 0; c0 < cols; c0 += 32) {
    const int c = c0 + lane;
    const int64_t v = c < cols ? (int64_t)a[c] : -1;
    const bool keep = v >= 0 && v >= lo && v < hi;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) b[n + __popc(m & ((1u << lane) - 1u))] = (int32_t)(v + delta);
    n += __popc(m);
  }
  for (int c = n + lane; c < cols; c += 32) b[c] = -1;
}

// One thread per (row, dimension).  o_parts: [G][rows][d] bf16, lse_parts: [G][rows].
__global__ void lse_merge_kernel(const uint16_t* __restrict__ o_parts, const float* __restrict__ lse_parts, int G,
                                 int64_t rows, int d, uint16_t* __restrict__ o, float* __restrict__ lse) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= rows * d) return;
  const int64_t row = t / d;
  float L = -INFINITY;
  for (int g = 0; g < G; ++g) L = fmaxf(L, lse_parts[g * rows + row]);
  float s = 0.f, acc = 0.f;
  if (L != -INFINITY) {
    for (int g = 0; g < G; ++g) {
      const float wgt = expf(lse_parts[g * rows + row] - L);
      s += wgt;
      acc = fmaf(wgt, bf16_lo((uint32_t)o_parts[g * rows * d + t]), acc);
    }
  }
  const __nv_bfloat16 ob = __float2bfloat16_rn(s > 0.f ? acc / s : 0.f);
  o[t] = *reinterpret_cast<const uint16_t*>(&ob);
  if (lse && t % d == 0) lse[row] = s > 0.f ? L + logf(s) : -INFINITY;
}

}  // namespace

cudaError_t launch_block_candidates(const Shape& s, const float* scores, int64_t first, int64_t c, int r,
                                    float* cand_scores, int32_t* cand_ids, cudaStream_t st) {
  block_candidates_kernel<<<(unsigned)s.n_query, kCandThreads, 0, st>>>(scores, s.n_blk, first, c, r, cand_scores,
                                                                         cand_ids);
  return cudaGetLastError();
}

cudaError_t launch_topk_merge(const float* scores, const int32_t* ids, int n_parts, int64_t rows, int n_per, int k,
                              int32_t* out_ids, float* out_scores, cudaStream_t st) {
  if ((int64_t)n_parts * n_per <= 4096)
    topk_merge_kernel<256><<<(unsigned)rows, 256, 0, st>>>(scores, ids, n_parts, rows, n_per, k, out_ids, out_scores);
  else
    topk_merge_kernel<1024><<<(unsigned)rows, 1024, 0, st>>>(scores, ids, n_parts, rows, n_per, k, out_ids,
                                                             out_scores);
  return cudaGetLastError();
}

cudaError_t launch_remap_ids(const int32_t* in, int64_t rows, int cols, int64_t lo, int64_t hi, int64_t delta,
                             int32_t* out, cudaStream_t st) {
  remap_ids_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(in, rows, cols, lo, hi, delta, out);
  return cudaGetLastError();
}

cudaError_t launch_lse_merge(const void* o_parts, const float* lse_parts, int G, int64_t rows, int d, void* o,
                             float* lse, cudaStream_t st) {
  const int64_t n = rows * d;
  lse_merge_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(static_cast<const uint16_t*>(o_parts), lse_parts, G,
                                                                 rows, d, static_cast<uint16_t*>(o), lse);
  return cudaGetLastError();
}

}  // namespace hisa
