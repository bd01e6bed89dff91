// Steps 2-3: score each query against the block keys it can see and keep m
// blocks, the first block and the query's own block always among them.
// "北大HISA稀疏注意力机制" section 1.2.1 items 2-3; QbitAI HISA article,
// "塊級粗過濾" and the forced first/last block remark of "塊內精挑字符".
//
// block_score_kernel is the CUDA-core scorer (decode: one query per sequence
// makes this a GEMV streaming n_blk * d_idx * 4 B of block keys from HBM);
// block_score_mh_kernel scores with the multi-head weighted form.
// block_topm_kernel runs one CTA per query: the scores of blocks 1..c-1 become
// order-preserving keys in shared memory and a CTA radix selection keeps the
// best m-2 of them (ties to the lower block id).
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace hisa {
namespace {

constexpr int kScoreBlocksPerCta = 64;

template <int D>
__global__ void __launch_bounds__(256) block_score_kernel(const uint16_t* __restrict__ q_idx,
                                                          const float* __restrict__ bk, float* __restrict__ scores,
                                                          int64_t n_q, int64_t n_kv, int B, int64_t n_blk,
                                                          int chunks) {
  constexpr int PER = D / 32;  // dimensions per lane
  const int64_t qg = blockIdx.x / chunks;
  const int chunk = blockIdx.x % chunks;
  const int seq = (int)(qg / n_q);
  const int64_t p = n_kv - n_q + qg % n_q;
  const int64_t c = p / B;
  const int64_t j0 = (int64_t)chunk * kScoreBlocksPerCta;
  if (j0 > c) return;
  const int64_t j1 = min(j0 + kScoreBlocksPerCta, c + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  float qv[PER];
  const uint16_t* qrow = q_idx + qg * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(qrow + e);
    qv[e] = bf16_lo(w);
    qv[e + 1] = bf16_hi(w);
  }
  const float* bks = bk + (int64_t)seq * n_blk * D + lane * PER;
  for (int64_t j = j0 + warp; j < j1; j += 8) {
    const float* row = bks + j * D;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < PER; e += 2) {
      const float2 b2 = *reinterpret_cast<const float2*>(row + e);
      dot = fmaf(qv[e], b2.x, dot);
      dot = fmaf(qv[e + 1], b2.y, dot);
    }
    dot = warp_sum(dot);
    if (lane == 0) scores[qg * n_blk + j] = dot;
  }
}

// The multi-head indexer score sum_j w_j * max(0, q_j . bk) (n_idx_heads = HI >= 1): the query's
// HI heads go to shared memory as fp32, a warp takes one block key at a time (lane = D/32
// dimensions), and the per-head dot products are summed over the warp one head after another.
template <int D>
__global__ void __launch_bounds__(256) block_score_mh_kernel(const uint16_t* __restrict__ q_idx,
                                                             const float* __restrict__ w_idx,
                                                             const float* __restrict__ bk, float* __restrict__ scores,
                                                             int64_t n_q, int64_t n_kv, int B, int64_t n_blk,
                                                             int chunks, int HI) {
  constexpr int PER = D / 32;
  extern __shared__ float sq[];  // [HI][D] query heads, then [HI] weights
  const int64_t qg = blockIdx.x / chunks;
  const int chunk = blockIdx.x % chunks;
  const int seq = (int)(qg / n_q);
  const int64_t p = n_kv - n_q + qg % n_q;
  const int64_t c = p / B;
  const int64_t j0 = (int64_t)chunk * kScoreBlocksPerCta;
  if (j0 > c) return;
  const int64_t j1 = min(j0 + kScoreBlocksPerCta, c + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint16_t* qrow = q_idx + qg * HI * D;
  for (int i = threadIdx.x; i < HI * D; i += 256) sq[i] = __uint_as_float((uint32_t)qrow[i] << 16);
  for (int i = threadIdx.x; i < HI; i += 256) sq[HI * D + i] = w_idx[qg * HI + i];
  __syncthreads();
  const float* bks = bk + (int64_t)seq * n_blk * D + lane * PER;
  for (int64_t j = j0 + warp; j < j1; j += 8) {
    float b[PER];
#pragma unroll
    for (int e = 0; e < PER; e += 2) {
      const float2 b2 = *reinterpret_cast<const float2*>(bks + j * D + e);
      b[e] = b2.x;
      b[e + 1] = b2.y;
    }
    float score = 0.f;
    for (int h = 0; h < HI; ++h) {
      const float* qh = sq + h * D + lane * PER;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) dot = fmaf(qh[e], b[e], dot);
      dot = warp_sum(dot);
      score = fmaf(sq[HI * D + h], fmaxf(dot, 0.f), score);
    }
    if (lane == 0) scores[qg * n_blk + j] = score;
  }
}

template <int NT>
__global__ void __launch_bounds__(NT) block_topm_kernel(const float* __restrict__ scores, int32_t* __restrict__ block_idx,
                                                        float* __restrict__ block_scores, int64_t n_q, int64_t n_kv,
                                                        int B, int64_t n_blk, int m, int keys_in_smem) {
  __shared__ SelectShared<NT> sm;
  extern __shared__ uint32_t skeys[];
  const int64_t qg = blockIdx.x;
  const int64_t p = n_kv - n_q + qg % n_q;
  const int64_t c = p / B;
  const int64_t n_vis = c + 1;
  const int64_t s_sel = min((int64_t)m, n_vis);
  int32_t* out = block_idx + qg * m;
  const float* sc = scores + qg * n_blk;

  if (s_sel == n_vis) {
    for (int r = threadIdx.x; r < m; r += NT) out[r] = r < n_vis ? r : -1;
  } else {
    // s_sel = m < c + 1: block 0, block c and the best m-2 of blocks 1..c-1.
    const int n = (int)(c - 1);
    const int K = (int)(s_sel - 2);
    if (threadIdx.x == 0) {
      out[0] = 0;
      out[s_sel - 1] = (int32_t)c;
    }
    for (int r = (int)s_sel + threadIdx.x; r < m; r += NT) out[r] = -1;
    if (K > 0) {
      if (keys_in_smem) {
        for (int i = threadIdx.x; i < n; i += NT) skeys[i] = score_key(sc[1 + i]);
        __syncthreads();
      }
      auto key = [&](int i) -> uint32_t { return keys_in_smem ? skeys[i] : score_key(sc[1 + i]); };
      const SelectResult r = radix_select<NT>(key, n, K, sm);
      emit_selected<NT>(key, n, r, sm, [&](int i, int rank) { out[1 + rank] = 1 + i; });
    }
  }
  if (block_scores) {
    __syncthreads();
    for (int r = threadIdx.x; r < m; r += NT) {
      const int j = out[r];
      block_scores[qg * m + r] = j >= 0 ? sc[j] : __int_as_float(0x7FC00000);
    }
  }
}

constexpr int kTopmThreads = 128;
constexpr int kTopmThreadsWide = 1024;
constexpr int64_t kTopmSmemKeys = 32768;

}  // namespace

cudaError_t launch_block_score(const Shape& s, const void* q_idx, const float* block_keys, float* scores,
                               cudaStream_t st) {
  const int chunks = (int)((s.n_blk + kScoreBlocksPerCta - 1) / kScoreBlocksPerCta);
  const int64_t grid = s.n_query * chunks;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  const uint16_t* qp = static_cast<const uint16_t*>(q_idx);
  if (s.HI > 0) {
    const int smem = (s.HI * s.d_idx + s.HI) * (int)sizeof(float);
    switch (s.d_idx) {
      case 64:
        block_score_mh_kernel<64><<<(unsigned)grid, 256, smem, st>>>(qp, s.w_idx, block_keys, scores, s.n_q, s.n_kv,
                                                                     s.B, s.n_blk, chunks, s.HI);
        break;
      case 128:
        block_score_mh_kernel<128><<<(unsigned)grid, 256, smem, st>>>(qp, s.w_idx, block_keys, scores, s.n_q, s.n_kv,
                                                                      s.B, s.n_blk, chunks, s.HI);
        break;
      case 256:
        block_score_mh_kernel<256><<<(unsigned)grid, 256, smem, st>>>(qp, s.w_idx, block_keys, scores, s.n_q, s.n_kv,
                                                                      s.B, s.n_blk, chunks, s.HI);
        break;
      default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
  }
  switch (s.d_idx) {
    case 64:
      block_score_kernel<64><<<(unsigned)grid, 256, 0, st>>>(qp, block_keys, scores, s.n_q, s.n_kv, s.B, s.n_blk, chunks);
      break;
    case 128:
      block_score_kernel<128><<<(unsigned)grid, 256, 0, st>>>(qp, block_keys, scores, s.n_q, s.n_kv, s.B, s.n_blk, chunks);
      break;
    case 256:
      block_score_kernel<256><<<(unsigned)grid, 256, 0, st>>>(qp, block_keys, scores, s.n_q, s.n_kv, s.B, s.n_blk, chunks);
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_block_topm(const Shape& s, const float* scores, int32_t* block_idx, float* block_scores,
                              cudaStream_t st) {
  const int in_smem = s.n_blk <= kTopmSmemKeys ? 1 : 0;
  const int smem = in_smem ? (int)(s.n_blk * 4) : 0;
  // Few queries (decode): wide CTAs over the long block lists.
  const bool wide = s.n_query < 2 * 148;
  auto kern = wide ? block_topm_kernel<kTopmThreadsWide> : block_topm_kernel<kTopmThreads>;
  const int nt = wide ? kTopmThreadsWide : kTopmThreads;
  const int stat = (int)(wide ? sizeof(SelectShared<kTopmThreadsWide>) : sizeof(SelectShared<kTopmThreads>));
  cudaError_t e = ensure_smem((const void*)kern, smem, stat);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)s.n_query, nt, smem, st>>>(scores, block_idx, block_scores, s.n_q, s.n_kv, s.B, s.n_blk, s.m,
                                              in_smem);
  return cudaGetLastError();
}

}  // namespace hisa
