// Steps 4-5: score the query against the tokens of its kept blocks and keep
// the top k.  "北大HISA稀疏注意力机制" section 1.2.2 items 1-2; QbitAI HISA
// article, "塊內精挑字符".  The flat indexer (every block is a slot) uses the
// same two kernels, which keeps the speed comparison like for like.
//
// token_score_kernel: one CTA per (query, run of slots).  A kept block is one
// contiguous B x d_idx tile of k_idx; 8 lanes share a token row (16-byte
// loads, each lane 8*d_idx/64 dimensions), several rows in flight per lane,
// fp32 FMA, 3-step shuffle reduction.  Each candidate's score is written as
// an order-preserving u32 key at [slot * B + offset] of the query's row;
// positions past the query or in unused slots get key 0 ("empty").
//
// token_score_mh_kernel: the same for the multi-head weighted score.
//
// token_select_staged_kernel: one CTA per query; the row of keys is staged in
// shared memory and a CTA radix selection in three wide digits takes the best
// min(k, candidates), emitted in ascending token order (token_select_kernel:
// the same for rows too long to stage, from global memory in 8-bit digits).
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace hisa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kMaxSlotsPerCta = 64;
constexpr int kSelectThreads = 256;
constexpr int kSelectThreadsWide = 1024;
constexpr int kSelectSmemKeys = 49152;  // 192 KiB of keys

template <int D>
__global__ void __launch_bounds__(kScoreThreads)
    token_score_kernel(const uint16_t* __restrict__ q_idx, const uint16_t* __restrict__ k_idx,
                       const int32_t* __restrict__ block_idx, int slots, uint32_t* __restrict__ keys,
                       int32_t* __restrict__ status, int64_t n_q, int64_t n_kv, int B, int spc, int chunks,
                       int64_t q0, int blk_lo) {
  constexpr int CPL = D / 64;  // 16-byte chunks per lane
  constexpr int U = 4;         // token rows in flight per lane group
  __shared__ int s_blk[kMaxSlotsPerCta];
  __shared__ int s_len[kMaxSlotsPerCta];

  const int64_t lq = blockIdx.x / chunks;
  const int chunk = blockIdx.x % chunks;
  const int64_t qg = q0 + lq;
  const int seq = (int)(qg / n_q);
  const int64_t p = n_kv - n_q + qg % n_q;
  const int64_t c = p / B;
  const int r0 = chunk * spc;
  const int nr = min(spc, slots - r0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // Which slots are usable: an entry is used if it lies in [0, c] and is
  // greater than every in-range entry before it (ascending, no repeats).
  for (int rr = warp; rr < nr; rr += kScoreThreads / 32) {
    const int r = r0 + rr;
    int blk;
    bool ok;
    if (block_idx) {
      const int32_t* row = block_idx + qg * slots;
      blk = row[r];
      int mx = -1;
      for (int t = lane; t < r; t += 32) {
        const int v = row[t];
        if (v >= 0 && v <= c) mx = max(mx, v);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      ok = blk >= 0 && blk <= c && blk > mx;
      if (!ok && blk != -1 && lane == 0 && status) atomicOr(status, kStatusBadIndex);
    } else {
      blk = blk_lo + r;
      ok = blk <= c;
    }
    if (lane == 0) {
      s_blk[rr] = ok ? blk : -1;
      s_len[rr] = ok ? visible_len(blk, B, p) : 0;
    }
  }

  // This thread's share of the query: chunks sub + 8u of the row.
  const int grp = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const unsigned gmask = 0xFFu << (lane & ~7);
  float qf[8 * CPL];
  const uint16_t* qrow = q_idx + qg * D;
#pragma unroll
  for (int u = 0; u < CPL; ++u) {
    const uint4 w = *reinterpret_cast<const uint4*>(qrow + (sub + 8 * u) * 8);
    qf[8 * u + 0] = bf16_lo(w.x); qf[8 * u + 1] = bf16_hi(w.x);
    qf[8 * u + 2] = bf16_lo(w.y); qf[8 * u + 3] = bf16_hi(w.y);
    qf[8 * u + 4] = bf16_lo(w.z); qf[8 * u + 5] = bf16_hi(w.z);
    qf[8 * u + 6] = bf16_lo(w.w); qf[8 * u + 7] = bf16_hi(w.w);
  }
  __syncthreads();

  constexpr int NG = kScoreThreads / 8;  // token rows per CTA step
  uint32_t* krow = keys + lq * (int64_t)slots * B;
  for (int rr = 0; rr < nr; ++rr) {
    const int blk = s_blk[rr], len = s_len[rr];
    const uint16_t* kb = k_idx + ((int64_t)seq * n_kv + (int64_t)(blk < 0 ? 0 : blk) * B) * D + sub * 8;
    uint32_t* dst = krow + (int64_t)(r0 + rr) * B;
    for (int o0 = grp; o0 < B; o0 += NG * U) {
      uint4 v[U][CPL];
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int o = o0 + j * NG;
#pragma unroll
        for (int u = 0; u < CPL; ++u)
          v[j][u] = o < len ? ld_nc_v4(kb + (int64_t)o * D + u * 64) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int o = o0 + j * NG;
        float dot = 0.f;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
          const float* qq = qf + 8 * u;
          dot = fmaf(qq[0], bf16_lo(v[j][u].x), dot); dot = fmaf(qq[1], bf16_hi(v[j][u].x), dot);
          dot = fmaf(qq[2], bf16_lo(v[j][u].y), dot); dot = fmaf(qq[3], bf16_hi(v[j][u].y), dot);
          dot = fmaf(qq[4], bf16_lo(v[j][u].z), dot); dot = fmaf(qq[5], bf16_hi(v[j][u].z), dot);
          dot = fmaf(qq[6], bf16_lo(v[j][u].w), dot); dot = fmaf(qq[7], bf16_hi(v[j][u].w), dot);
        }
        dot += __shfl_xor_sync(gmask, dot, 4);
        dot += __shfl_xor_sync(gmask, dot, 2);
        dot += __shfl_xor_sync(gmask, dot, 1);
        if (sub == 0 && o < B) dst[o] = o < len ? score_key(dot) : 0u;
      }
    }
  }
}

// The multi-head indexer score sum_j w_j * max(0, q_j . k_t) (n_idx_heads = HI >= 1).  Same
// work split and slot rules as token_score_kernel; the query's HI heads sit in shared memory as
// fp32 and every token row, read once, is scored against each head in turn.
template <int D>
__global__ void __launch_bounds__(kScoreThreads)
    token_score_mh_kernel(const uint16_t* __restrict__ q_idx, const float* __restrict__ w_idx,
                          const uint16_t* __restrict__ k_idx, const int32_t* __restrict__ block_idx, int slots,
                          uint32_t* __restrict__ keys, int32_t* __restrict__ status, int64_t n_q, int64_t n_kv, int B,
                          int spc, int chunks, int64_t q0, int HI, int blk_lo) {
  constexpr int CPL = D / 64;  // 16-byte chunks per lane
  __shared__ int s_blk[kMaxSlotsPerCta];
  __shared__ int s_len[kMaxSlotsPerCta];
  extern __shared__ float sq[];  // [HI][D] query heads, then [HI] weights

  const int64_t lq = blockIdx.x / chunks;
  const int chunk = blockIdx.x % chunks;
  const int64_t qg = q0 + lq;
  const int seq = (int)(qg / n_q);
  const int64_t p = n_kv - n_q + qg % n_q;
  const int64_t c = p / B;
  const int r0 = chunk * spc;
  const int nr = min(spc, slots - r0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  for (int rr = warp; rr < nr; rr += kScoreThreads / 32) {
    const int r = r0 + rr;
    int blk;
    bool ok;
    if (block_idx) {
      const int32_t* row = block_idx + qg * slots;
      blk = row[r];
      int mx = -1;
      for (int t = lane; t < r; t += 32) {
        const int v = row[t];
        if (v >= 0 && v <= c) mx = max(mx, v);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      ok = blk >= 0 && blk <= c && blk > mx;
      if (!ok && blk != -1 && lane == 0 && status) atomicOr(status, kStatusBadIndex);
    } else {
      blk = blk_lo + r;
      ok = blk <= c;
    }
    if (lane == 0) {
      s_blk[rr] = ok ? blk : -1;
      s_len[rr] = ok ? visible_len(blk, B, p) : 0;
    }
  }
  const uint16_t* qrow = q_idx + qg * HI * D;
  for (int i = threadIdx.x; i < HI * D; i += kScoreThreads) sq[i] = __uint_as_float((uint32_t)qrow[i] << 16);
  for (int i = threadIdx.x; i < HI; i += kScoreThreads) sq[HI * D + i] = w_idx[qg * HI + i];
  __syncthreads();

  const int grp = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const unsigned gmask = 0xFFu << (lane & ~7);
  constexpr int NG = kScoreThreads / 8;  // token rows per CTA step
  uint32_t* krow = keys + lq * (int64_t)slots * B;
  for (int rr = 0; rr < nr; ++rr) {
    const int blk = s_blk[rr], len = s_len[rr];
    const uint16_t* kb = k_idx + ((int64_t)seq * n_kv + (int64_t)(blk < 0 ? 0 : blk) * B) * D + sub * 8;
    uint32_t* dst = krow + (int64_t)(r0 + rr) * B;
    for (int o = grp; o < B; o += NG) {  // warp-uniform trip count: rows o of a lane group
      float kv[8 * CPL];
#pragma unroll
      for (int u = 0; u < CPL; ++u) {
        const uint4 w = o < len ? ld_nc_v4(kb + (int64_t)o * D + u * 64) : make_uint4(0, 0, 0, 0);
        kv[8 * u + 0] = bf16_lo(w.x); kv[8 * u + 1] = bf16_hi(w.x);
        kv[8 * u + 2] = bf16_lo(w.y); kv[8 * u + 3] = bf16_hi(w.y);
        kv[8 * u + 4] = bf16_lo(w.z); kv[8 * u + 5] = bf16_hi(w.z);
        kv[8 * u + 6] = bf16_lo(w.w); kv[8 * u + 7] = bf16_hi(w.w);
      }
      float score = 0.f;
      for (int h = 0; h < HI; ++h) {
        float dot = 0.f;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
          const float* qq = sq + h * D + (sub + 8 * u) * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) dot = fmaf(qq[e], kv[8 * u + e], dot);
        }
        dot += __shfl_xor_sync(gmask, dot, 4);
        dot += __shfl_xor_sync(gmask, dot, 2);
        dot += __shfl_xor_sync(gmask, dot, 1);
        score = fmaf(sq[HI * D + h], fmaxf(dot, 0.f), score);
      }
      if (sub == 0) dst[o] = o < len ? score_key(score) : 0u;
    }
  }
}

// One CTA per query; the row of keys, read from global memory, is staged in
// shared memory and the first selection digit counted on the way in (three
// sweeps of the row in all: staging, the candidate sweep and the emit sweep).
// V = 4: the row length is a multiple of four (16-byte staging).  SC: scores are written too.
template <int NT, int V, bool SC>
__global__ void __launch_bounds__(NT)
    token_select_staged_kernel(const uint32_t* __restrict__ keys, const int32_t* __restrict__ block_idx, int slots,
                               int32_t* __restrict__ token_idx, float* __restrict__ token_scores, int log2B, int k,
                               int64_t q0, int blk_lo) {
  __shared__ StagedSelectShared<NT> sm;
  extern __shared__ __align__(16) uint32_t dsm[];
  const int B = 1 << log2B;
  const int64_t lq = blockIdx.x;
  const int64_t qg = q0 + lq;
  const int n = slots * B;
  const uint32_t* row = keys + lq * (int64_t)n;
  uint32_t* skeys = dsm;
  int32_t* sblk = reinterpret_cast<int32_t*>(dsm + n);

  for (int r = threadIdx.x; r < slots; r += NT) sblk[r] = block_idx ? block_idx[qg * slots + r] : blk_lo + r;
  for (int i = threadIdx.x; i < kWideBins / 4; i += NT)
    reinterpret_cast<uint4*>(sm.u.hist)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if constexpr (V == 4) {
    const uint4* src = reinterpret_cast<const uint4*>(row);
    uint4* dst = reinterpret_cast<uint4*>(skeys);
#pragma unroll 4
    for (int i = threadIdx.x; i < n / 4; i += NT) {
      const uint4 v = src[i];
      dst[i] = v;
      counts_first_digit(sm.u.hist, v.x);
      counts_first_digit(sm.u.hist, v.y);
      counts_first_digit(sm.u.hist, v.z);
      counts_first_digit(sm.u.hist, v.w);
    }
  } else {
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t v = row[i];
      skeys[i] = v;
      counts_first_digit(sm.u.hist, v);
    }
  }
  __syncthreads();
  int32_t* out = token_idx + qg * k;
  float* osc = token_scores ? token_scores + qg * k : nullptr;
  const int K = staged_select<NT>(
      skeys, n, k, sm, [&](int i, uint32_t) { return sblk[i >> log2B] * B + (i & (B - 1)); },
      [&](int rank, int32_t id, uint32_t key) {
        out[rank] = id;
        if constexpr (SC) osc[rank] = key_score(key);
      });
  for (int r = K + threadIdx.x; r < k; r += NT) {
    out[r] = -1;
    if (osc) osc[r] = __int_as_float(0x7FC00000);
  }
}

// The flat indexer's streaming top-k, one window after the first: row r stages its running list
// (k entries, ids run_ids[r], tokens of the earlier windows, ascending) ahead of the window's n
// keys (tokens blk_lo * B ..), so the selection's lowest-position rule is the lowest-token rule,
// and keeps the best k of both.
template <int NT>
__global__ void __launch_bounds__(NT)
    flat_select_kernel(const uint32_t* __restrict__ keys, int n, const int32_t* __restrict__ run_ids,
                       const float* __restrict__ run_sc, int k, int64_t tok0, int32_t* __restrict__ out_ids,
                       float* __restrict__ out_sc) {
  __shared__ StagedSelectShared<NT> sm;
  extern __shared__ __align__(16) uint32_t dsm[];
  const int64_t row = blockIdx.x;
  const int32_t* ri = run_ids + row * k;
  const float* rs = run_sc + row * k;
  const uint32_t* wk = keys + row * (int64_t)n;
  uint32_t* skeys = dsm;
  for (int i = threadIdx.x; i < kWideBins / 4; i += NT)
    reinterpret_cast<uint4*>(sm.u.hist)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  for (int i = threadIdx.x; i < k; i += NT) {
    const uint32_t key = ri[i] >= 0 ? score_key(rs[i]) : 0u;
    skeys[i] = key;
    counts_first_digit(sm.u.hist, key);
  }
  if ((n & 3) == 0 && (k & 3) == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(wk);
    uint4* dst = reinterpret_cast<uint4*>(skeys + k);
    for (int i = threadIdx.x; i < n / 4; i += NT) {
      const uint4 v = src[i];
      dst[i] = v;
      counts_first_digit(sm.u.hist, v.x);
      counts_first_digit(sm.u.hist, v.y);
      counts_first_digit(sm.u.hist, v.z);
      counts_first_digit(sm.u.hist, v.w);
    }
  } else {
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t v = wk[i];
      skeys[k + i] = v;
      counts_first_digit(sm.u.hist, v);
    }
  }
  __syncthreads();
  int32_t* oi = out_ids + row * k;
  float* os = out_sc ? out_sc + row * k : nullptr;
  const int K = staged_select<NT>(
      skeys, n + k, k, sm, [&](int i, uint32_t) { return i < k ? ri[i] : (int32_t)(tok0 + (i - k)); },
      [&](int rank, int32_t id, uint32_t key) {
        oi[rank] = id;
        if (os) os[rank] = key_score(key);
      });
  for (int r = K + threadIdx.x; r < k; r += NT) {
    oi[r] = -1;
    if (os) os[r] = __int_as_float(0x7FC00000);
  }
}

// Rows too long for shared memory: the selection reads the keys from global memory on every pass.
template <int NT>
__global__ void __launch_bounds__(NT)
    token_select_kernel(const uint32_t* __restrict__ keys, const int32_t* __restrict__ block_idx, int slots,
                        int32_t* __restrict__ token_idx, float* __restrict__ token_scores, int log2B, int k,
                        int64_t q0, int blk_lo) {
  __shared__ SelectShared<NT> sm;
  extern __shared__ __align__(16) uint32_t dsm[];
  const int B = 1 << log2B;
  const int64_t lq = blockIdx.x;
  const int64_t qg = q0 + lq;
  const int n = slots * B;
  const uint32_t* row = keys + lq * (int64_t)n;
  int32_t* sblk = reinterpret_cast<int32_t*>(dsm);

  for (int r = threadIdx.x; r < slots; r += NT) sblk[r] = block_idx ? block_idx[qg * slots + r] : blk_lo + r;
  __syncthreads();
  auto key = [&](int i) -> uint32_t { return row[i]; };
  const int nv = count_nonzero<NT>(key, n, sm);
  const int K = min(k, nv);
  int32_t* out = token_idx + qg * k;
  float* osc = token_scores ? token_scores + qg * k : nullptr;
  if (K > 0) {
    const SelectResult r = (K == nv) ? select_all_nonzero() : radix_select<NT>(key, n, K, sm);
    emit_selected<NT>(key, n, r, sm, [&](int i, int rank) {
      const int slot = i >> log2B;
      out[rank] = sblk[slot] * B + (i & (B - 1));
      if (osc) osc[rank] = key_score(key(i));
    });
  }
  for (int r = K + threadIdx.x; r < k; r += NT) {
    out[r] = -1;
    if (osc) osc[r] = __int_as_float(0x7FC00000);
  }
}

}  // namespace

cudaError_t launch_token_score(const Shape& s, const void* q_idx, const void* k_idx, const int32_t* block_idx,
                               int slots, uint32_t* keys, int32_t* status, int64_t q0, int64_t nq, cudaStream_t st,
                               int blk_lo) {
  if (nq <= 0) return cudaSuccess;
  // Many queries per sequence: tensor-core tiles of 128 queries x one key block.
  if (token_score_tc_eligible(s, slots)) {
    const cudaError_t e = launch_token_score_tc(s, q_idx, k_idx, block_idx, slots, keys, status, q0, nq, st, blk_lo);
    if (e != cudaErrorNotSupported) return e;
  }
  // Up to 1024 tokens per CTA; with few queries (decode) fewer, so that the grid has about four
  // CTAs per SM to hide the gathers' latency.
  int spc = 1024 / s.B;
  const int64_t want = (nq * slots + 4 * 148 - 1) / (4 * 148);  // slots per CTA for ~4 waves
  if (want < spc) spc = (int)want;
  spc = spc < 1 ? 1 : (spc > kMaxSlotsPerCta ? kMaxSlotsPerCta : spc);
  if (spc > slots) spc = slots;
  const int chunks = (slots + spc - 1) / spc;
  const int64_t grid = nq * chunks;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  const uint16_t* qp = static_cast<const uint16_t*>(q_idx);
  const uint16_t* kp = static_cast<const uint16_t*>(k_idx);
  if (s.HI > 0) {
    const int smem = (s.HI * s.d_idx + s.HI) * (int)sizeof(float);
    switch (s.d_idx) {
      case 64:
        token_score_mh_kernel<64><<<(unsigned)grid, kScoreThreads, smem, st>>>(
            qp, s.w_idx, kp, block_idx, slots, keys, status, s.n_q, s.n_kv, s.B, spc, chunks, q0, s.HI, blk_lo);
        break;
      case 128:
        token_score_mh_kernel<128><<<(unsigned)grid, kScoreThreads, smem, st>>>(
            qp, s.w_idx, kp, block_idx, slots, keys, status, s.n_q, s.n_kv, s.B, spc, chunks, q0, s.HI, blk_lo);
        break;
      case 256:
        token_score_mh_kernel<256><<<(unsigned)grid, kScoreThreads, smem, st>>>(
            qp, s.w_idx, kp, block_idx, slots, keys, status, s.n_q, s.n_kv, s.B, spc, chunks, q0, s.HI, blk_lo);
        break;
      default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
  }
  switch (s.d_idx) {
    case 64:
      token_score_kernel<64><<<(unsigned)grid, kScoreThreads, 0, st>>>(qp, kp, block_idx, slots, keys, status, s.n_q,
                                                                       s.n_kv, s.B, spc, chunks, q0, blk_lo);
      break;
    case 128:
      token_score_kernel<128><<<(unsigned)grid, kScoreThreads, 0, st>>>(qp, kp, block_idx, slots, keys, status, s.n_q,
                                                                        s.n_kv, s.B, spc, chunks, q0, blk_lo);
      break;
    case 256:
      token_score_kernel<256><<<(unsigned)grid, kScoreThreads, 0, st>>>(qp, kp, block_idx, slots, keys, status, s.n_q,
                                                                        s.n_kv, s.B, spc, chunks, q0, blk_lo);
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_token_select(const Shape& s, const uint32_t* keys, const int32_t* block_idx, int slots,
                                int32_t* token_idx, float* token_scores, int64_t q0, int64_t nq, cudaStream_t st,
                                int blk_lo) {
  if (nq <= 0) return cudaSuccess;
  const int64_t n = (int64_t)slots * s.B;
  int log2B = 0;
  while ((1 << log2B) < s.B) ++log2B;
  // Few queries (decode): one wide CTA per query keeps the selection from being latency-bound.
  const bool wide = nq < 2 * 148;
  const int nt = wide ? kSelectThreadsWide : kSelectThreads;
  const size_t stat = wide ? sizeof(StagedSelectShared<kSelectThreadsWide>) : sizeof(StagedSelectShared<kSelectThreads>);
  const int64_t staged = n * 4 + (int64_t)slots * 4;
  if (n <= kSelectSmemKeys && staged + (int64_t)stat <= 227 * 1024) {
    const bool v4 = (n & 3) == 0, sc = token_scores != nullptr;
#define HISA_SEL(NT) \
  (v4 ? (sc ? token_select_staged_kernel<NT, 4, true> : token_select_staged_kernel<NT, 4, false>) \
      : (sc ? token_select_staged_kernel<NT, 1, true> : token_select_staged_kernel<NT, 1, false>))
    auto kern = wide ? HISA_SEL(kSelectThreadsWide) : HISA_SEL(kSelectThreads);
#undef HISA_SEL
    cudaError_t e = ensure_smem((const void*)kern, (int)staged, (int)stat);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)nq, nt, (int)staged, st>>>(keys, block_idx, slots, token_idx, token_scores, log2B, s.k, q0,
                                                 blk_lo);
    return cudaGetLastError();
  }
  const int smem = slots * 4;
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  auto kern = wide ? token_select_kernel<kSelectThreadsWide> : token_select_kernel<kSelectThreads>;
  const int gstat = (int)(wide ? sizeof(SelectShared<kSelectThreadsWide>) : sizeof(SelectShared<kSelectThreads>));
  cudaError_t e = ensure_smem((const void*)kern, smem, gstat);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)nq, nt, smem, st>>>(keys, block_idx, slots, token_idx, token_scores, log2B, s.k, q0, blk_lo);
  return cudaGetLastError();
}

cudaError_t launch_flat_select(const uint32_t* keys, int n, const int32_t* run_ids, const float* run_scores, int k,
                               int64_t tok0, int64_t rows, int32_t* out_ids, float* out_scores, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const int64_t smem = ((int64_t)n + k) * 4;
  const int stat = (int)sizeof(StagedSelectShared<kSelectThreads>);
  if (k < 1 || n < 1 || (int64_t)n + k >= 65536 || smem + stat > 227 * 1024 || rows > 0x7FFFFFFFLL)
    return cudaErrorInvalidValue;
  auto kern = flat_select_kernel<kSelectThreads>;
  cudaError_t e = ensure_smem((const void*)kern, (int)smem, stat);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)rows, kSelectThreads, (int)smem, st>>>(keys, n, run_ids, run_scores, k, tok0, out_ids,
                                                           out_scores);
  return cudaGetLastError();
}

}  // namespace hisa
