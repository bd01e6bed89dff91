// CTA-wide top-K selection over 32-bit order-preserving keys.
//
// The selection order is "higher key first, then lower position": of the
// keys equal to the K-th largest key, the ones at the lowest positions are
// taken.  Keys of value 0 mark empty slots and are never taken as long as
// K <= (number of nonzero keys).
//
// Method: MSD radix selection, 8 bits per pass.  Each pass histograms the
// digit of the keys that still match the prefix chosen so far and locates the
// digit holding the K-th largest key with one warp-wide scan; it stops early
// when every key of that digit is taken.  A final pass in position order
// emits the taken positions (ascending) with ballot-based CTA scans.
#pragma once

#include "common.cuh"

namespace hisa {

template <int NT>
struct SelectShared {
  uint32_t hist[256];
  uint32_t warp_cnt[NT / 32][2];
  uint32_t bcast[3];
};

struct SelectResult {
  uint32_t prefix;  // key bits fixed by the selection (under `mask`)
  uint32_t mask;
  int take_eq;      // keys equal to prefix under mask: -1 = take all, else take the first take_eq
};

// All NT threads must call.  keys(i) returns the key at position i in [0, n).
// Requires 1 <= K <= number of nonzero keys.
template <int NT, class KeyFn>
__device__ SelectResult radix_select(KeyFn keys, int n, int K, SelectShared<NT>& sm) {
  uint32_t prefix = 0, mask = 0;
  uint32_t krem = (uint32_t)K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t k = keys(i);
      if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        c[b] = sm.hist[255 - 8 * lane - b];  // lane 0 holds the highest digits
        tot += c[b];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - tot;
      if (excl < krem && krem <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (acc + c[b] >= krem) {
            sm.bcast[0] = 255u - 8u * lane - b;
            sm.bcast[1] = acc;
            sm.bcast[2] = c[b];
            break;
          }
          acc += c[b];
        }
      }
    }
    __syncthreads();
    const uint32_t digit = sm.bcast[0], above = sm.bcast[1], at = sm.bcast[2];
    krem -= above;
    prefix |= digit << shift;
    mask |= 255u << shift;
    if (at == krem) return SelectResult{prefix, mask, -1};
  }
  return SelectResult{prefix, mask, (int)krem};
}

// "Take every nonzero key" as a SelectResult.
__device__ __forceinline__ SelectResult select_all_nonzero() { return SelectResult{0u, 0xFFFFFFFFu, 0}; }

// Emit the taken positions in ascending order: emit(i, rank) for each taken i.
// Returns the number emitted.  All NT threads must call.  Each warp owns one
// contiguous range of positions (read 32 at a time, so shared-memory reads stay
// conflict-free); a first sweep counts what each warp takes, one CTA scan turns
// the counts into offsets, and a second sweep emits.  Ties at the threshold are
// taken in position order across warps.
template <int NT, class KeyFn, class Emit>
__device__ int emit_selected(KeyFn keys, int n, SelectResult r, SelectShared<NT>& sm, Emit emit) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int span = ((n + NW - 1) / NW + 31) & ~31;  // positions per warp, a multiple of 32
  const int w0 = min(warp * span, n), w1 = min(w0 + span, n);
  auto classify = [&](int i, bool& gt, bool& eq) {
    const uint32_t km = (i < w1 ? keys(i) : 0u) & r.mask;
    gt = i < w1 && km > r.prefix;
    eq = i < w1 && km == r.prefix;
  };
  // sweep 1: how many keys above the threshold and at it does this warp hold?
  int n_gt = 0, n_eq = 0;
  for (int c0 = w0; c0 < w1; c0 += 32) {
    bool gt, eq;
    classify(c0 + lane, gt, eq);
    n_gt += __popc(__ballot_sync(0xFFFFFFFFu, gt));
    n_eq += __popc(__ballot_sync(0xFFFFFFFFu, eq));
  }
  if (lane == 0) {
    sm.warp_cnt[warp][0] = (uint32_t)n_gt;
    sm.warp_cnt[warp][1] = (uint32_t)n_eq;
  }
  __syncthreads();
  // offsets of this warp: keys taken and ties seen before it
  const int take_eq = r.take_eq < 0 ? 0x7FFFFFFF : r.take_eq;
  int eq_before = 0, taken_before = 0, total = 0, eqb = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int g = (int)sm.warp_cnt[w][0], e = (int)sm.warp_cnt[w][1];
    const int t = g + max(0, min(e, take_eq - eqb));
    if (w < warp) {
      taken_before += t;
      eq_before += e;
    }
    total += t;
    eqb += e;
  }
  // sweep 2: emit in order
  int rank = taken_before, eq_seen = eq_before;
  for (int c0 = w0; c0 < w1; c0 += 32) {
    const int i = c0 + lane;
    bool gt, eq;
    classify(i, gt, eq);
    const uint32_t be = __ballot_sync(0xFFFFFFFFu, eq);
    const bool sel = gt || (eq && eq_seen + __popc(be & below) < take_eq);
    const uint32_t bs = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel) emit(i, rank + __popc(bs & below));
    rank += __popc(bs);
    eq_seen += __popc(be);
  }
  __syncthreads();
  return total;
}

// Sum of one int per thread, CTA-wide (all threads get the result).  All NT threads must call.
template <int NT>
__device__ int cta_sum(int c, SelectShared<NT>& sm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
  if ((threadIdx.x & 31) == 0) sm.warp_cnt[threadIdx.x >> 5][0] = (uint32_t)c;
  __syncthreads();
  int tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) tot += (int)sm.warp_cnt[w][0];
  __syncthreads();
  return tot;
}

// Count of nonzero keys, CTA-wide (all threads get the result).
template <int NT, class KeyFn>
__device__ int count_nonzero(KeyFn keys, int n, SelectShared<NT>& sm) {
  int c = 0;
  for (int i = threadIdx.x; i < n; i += NT) c += keys(i) != 0u;
  return cta_sum<NT>(c, sm);
}

}  // namespace hisa
