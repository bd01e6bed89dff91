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

// Positions [w0, w1) of warp `warp` in the emit order: contiguous ranges, a
// multiple of 32 positions each (so shared-memory reads stay conflict-free).
template <int NT>
__device__ __forceinline__ void warp_span(int n, int warp, int& w0, int& w1) {
  constexpr int NW = NT / 32;
  const int span = ((n + NW - 1) / NW + 31) & ~31;
  w0 = min(warp * span, n);
  w1 = min(w0 + span, n);
}

// Second half of emit_selected: sm.warp_cnt[w] holds, for every warp w, the
// number of its keys above the threshold and at it (under r.mask).  Emits the
// taken positions in ascending order and returns the number emitted.  All NT
// threads must call.
template <int NT, class KeyFn, class Emit>
__device__ int emit_counted(KeyFn keys, int n, SelectResult r, SelectShared<NT>& sm, Emit emit) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t below = (1u << lane) - 1u;
  int w0, w1;
  warp_span<NT>(n, warp, w0, w1);
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
  int rank = taken_before, eq_seen = eq_before;
  for (int c0 = w0; c0 < w1; c0 += 32) {
    const int i = c0 + lane;
    const uint32_t km = (i < w1 ? keys(i) : 0u) & r.mask;
    const bool gt = i < w1 && km > r.prefix;
    const bool eq = i < w1 && km == r.prefix;
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

// Emit the taken positions in ascending order: emit(i, rank) for each taken i.
// Returns the number emitted.  All NT threads must call.  Each warp owns one
// contiguous range of positions; a first sweep counts what each warp takes,
// one CTA scan turns the counts into offsets, and a second sweep emits.  Ties
// at the threshold are taken in position order across warps.
template <int NT, class KeyFn, class Emit>
__device__ int emit_selected(KeyFn keys, int n, SelectResult r, SelectShared<NT>& sm, Emit emit) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int w0, w1;
  warp_span<NT>(n, warp, w0, w1);
  int n_gt = 0, n_eq = 0;
  for (int c0 = w0; c0 < w1; c0 += 32) {
    const int i = c0 + lane;
    const uint32_t km = (i < w1 ? keys(i) : 0u) & r.mask;
    n_gt += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && km > r.prefix));
    n_eq += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && km == r.prefix));
  }
  if (lane == 0) {
    sm.warp_cnt[warp][0] = (uint32_t)n_gt;
    sm.warp_cnt[warp][1] = (uint32_t)n_eq;
  }
  __syncthreads();
  return emit_counted<NT>(keys, n, r, sm, emit);
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


// ---------------------------------------------------------------------------
// Selection of a row staged in shared memory.
//
// Same order and result as radix_select + emit_selected, with two exceptions
// of definition: keys below 2^21 (the empty key 0, and the order-preserving
// images of negative NaNs with large payloads, which no arithmetic produces)
// are never taken, and the number of keys at or above 2^21 replaces the
// count of nonzero keys.
//
// The first digit is key bits 31-21 (2048 counters); the caller counts it
// while it stages the row (one atomic per key).  One sweep then counts, per
// warp, the keys above the threshold digit and gathers the keys of that digit
// (the candidates, usually a few percent of the row) into per-warp segments
// of the counters' space; the remaining 21 bits are resolved over the
// candidates alone in 8-bit digits; one more sweep hands out the taken
// positions in order.  Both sweeps work on groups of 32 consecutive positions
// with one ballot per group, and skip the candidate and tie work of groups
// that hold no key of the threshold (a warp-uniform test).  A warp whose
// candidates overflow its segment sends the later digits over the whole row
// (same result, slower).
// ---------------------------------------------------------------------------

constexpr int kWideBins = 2048;

template <int NT>
struct StagedSelectShared {
  static constexpr int NW = NT / 32;
  static constexpr int SEG = kWideBins / NW;  // candidate slots per warp
  union {
    uint32_t hist[kWideBins];  // first-digit counters
    uint32_t cand[kWideBins];  // then the candidates, SEG per warp
  } u;
  uint32_t seg_n[NW];  // candidates found by each warp (may exceed SEG)
  uint32_t gt_n[NW];   // keys above the threshold digit, per warp
  uint32_t bc[3];
  SelectShared<NT> sel;
};

// Staging-time count of key k into the first-digit counters.
__device__ __forceinline__ void counts_first_digit(uint32_t* hist, uint32_t k) { atomicAdd(&hist[k >> 21], 1u); }

// The digit holding the krem-th largest counted key of sm.u.hist, the count
// above it and the count in it.  Warp 0 scans (64 counters a lane, in eight
// groups of eight); all NT threads call and return synchronised.
template <int NT>
__device__ void wide_scan(StagedSelectShared<NT>& sm, uint32_t krem, uint32_t& digit, uint32_t& above,
                          uint32_t& at) {
  static_assert(kWideBins == 64 * 32, "64 counters per lane");
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int top = kWideBins - 64 * lane;  // the lane holds digits [top - 64, top), highest first
    uint32_t gs[8], tot = 0;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const uint4* h = reinterpret_cast<const uint4*>(&sm.u.hist[top - 8 * (g + 1)]);
      const uint4 x = h[0], y = h[1];
      gs[g] = x.x + x.y + x.z + x.w + y.x + y.y + y.z + y.w;
      tot += gs[g];
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
      int g = 0;
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) {
        if (acc + gs[gg] >= krem) {
          g = gg;
          break;
        }
        acc += gs[gg];
      }
      for (int d = top - 8 * g - 1; d >= top - 8 * (g + 1); --d) {
        const uint32_t c = sm.u.hist[d];
        if (acc + c >= krem) {
          sm.bc[0] = (uint32_t)d;
          sm.bc[1] = acc;
          sm.bc[2] = c;
          break;
        }
        acc += c;
      }
    }
  }
  __syncthreads();
  digit = sm.bc[0];
  above = sm.bc[1];
  at = sm.bc[2];
}

// One 8-bit digit (k >> shift) & 255 of the keys the threads visit through
// visit(fn) (fn(key) per key; keys not matching prefix under mask are
// skipped): counts, finds the digit of the krem-th largest and narrows
// prefix, mask, krem and take_eq.  All NT threads call; returns synchronised.
template <int NT, class Visit>
__device__ void narrow_digit(Visit visit, int shift, uint32_t& prefix, uint32_t& mask, uint32_t& krem, int& take_eq,
                             SelectShared<NT>& sm) {
  for (int i = threadIdx.x; i < 256; i += NT) sm.hist[i] = 0;
  __syncthreads();
  const uint32_t pf = prefix, mk = mask;
  visit([&](uint32_t k) {
    if ((k & mk) == pf) atomicAdd(&sm.hist[(k >> shift) & 255u], 1u);
  });
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t c[8], tot = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      c[b] = sm.hist[255 - 8 * lane - b];
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
  take_eq = at == krem ? -1 : (int)krem;
}

// Selects the best min(k, keys >= 2^21) keys of skeys[0, n) (n < 65536) and
// hands them out in ascending position order: store(rank, ident(position, key),
// key) -- ident runs on every lane of a group whose position lies in the row,
// store only on the taken ones (a lone guarded store, so that no lane diverges
// around a lookup).  On
// entry sm.u.hist holds the first-digit counts of all n keys and the threads
// are synchronised.  All NT threads call; returns the number taken.
template <int NT, class Ident, class Store>
__device__ int staged_select(const uint32_t* skeys, int n, int k, StagedSelectShared<NT>& sm, Ident ident,
                             Store store) {
  using SS = StagedSelectShared<NT>;
  constexpr int NW = SS::NW, SEG = SS::SEG;
  constexpr int U = 4;  // groups of 32 positions per step
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int nv = n - (int)sm.u.hist[0];
  const int K = min(k, nv);
  if (K <= 0) return 0;

  uint32_t prefix = 0u, mask = 0xFFE00000u, krem = (uint32_t)K;
  int take_eq = 0;  // K = nv: every key from 2^21 up ("above" prefix 0), none of digit 0
  if (K < nv) {
    uint32_t digit, above, at;
    wide_scan<NT>(sm, krem, digit, above, at);  // digit >= 1: digits 1.. hold nv >= K keys
    krem -= above;
    prefix = digit << 21;
    take_eq = at == krem ? -1 : (int)krem;
  }
  const bool collect = take_eq > 0;  // the threshold digit is split: gather its keys

  // sweep: keys above the threshold digit, and the candidates, per warp
  int w0, w1;
  warp_span<NT>(n, warp, w0, w1);
  uint32_t* seg = sm.u.cand + warp * SEG;
  int ng = 0, nc = 0;
  auto sweep = [&](int c0, bool full) {
    uint32_t kk[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int i = c0 + 32 * j + lane;
      kk[j] = (full || i < w1) ? skeys[i] : 0u;
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const uint32_t km = kk[j] & mask;
      ng += km > prefix;
      if (collect) {
        const uint32_t b = __ballot_sync(0xFFFFFFFFu, km == prefix);
        if (b) {
          const int o = nc + __popc(b & below);
          if (km == prefix && o < SEG) seg[o] = kk[j];
          nc += __popc(b);
        }
      } else {
        nc += km == prefix;
      }
    }
  };
  int c0 = w0;
  for (; c0 + 32 * U <= w1; c0 += 32 * U) sweep(c0, true);  // whole steps: no bound tests
  if (c0 < w1) sweep(c0, false);
  ng = __reduce_add_sync(0xFFFFFFFFu, ng);
  if (!collect) nc = __reduce_add_sync(0xFFFFFFFFu, nc);
  if (lane == 0) {
    sm.gt_n[warp] = (uint32_t)ng;
    sm.seg_n[warp] = (uint32_t)nc;
  }
  __syncthreads();

  if (collect) {
    bool overflow = false;
#pragma unroll 1
    for (int w = 0; w < NW; ++w) overflow |= sm.seg_n[w] > (uint32_t)SEG;
    const int cn = min((int)sm.seg_n[warp], SEG);
    auto visit_cand = [&](auto fn) {
      for (int j = lane; j < cn; j += 32) fn(seg[j]);
    };
    auto visit_row = [&](auto fn) {
      for (int i = threadIdx.x; i < n; i += NT) fn(skeys[i]);
    };
#pragma unroll 1
    for (int shift = 13; take_eq >= 0 && shift >= 0; shift = shift > 5 ? 5 : (shift == 5 ? 0 : -1)) {
      if (overflow)
        narrow_digit<NT>(visit_row, shift, prefix, mask, krem, take_eq, sm.sel);
      else
        narrow_digit<NT>(visit_cand, shift, prefix, mask, krem, take_eq, sm.sel);
    }
    // per-warp counts under the final threshold
    int g = 0, e = 0;
    if (!overflow) {
      for (int j = lane; j < cn; j += 32) {
        const uint32_t km = seg[j] & mask;
        g += km > prefix;
        e += km == prefix;
      }
    } else {
      for (int i = w0 + lane; i < w1; i += 32) {
        const uint32_t km = skeys[i] & mask;
        g += km > prefix;
        e += km == prefix;
      }
    }
    g = __reduce_add_sync(0xFFFFFFFFu, g);
    e = __reduce_add_sync(0xFFFFFFFFu, e);
    if (!overflow) g += (int)sm.gt_n[warp];  // the keys above the threshold digit
    if (lane == 0) {
      sm.sel.warp_cnt[warp][0] = (uint32_t)g;
      sm.sel.warp_cnt[warp][1] = (uint32_t)e;
    }
  } else if (lane == 0) {
    sm.sel.warp_cnt[warp][0] = (uint32_t)ng;
    sm.sel.warp_cnt[warp][1] = (uint32_t)nc;
  }
  __syncthreads();

  // offsets of this warp: keys taken and ties seen before it
  const int teq = take_eq < 0 ? 0x7FFFFFFF : take_eq;
  int eq_before = 0, taken_before = 0, eqb = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int gw = (int)sm.sel.warp_cnt[w][0], ew = (int)sm.sel.warp_cnt[w][1];
    if (w < warp) {
      taken_before += gw + max(0, min(ew, teq - eqb));
      eq_before += ew;
    }
    eqb += ew;
  }
  int rank = taken_before, eq_seen = eq_before;
  auto emit = [&](int c0, bool full) {
    uint32_t kk[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int i = c0 + 32 * j + lane;
      kk[j] = (full || i < w1) ? skeys[i] : 0u;
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int i = c0 + 32 * j + lane;
      const uint32_t km = kk[j] & mask;
      const bool in = full || i < w1;
      bool sel = km > prefix;
      const uint32_t be = __ballot_sync(0xFFFFFFFFu, km == prefix && in);
      if (be) {  // keys at the threshold in this group
        const bool eq = km == prefix && in;
        sel = sel || (eq && eq_seen + __popc(be & below) < teq);
        eq_seen += __popc(be);
      }
      const uint32_t bs = __ballot_sync(0xFFFFFFFFu, sel);
      int32_t id = 0;
      if (in) id = ident(i, kk[j]);  // positions past the row have no identity (nor a slot)
      const int o = rank + __popc(bs & below);
      if (sel) store(o, id, kk[j]);
      rank += __popc(bs);
    }
  };
  for (c0 = w0; c0 + 32 * U <= w1; c0 += 32 * U) emit(c0, true);
  if (c0 < w1) emit(c0, false);
  __syncthreads();
  return K;
}

}  // namespace hisa
