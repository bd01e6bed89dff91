// Step 6 on the 5th-generation tensor cores, head dimension 128.
// QbitAI HISA article, "HISA的關鍵優勢在於": the indexer's output keeps the
// original format and the attention after it is the usual one, softmax of the
// scaled scores times V, here over the selected tokens of each query.
//
// The selected token list is shared by all heads of a query, so the heads of
// one KV group (n_heads / n_kv_heads of them, GQA/MQA; one with MHA) read the
// very same gathered K and V rows.  A work item is (KV head, group of up to GS
// of its heads, query, split); persistent CTAs (one per SM) walk the items
// with the KV heads outermost, so the CTAs running at the same time gather
// from one head's K and V, which the L2 then serves to many queries.  The
// list is compacted into tiles of 128 valid entries (-1 padding and
// out-of-range entries dropped, the latter flagged in bit 0 of the status
// word).  Per tile:
//   * 4 producer warps copy the 128 K rows and 128 V rows (and the item's q
//     rows) with 16-byte cp.async straight into the 128-byte-swizzled layout
//     of the MMA operands; the copies complete on the stage's mbarrier
//     (3 stages in flight).  Warp 0 compacts the list one tile ahead, its
//     list window read one more tile ahead;
//   * one thread issues S = K_tile x [q_1 .. q_GS]ᵀ (tcgen05.mma, M = 128
//     tokens, N = 16, fp32 in TMEM);
//   * 4 softmax warps, one thread per token (TMEM lane = token), read the GS
//     scores of their token, reduce the per-head tile maxima across the CTA,
//     raise each head's running max lazily (the TMEM accumulator is rescaled
//     only when a weight would exceed 2^8), and write the weights as bf16
//     pairs hi + lo (~16 significant bits) into the B operand of the output
//     MMA;
//   * a second thread issues Oᵀ += V_tileᵀ x [p_hi; p_lo]ᵀ (M = 128
//     dimensions, N = 2 GS, K = 128 tokens; V is read MN-major straight from
//     its gathered rows).
// At an item's end one softmax thread per output dimension reads Oᵀ back and
// writes O and the LSE of every head of the item, or the partial
// (max, sum, O) states of its split.  The scores of tile t+1 are computed
// while the softmax of tile t runs.  Every wait is bounded (1 s): a timeout
// sets status bit 1 and the CTA stops.
#include <atomic>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

#ifndef HISA_ATTN_TC
#define HISA_ATTN_TC 1
#endif
// Smallest number of heads per KV head routed to this kernel.
#ifndef HISA_ATTN_TC_MIN_GROUP
#define HISA_ATTN_TC_MIN_GROUP 2
#endif

namespace hisa {
namespace {

using namespace tc;

constexpr int kD = 128;        // head dimension of this kernel
constexpr int kTok = 128;      // list entries per tile
constexpr int kNS = 3;         // K/V stages
constexpr int kProd = 4;       // producer warps 0-3; softmax warps 4-7 (TMEM lane quarter = warp % 4)
constexpr int kWarpQK = 8;     // issues the score MMAs, owns the TMEM allocation
constexpr int kWarpPV = 9;     // issues the output MMAs
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 64;

template <int GS>
struct Cfg {
  static constexpr int LOG = GS == 1 ? 0 : GS == 2 ? 1 : GS == 4 ? 2 : GS == 8 ? 3 : 4;
  static constexpr int NQ = 16;                         // N of the score MMA (q rows, GS <= 16 used)
  static constexpr int NO = 2 * GS < 16 ? 16 : 2 * GS;  // N of the output MMA: GS hi rows, then GS lo rows
  static constexpr int HALF = kTok * 128;               // 64 dimensions of the tile's rows: 16 KB
  static constexpr int KV = 2 * HALF;
  static constexpr int QOP = 2 * NQ * 128;              // q operand (two 64-element K atoms)
  static constexpr int POP = 2 * NO * 128;              // weight operand (two 64-token K atoms)
  static constexpr int K_OFF = 0, V_OFF = KV, Q_OFF = 2 * KV;
  static constexpr int STAGE = 2 * KV + QOP;
  static constexpr int P_OFF = kNS * STAGE;
  static constexpr int IDX_OFF = P_OFF + 2 * POP;           // 3 x kTok token ids
  static constexpr int PINFO_OFF = IDX_OFF + 3 * kTok * 4;  // 3 x (count, last)
  static constexpr int META_OFF = PINFO_OFF + 3 * 8;        // kNS x (count, first | last << 1)
  static constexpr int RED_OFF = META_OFF + kNS * 8;        // [2][4][16] maxima, [4][16] sums, [4] errors
  static constexpr int RED_FLOATS = 2 * 4 * 16 + 4 * 16 + 4;
  static constexpr int BAR_OFF = (RED_OFF + RED_FLOATS * 4 + 7) & ~7;
  static constexpr int NBAR = 2 * kNS + 8;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;
  static constexpr uint32_t COL_O = 32;  // TMEM columns: S0 0-15, S1 16-31, O 32 .. 32 + NO - 1
  static_assert(GS == (1 << LOG) && GS <= 16, "heads per item: a power of two up to 16");
  static_assert(STAGE % 1024 == 0 && P_OFF % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(COL_O + NO <= kTmemCols, "TMEM columns");
};

// mbarrier indices
constexpr int B_FULL = 0, B_EMPTY = kNS, B_SFULL = 2 * kNS, B_PREADY = 2 * kNS + 2, B_PFREE = 2 * kNS + 4,
              B_DRAIN = 2 * kNS + 6;  // [2]: one per MMA thread

struct Item {
  int g, sub;
  int64_t qg;
  int split;
};

__device__ __forceinline__ Item item_of(int64_t it, int n_sub, int64_t n_query, int splits) {
  const int64_t per_sub = n_query * splits;
  const int64_t per_g = per_sub * n_sub;
  Item r;
  r.g = (int)(it / per_g);
  int64_t rem = it - (int64_t)r.g * per_g;
  r.sub = (int)(rem / per_sub);
  rem -= (int64_t)r.sub * per_sub;
  r.qg = rem / splits;
  r.split = (int)(rem - r.qg * splits);
  return r;
}

__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier of the producer warps that also ANDs a flag over them.
__device__ __forceinline__ int producer_sync_and(int flag) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.b32 p, %1, 0;\n bar.red.and.pred q, 2, 128, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(flag)
      : "memory");
  return (int)r;
}

__device__ __forceinline__ void cp_async16_all(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Arrive on `bar` once every cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Column reduction over a warp of GS values per lane.  Returns, in every lane,
// the reduction over the 32 lanes of column (lane >> (5 - log2 GS)).
template <int GS, class Op>
__device__ __forceinline__ float warp_col_reduce(float (&v)[GS], int lane, Op op) {
  constexpr int LOG = Cfg<GS>::LOG;
#pragma unroll
  for (int m = 0; m < LOG; ++m) {
    const int o = 16 >> m;
    const int half = GS >> (m + 1);
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < GS / 2; ++j) {
      if (j < half) {
        const float send = up ? v[j] : v[j + half];
        const float keep = up ? v[j + half] : v[j];
        v[j] = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, o));
      }
    }
  }
#pragma unroll
  for (int o = 16 >> LOG; o > 0; o >>= 1) v[0] = op(v[0], __shfl_xor_sync(0xFFFFFFFFu, v[0], o));
  return v[0];
}

// kTok list entries from `base` (lane l holds entries base + l + 32 j); -1 past e1.
struct Window {
  int tok[4];
  int64_t base;
};

__device__ __forceinline__ Window load_window(const int32_t* __restrict__ list, int64_t base, int64_t e1, int lane) {
  Window w;
  w.base = base;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t e = base + 32 * j + lane;
    w.tok[j] = e < e1 ? __ldg(list + e) : -1;
  }
  return w;
}

// Warp 0: gather the next (up to) kTok valid entries of list[pos, e1) into
// dst, in list order.  Entries equal to -1 are padding; other entries outside
// [0, p] are skipped and flagged.  Returns the count; pos moves past what was
// consumed.  `pre` is the window at pos when it was loaded ahead of time.
__device__ int fill_tile(const int32_t* __restrict__ list, int64_t& pos, int64_t e1, int64_t p, int32_t* dst,
                         int lane, int32_t* status, const Window& pre) {
  __syncwarp();
  const uint32_t lt = (1u << lane) - 1u;
  int filled = 0;
  bool use_pre = pre.base == pos;
  while (filled < kTok && pos < e1) {
    int tok[4];
    if (use_pre) {
#pragma unroll
      for (int j = 0; j < 4; ++j) tok[j] = pre.tok[j];
      use_pre = false;
    } else {
      const Window w = load_window(list, pos, e1, lane);
#pragma unroll
      for (int j = 0; j < 4; ++j) tok[j] = w.tok[j];
    }
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (filled < kTok && pos < e1) {  // warp-uniform
        const bool ok = tok[j] >= 0 && (int64_t)tok[j] <= p;
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
        const int rank = __popc(m & lt);
        const int room = kTok - filled;
        int take = 32;  // lanes of this chunk consumed
        if (__popc(m) > room) take = __ffs(__ballot_sync(0xFFFFFFFFu, ok && rank == room)) - 1;
        if (ok && lane < take) dst[filled + rank] = tok[j];
        bad |= lane < take && tok[j] != -1 && !ok;
        filled += __popc(m & (take == 32 ? 0xFFFFFFFFu : ((1u << take) - 1u)));
        pos = min(pos + take, e1);
      }
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0 && status) atomicOr(status, kStatusBadIndex);
  }
  __syncwarp();
  return filled;
}

// Ten warps put three on some SM sub-partitions, which caps a thread at 168 registers.
template <int GS>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_tc_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                          const uint16_t* __restrict__ v, const int32_t* __restrict__ token_idx,
                          uint16_t* __restrict__ o, float* __restrict__ lse, int32_t* __restrict__ status,
                          float* __restrict__ partial, int64_t n_q, int64_t n_kv, int H, int Hkv, int topk, int splits,
                          float qscale, int64_t n_query, int n_sub, int64_t n_items) {
  using C = Cfg<GS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = H / Hkv;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  int2* meta = reinterpret_cast<int2*>(smem + C::META_OFF);
  auto fail = [&]() {
    *abort_flag = 1;
    if (status) atomicOr(status, kStatusTimeout);
  };

  // Rows of the q and weight operands that no copy writes stay zero.
  for (int i = tid; i < kNS * (C::QOP / 16); i += kThreads) {
    const int stg = i / (C::QOP / 16), c = i % (C::QOP / 16);
    *reinterpret_cast<uint4*>(smem + stg * C::STAGE + C::Q_OFF + c * 16) = make_uint4(0, 0, 0, 0);
  }
  for (int i = tid; i < 2 * (C::POP / 16); i += kThreads)
    *reinterpret_cast<uint4*>(smem + C::P_OFF + i * 16) = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  if (warp == kWarpQK) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(bar(B_FULL + i), kProd * 32 + 1);  // every producer thread's copies + the metadata
      mbar_init(bar(B_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PREADY + i), 128);
      mbar_init(bar(B_PFREE + i), 1);
      mbar_init(bar(B_DRAIN + i), 1);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kProd) {
    // ---------------- producers ----------------
    int32_t* ids = reinterpret_cast<int32_t*>(smem + C::IDX_OFF);  // [3][kTok]
    int2* pinfo = reinterpret_cast<int2*>(smem + C::PINFO_OFF);    // [3]
    const int rin = lane >> 4, cg = lane & 15, hh = cg >> 3, cc = cg & 7;
    const size_t tstride = (size_t)Hkv * kD;
    uint32_t gt = 0;  // tiles issued by this CTA
    bool stop = false;
    for (int64_t it = blockIdx.x; it < n_items && !stop; it += gridDim.x) {
      const Item w = item_of(it, n_sub, n_query, splits);
      const int64_t seq = w.qg / n_q;
      const int64_t p = n_kv - n_q + w.qg % n_q;
      const int h0 = w.g * G + w.sub * GS;
      const int gs = min(GS, G - w.sub * GS);
      const int32_t* list = token_idx + w.qg * topk;
      const int per = (topk + splits - 1) / splits;
      int64_t pos = min((int64_t)w.split * per, (int64_t)topk);
      const int64_t e1 = min(pos + per, (int64_t)topk);
      const uint16_t* kb = k + ((size_t)seq * n_kv * Hkv + w.g) * kD + cg * 8;
      const uint16_t* vb = v + ((size_t)seq * n_kv * Hkv + w.g) * kD + cg * 8;
      int cnt = 0;  // warp 0: valid entries of the tile about to be published
      Window win;   // warp 0: list window of the tile after the one being filled
      if (warp == 0) {
        // The next item's list entries go to L2 now; its first tile is filled after this item's last.
        const int64_t nit = it + gridDim.x;
        if (nit < n_items) {
          const Item wn = item_of(nit, n_sub, n_query, splits);
          const int64_t n0 = min((int64_t)wn.split * per, (int64_t)topk), n1 = min(n0 + per, (int64_t)topk);
          const int32_t* nl = token_idx + wn.qg * topk;
          for (int64_t e = n0 + 32 * lane; e < n1; e += 32 * 32) prefetch_l2(nl + e);
        }
        cnt = fill_tile(list, pos, e1, p, ids + (gt % 3) * kTok, lane, status, load_window(list, pos, e1, lane));
        win = load_window(list, pos, e1, lane);
      }
      bool first = true;
      while (true) {
        const int s = (int)(gt % kNS), ib = (int)(gt % 3);
        if (warp == 0) {
          // One tile of look-ahead tells whether this tile is the item's last.  Its list window
          // was loaded one tile earlier, before that tile's copies queued up behind it.
          const int nxt = pos < e1 ? fill_tile(list, pos, e1, p, ids + ((gt + 1) % 3) * kTok, lane, status, win) : 0;
          win = load_window(list, pos, e1, lane);
          if (lane == 0) pinfo[ib] = make_int2(cnt, nxt == 0 ? 1 : 0);
          cnt = nxt;
        }
        int ok = 1;
        if (gt >= (uint32_t)kNS && lane == 0) ok = mbar_wait(bar(B_EMPTY + s), ((gt / kNS) + 1) & 1) ? 1 : 0;
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!producer_sync_and(ok)) {  // also publishes ids[ib] and pinfo[ib] to the producer warps
          if (warp == 0 && lane == 0) fail();
          stop = true;
          break;
        }
        const int2 pi = pinfo[ib];
        const bool last = pi.y != 0;
        const uint32_t st = sbase + (uint32_t)(s * C::STAGE);
        if (warp == 0 && lane == 0) {
          meta[s] = make_int2(pi.x, (first ? 1 : 0) | (last ? 2 : 0));
          mbar_arrive(bar(B_FULL + s));
        }
        // Rows 32 warp .. 32 warp + 31 of the tile (token 0 pads a short tile): 16 lanes per
        // 256-byte row, two rows per step.
        const int tok_l = 32 * warp + lane < pi.x ? ids[ib * kTok + 32 * warp + lane] : 0;
#pragma unroll 4
        for (int i2 = 0; i2 < 16; ++i2) {
          const int rr = 2 * i2 + rin;
          const int tok = __shfl_sync(0xFFFFFFFFu, tok_l, rr);
          const int r = 32 * warp + rr;
          const uint32_t dst = st + (uint32_t)(hh * C::HALF + r * 128 + ((cc ^ (r & 7)) << 4));
          cp_async16_all(dst + C::K_OFF, kb + (size_t)tok * tstride);
          cp_async16_all(dst + C::V_OFF, vb + (size_t)tok * tstride);
        }
        if (warp == 0) {  // q rows of the item's heads: row n of the 16-row operand
          for (int n = rin; n < gs; n += 2) {
            const uint16_t* src = q + ((size_t)w.qg * H + h0 + n) * kD + cg * 8;
            const uint32_t dst = st + (uint32_t)(C::Q_OFF + hh * (C::NQ * 128) + (n >> 3) * 1024 + (n & 7) * 128 +
                                                 ((cc ^ (n & 7)) << 4));
            cp_async16_all(dst, src);
          }
        }
        cp_async_arrive_noinc(bar(B_FULL + s));
        ++gt;
        first = false;
        if (last) break;
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // own copies land before the CTA can exit
  } else if (warp == kWarpQK || warp == kWarpPV) {
    // ---------------- MMA issuers ----------------
    if (lane == 0) {
      const bool is_qk = warp == kWarpQK;
      constexpr uint32_t kIdescS = idesc_bf16(128, C::NQ, false, false);
      constexpr uint32_t kIdescO = idesc_bf16(128, C::NO, true, false);
      uint32_t gt = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        int last = 0;
        do {
          const int s = (int)(gt % kNS), b = (int)(gt & 1);
          if (!mbar_wait(bar(B_FULL + s), (gt / kNS) & 1)) {
            ok = false;
            break;
          }
          const int2 mt = meta[s];  // read after the stage's wait (which clobbers memory)
          const uint32_t st = sbase + (uint32_t)(s * C::STAGE);
          if (is_qk) {
            // S[b] is free once the softmax of tile gt - 2 has read it.
            if (gt >= 2 && !mbar_wait(bar(B_PREADY + b), ((gt - 2) >> 1) & 1)) {
              ok = false;
              break;
            }
            fence_async_smem();
            tc_fence_after();
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + (uint32_t)(b * 16), desc_kmajor_sw128(st + C::K_OFF + h2 * C::HALF + kk * 32),
                          desc_kmajor_sw128(st + C::Q_OFF + h2 * (C::NQ * 128) + kk * 32), kIdescS,
                          (h2 | kk) ? 1u : 0u);
            umma_commit(bar(B_SFULL + b));
          } else {
            if (!mbar_wait(bar(B_PREADY + b), (gt >> 1) & 1)) {
              ok = false;
              break;
            }
            fence_async_smem();
            tc_fence_after();
            const uint32_t vt = st + C::V_OFF;
            const uint32_t pb = sbase + (uint32_t)(C::P_OFF + b * C::POP);
            const bool first = (mt.y & 1) != 0;
#pragma unroll
            for (int j = 0; j < kTok / 16; ++j)
              umma_bf16(tmem + C::COL_O, desc_mnmajor_sw128(vt + j * 2048, C::HALF),
                        desc_kmajor_sw128(pb + (j >> 2) * (C::NO * 128) + (j & 3) * 32), kIdescO,
                        (first && j == 0) ? 0u : 1u);
            umma_commit(bar(B_EMPTY + s));
            umma_commit(bar(B_PFREE + b));
          }
          last = mt.y & 2;
          ++gt;
        } while (!last);
      }
      if (!ok) fail();
      const int d = is_qk ? 0 : 1;
      umma_commit(bar(B_DRAIN + d));
      mbar_wait(bar(B_DRAIN + d), 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- softmax and output ----------------
    const int wq = warp - 4;
    const int i = tid - 128;  // token row of the tile / output dimension
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    volatile float* red = reinterpret_cast<volatile float*>(smem + C::RED_OFF);
    volatile float* red_sum = red + 2 * 4 * 16;
    volatile float* red_err = red_sum + 4 * 16;
    // Byte offset of this thread's token column in row n of the weight operand (K-major, 128-byte swizzle).
    const int ch = (i & 63) >> 3;
    const uint32_t pcol = (uint32_t)((i >> 6) * (C::NO * 128) + (i & 7) * 2);
    auto poff = [&](int n) { return pcol + (uint32_t)((n >> 3) * 1024 + (n & 7) * 128 + ((ch ^ (n & 7)) << 4)); };
    const float lim = 8.f / qscale;
    const int col_mine = lane >> (5 - C::LOG);  // column this lane holds after a reduction
    const bool col_writer = (lane & ((32 >> C::LOG) - 1)) == 0;
    uint32_t gt = 0;
    bool err = false;
    for (int64_t it = blockIdx.x; it < n_items && !err; it += gridDim.x) {
      const Item w = item_of(it, n_sub, n_query, splits);
      const int h0 = w.g * G + w.sub * GS;
      const int gs = min(GS, G - w.sub * GS);
      float m_run[GS], nmq[GS], lp[GS];  // running max (unscaled), -m_run * qscale, partial row sums
#pragma unroll
      for (int j = 0; j < GS; ++j) {
        m_run[j] = -INFINITY;
        nmq[j] = 0.f;
        lp[j] = 0.f;
      }
      int last = 0;
      do {
        const int s = (int)(gt % kNS), b = (int)(gt & 1);
        bool bad = !mbar_wait(bar(B_FULL + s), (gt / kNS) & 1);
        const int2 mt = meta[s];
        bad = bad || !mbar_wait(bar(B_SFULL + b), (gt >> 1) & 1);
        bad = __any_sync(0xFFFFFFFFu, bad || err);  // err: a wait of the previous tile gave up
        float sc[GS];
        {
          uint32_t raw[GS];
#pragma unroll
          for (int j = 0; j < GS; ++j) raw[j] = 0xFF800000u;  // -inf
          if (!bad) {
            tc_fence_after();
            tmem_ld<GS>(tl + (uint32_t)(b * 16), raw);
          }
#pragma unroll
          for (int j = 0; j < GS; ++j) sc[j] = (i < mt.x && j < gs) ? __uint_as_float(raw[j]) : -INFINITY;
        }
        {
          float tmp[GS];
#pragma unroll
          for (int j = 0; j < GS; ++j) tmp[j] = sc[j];
          const float cm = warp_col_reduce<GS>(tmp, lane, [](float a, float c) { return fmaxf(a, c); });
          if (col_writer) red[(b * 4 + wq) * 16 + col_mine] = cm;
          if (lane == 0) red_err[wq] = bad ? 1.f : 0.f;
        }
        softmax_sync();
        if (red_err[0] + red_err[1] + red_err[2] + red_err[3] != 0.f) {  // every softmax thread stops together
          err = true;
          break;
        }
        float alpha[GS];
        bool resc = false;
#pragma unroll
        for (int j = 0; j < GS; ++j) {
          const float tmax = fmaxf(fmaxf(red[(b * 4 + 0) * 16 + j], red[(b * 4 + 1) * 16 + j]),
                                   fmaxf(red[(b * 4 + 2) * 16 + j], red[(b * 4 + 3) * 16 + j]));
          alpha[j] = 1.f;
          if (tmax > m_run[j] + lim) {  // the same decision in all 128 threads
            const float m_new = fmaxf(m_run[j], tmax);
            alpha[j] = exp2f((m_run[j] - m_new) * qscale);
            lp[j] *= alpha[j];
            m_run[j] = m_new;
            nmq[j] = -m_new * qscale;
            resc = true;
          }
        }
        if (resc && !(mt.y & 1)) {  // the accumulator holds earlier tiles of this item
          const uint32_t tp = gt - 1;
          const bool bad2 = __any_sync(0xFFFFFFFFu, !mbar_wait(bar(B_PFREE + (int)(tp & 1)), (tp >> 1) & 1));
          if (!bad2) {
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part) {  // hi columns, then lo columns
              uint32_t ov[GS];
              tmem_ld<GS>(tl + C::COL_O + part * GS, ov);
#pragma unroll
              for (int j = 0; j < GS; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha[j]);
              tmem_st<GS>(tl + C::COL_O + part * GS, ov);
            }
          }
          err = err || bad2;
        }
        float pw[GS];
#pragma unroll
        for (int j = 0; j < GS; ++j) {
          pw[j] = fast_exp2(fmaf(sc[j], qscale, nmq[j]));  // 0 for masked rows and unused heads
          lp[j] += pw[j];
        }
        if (gt >= 2) err = err || __any_sync(0xFFFFFFFFu, !mbar_wait(bar(B_PFREE + b), ((gt - 2) >> 1) & 1));
        uint8_t* pbuf = smem + C::P_OFF + b * C::POP;
#pragma unroll
        for (int j = 0; j < GS; ++j) {
          const uint32_t pu = __float_as_uint(pw[j]);
          const __nv_bfloat16 lo = __float2bfloat16_rn(pw[j] - __uint_as_float(pu & 0xFFFF0000u));
          *reinterpret_cast<uint16_t*>(pbuf + poff(j)) = (uint16_t)(pu >> 16);
          *reinterpret_cast<__nv_bfloat16*>(pbuf + poff(GS + j)) = lo;
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_PREADY + b));
        last = mt.y & 2;
        if (last) {
          const bool bad3 = __any_sync(0xFFFFFFFFu, err || !mbar_wait(bar(B_PFREE + b), (gt >> 1) & 1));
          float oacc[GS];  // this dimension of every head's output: hi column + lo column
#pragma unroll
          for (int j = 0; j < GS; ++j) oacc[j] = 0.f;
          if (!bad3) {
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              uint32_t ov[GS];
              tmem_ld<GS>(tl + C::COL_O + part * GS, ov);
#pragma unroll
              for (int j = 0; j < GS; ++j) oacc[j] += __uint_as_float(ov[j]);
            }
            tc_fence_before();
          }
          {
            float tmp[GS];
#pragma unroll
            for (int j = 0; j < GS; ++j) tmp[j] = lp[j];
            const float cs = warp_col_reduce<GS>(tmp, lane, [](float a, float c) { return a + c; });
            if (col_writer) red_sum[wq * 16 + col_mine] = cs;
            if (lane == 0) red_err[wq] = bad3 ? 1.f : 0.f;
          }
          softmax_sync();
          if (red_err[0] + red_err[1] + red_err[2] + red_err[3] != 0.f) {
            err = true;
            break;
          }
#pragma unroll
          for (int j = 0; j < GS; ++j) {
            if (j < gs) {
              const float L =
                  (red_sum[0 * 16 + j] + red_sum[1 * 16 + j]) + (red_sum[2 * 16 + j] + red_sum[3 * 16 + j]);
              const float M = m_run[j] * qscale;
              const float O = oacc[j];
              const int64_t row = w.qg * H + h0 + j;
              if (splits == 1) {
                const __nv_bfloat16 ob = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
                o[row * kD + i] = *reinterpret_cast<const uint16_t*>(&ob);
                if (i == 0 && lse) lse[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
              } else {
                float* pt = partial + (row * splits + w.split) * (kD + 2);
                if (i == 0) {
                  pt[0] = M;
                  pt[1] = L;
                }
                pt[2 + i] = O;
              }
            }
          }
        }
        ++gt;
      } while (!last);
    }
    if (err && i == 0) fail();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpQK) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

int sm_count() {
  static std::atomic<int> cached[64] = {};  // per device; several host threads may launch at once
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int GS>
cudaError_t launch_gs(const Shape& s, const void* q, const void* k, const void* v, const int32_t* token_idx, void* o,
                      float* lse, int32_t* status, int splits, float* partial, cudaStream_t st) {
  auto kern = sparse_attn_tc_kernel<GS>;
  cudaError_t e = ensure_smem((const void*)kern, Cfg<GS>::SMEM);
  if (e != cudaSuccess) return e;
  const int G = s.H / s.Hkv;
  const int n_sub = (G + GS - 1) / GS;
  const int64_t n_items = (int64_t)s.Hkv * n_sub * s.n_query * splits;
  const int64_t grid = n_items < sm_count() ? n_items : sm_count();
  const float qscale = s.scale * 1.4426950408889634f;
  kern<<<(unsigned)grid, kThreads, Cfg<GS>::SMEM, st>>>(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), token_idx,
      static_cast<uint16_t*>(o), lse, status, partial, s.n_q, s.n_kv, s.H, s.Hkv, s.k, splits, qscale, s.n_query,
      n_sub, n_items);
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  return launch_attn_merge(s, partial, o, lse, splits, st);
}

}  // namespace

// Used where heads share K/V (GQA/MQA): with one head per KV head the gather-bound CUDA-core-issued
// kernel moves the rows faster than one CTA per SM can copy and score them.
bool sparse_attn_tc_eligible(const Shape& s) {
  return HISA_ATTN_TC && s.d == kD && s.k >= 1 && s.n_query >= 1 && s.H / s.Hkv >= HISA_ATTN_TC_MIN_GROUP;
}

cudaError_t launch_sparse_attn_tc(const Shape& s, const void* q, const void* k, const void* v,
                                  const int32_t* token_idx, void* o, float* lse, int32_t* status, int splits,
                                  float* partial, cudaStream_t st) {
  if (!sparse_attn_tc_eligible(s)) return cudaErrorNotSupported;
  const int G = s.H / s.Hkv;
  if (G >= 16) return launch_gs<16>(s, q, k, v, token_idx, o, lse, status, splits, partial, st);
  if (G > 4) return launch_gs<8>(s, q, k, v, token_idx, o, lse, status, splits, partial, st);
  if (G > 2) return launch_gs<4>(s, q, k, v, token_idx, o, lse, status, splits, partial, st);
  if (G == 2) return launch_gs<2>(s, q, k, v, token_idx, o, lse, status, splits, partial, st);
  return launch_gs<1>(s, q, k, v, token_idx, o, lse, status, splits, partial, st);
}

}  // namespace hisa
