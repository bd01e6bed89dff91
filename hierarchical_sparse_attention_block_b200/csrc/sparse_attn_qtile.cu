// Step 6 for many queries per sequence (prefill), head dimension 128, on the
// 5th-generation tensor cores.  QbitAI HISA article, "HISA的關鍵優勢在於": the
// attention after the indexer is the usual softmax attention, here over each
// query's selected tokens.
//
// Queries select their tokens independently, but a tile of 128 consecutive
// queries together touches nearly every visible block of 128 keys once the
// context is a few times m*B long (each query keeps m of the c+1 visible
// blocks).  So instead of gathering each query's k rows on its own, a CTA
// takes one (head, tile of 128 queries), walks the tile's visible key tiles of
// 128 tokens, stages each K and V tile once in shared memory (TMA, 128-byte
// swizzle) and scores all 128 queries against all 128 keys on the tensor
// cores.  A query's selection enters as a 128-bit mask per key tile: only the
// selected entries get a softmax weight, so the result is attention over the
// selected set exactly as the gather kernels compute it.  Every K/V row then
// crosses L2 -> SM once per query tile instead of once per query that keeps it.
//
// The masks are built first (attn_mask_kernel) from the token lists: bit
// (t mod 128) of word [query tile][key tile t / 128][row] is set for every
// entry t of a row's list that lies in [0, p] and exceeds every in-range entry
// before it; -1 entries are padding; other entries are skipped and flagged.
//
// Roles of the attention CTA (224 threads):
//   * warps 0-3, one thread per query row (TMEM lane = row): first the row's
//     q into tensor memory (the A operand of the score MMA); then per key
//     tile read the row's 128 scores, mask them, raise the running max lazily
//     (O in TMEM is rescaled only when a weight would exceed 2^8), write the
//     weights over the scores, and at the end write O / l and the LSE;
//   * warp 4, one thread: TMA loads of the K tiles into a ring of three slots,
//     a slot refilled as soon as its score MMA has read it;
//   * warp 6, one thread: TMA loads of the V tiles and 2 KB mask blocks into a
//     ring of three slots, refilled once the output MMA has read them;
//   * warp 5, one thread: S_j = Q K_jᵀ into one of two TMEM buffers
//     (tcgen05.mma kind::f16, M = 128 queries, N = 128 keys, q from tensor
//     memory), then O += P_{j-1} V_{j-1} (M = 128 queries, N = 128
//     dimensions; V read MN-major from its rows) with the weights P as the A
//     operand in tensor memory, in the buffer their scores came from: the
//     weights carry ~16 significant bits as a bf16 pair hi + lo (hi the upper
//     half of the fp32 weight, lo the rounded rest), so the output MMA runs
//     over K = 2 x 128 (hi columns, then lo columns, both against the same V
//     rows).  MMAs of one thread run in issue order, so S_{j+2} is written
//     into the buffer only after P_j has been read from it.
// Every wait is bounded (1 s): a timeout sets status bit 1 and the CTA stops.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

#ifndef HISA_ATTN_QT
#define HISA_ATTN_QT 1
#endif
// The query-tile kernel is used while the keys a query can see, averaged over the queries, are at
// most this many times the tokens it keeps: a tile costs about the visible keys, a gather about
// the kept tokens.
#ifndef HISA_ATTN_QT_RATIO
#define HISA_ATTN_QT_RATIO 48
#endif
// Fewest queries per sequence for the query-tile kernel.
#ifndef HISA_ATTN_QT_MIN_NQ
#define HISA_ATTN_QT_MIN_NQ 64
#endif

namespace hisa {
namespace {

using namespace tc;

constexpr int kRows = 128;  // queries per tile = keys per key tile
constexpr int kD = 128;     // head dimension
constexpr int kNS = 3;      // slots of the K ring and of the V ring
constexpr int kThreads = 224;
constexpr int kWarpK = 4, kWarpMMA = 5, kWarpV = 6;
// Tensor memory: scores / weights buffer 0 at columns 0-127, buffer 1 at 128-255, output O at
// 256-383, the query tile (bf16 pairs) at 384-447.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256, kColQ = 384;

constexpr int kHalf = kRows * 128;      // 64 columns of 128 rows of bf16 (one 128-byte swizzle span): 16 KB
constexpr int kTile = 2 * kHalf;        // a 128 x 128 bf16 tile as two column halves
constexpr int kMaskBytes = kRows * 16;  // 128 rows x 128 bits
constexpr int K_OFF = 0;                        // K slot i at K_OFF + i * kTile
constexpr int V_OFF = K_OFF + kNS * kTile;      // V slot i at V_OFF + i * kTile
constexpr int MASK_OFF = V_OFF + kNS * kTile;   // mask of V slot i at MASK_OFF + i * kMaskBytes
constexpr int BAR_OFF = MASK_OFF + kNS * kMaskBytes;
enum : int {
  B_KFULL = 0,
  B_KEMPTY = kNS,
  B_VFULL = 2 * kNS,
  B_VEMPTY = 3 * kNS,
  B_QREADY = 4 * kNS,
  B_SFULL,  // [2]
  B_PREADY = B_SFULL + 2,
  B_PFREE,
  B_DRAIN,
  kNBar
};
constexpr int MISC_OFF = BAR_OFF + kNBar * 8;
constexpr int kSmem = MISC_OFF + 16 + 1024;  // + slack for the 1024-byte alignment of the swizzled tiles
static_assert(kSmem <= 227 * 1024, "shared memory budget");
static_assert(V_OFF % 1024 == 0 && kTile % 1024 == 0, "swizzle atoms stay 1024-byte aligned");

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// Upper halves of two fp32 values as a bf16 pair (x0 in the low half): truncation, exact in bf16.
__device__ __forceinline__ uint32_t pack_hi(float x0, float x1) {
  return (__float_as_uint(x0) >> 16) | (__float_as_uint(x1) & 0xFFFF0000u);
}

// Masks of one query tile: [key tile][row] x 128 bits, key tiles 0 .. (last position of the tile) / 128.
__global__ void __launch_bounds__(kRows) attn_mask_kernel(const int32_t* __restrict__ token_idx,
                                                          uint4* __restrict__ masks, int32_t* __restrict__ status,
                                                          int64_t n_q, int64_t n_kv, int topk, int nqt, int nkt) {
  const int qt = blockIdx.x, seq = blockIdx.y, r = threadIdx.x;
  const int64_t i0 = (int64_t)qt * kRows;
  const int nr = (int)min((int64_t)kRows, n_q - i0);
  const int64_t pos0 = n_kv - n_q + i0;
  const int64_t nv = (pos0 + nr - 1) / kRows + 1;
  uint4* base = masks + ((int64_t)seq * nqt + qt) * nkt * kRows;
  for (int64_t e = r; e < nv * kRows; e += kRows) base[e] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (r >= nr) return;
  const int64_t p = pos0 + r;
  const int32_t* list = token_idx + ((int64_t)seq * n_q + i0 + r) * topk;
  uint32_t* row = reinterpret_cast<uint32_t*>(base) + r * 4;  // word w of key tile kt: row[kt * 4 * kRows + w]
  int64_t last = -1;                                          // largest in-range entry so far
  int64_t word = -1;                                          // word being filled (t >> 5)
  uint32_t bits = 0;
  bool bad = false;
  auto take = [&](int t) {
    if (t == -1) return;
    if (t < 0 || (int64_t)t > p || (int64_t)t <= last) {
      bad = true;
      return;
    }
    last = t;
    const int64_t w = t >> 5;
    if (w != word) {
      if (word >= 0) row[(word >> 2) * (4 * kRows) + (word & 3)] = bits;
      word = w;
      bits = 0;
    }
    bits |= 1u << (t & 31);
  };
  if ((topk & 3) == 0) {
    const int4* l4 = reinterpret_cast<const int4*>(list);
    for (int e = 0; e < topk / 4; ++e) {
      const int4 t4 = __ldg(l4 + e);
      take(t4.x);
      take(t4.y);
      take(t4.z);
      take(t4.w);
    }
  } else {
    for (int e = 0; e < topk; ++e) take(__ldg(list + e));
  }
  if (word >= 0) row[(word >> 2) * (4 * kRows) + (word & 3)] = bits;
  if (bad && status) atomicOr(status, kStatusBadIndex);
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_qtile_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                             const uint16_t* __restrict__ q, const uint4* __restrict__ masks,
                             uint16_t* __restrict__ o, float* __restrict__ lse, int32_t* __restrict__ status,
                             int64_t n_q, int64_t n_kv, int H, int Hkv, int batch, int nqt, int nkt, float qscale) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return sb + (uint32_t)BAR_OFF + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + MISC_OFF + 4);
  auto fail = [&]() {
    *abort_flag = 1;
    if (status) atomicOr(status, kStatusTimeout);
  };

  // Work unit: heads outermost (the CTAs running together read one head's K and V, which the L2
  // keeps), then query tiles from the longest, then sequences.
  const int64_t per_head = (int64_t)nqt * batch;
  const int h = (int)(blockIdx.x / per_head);
  const int64_t rem = blockIdx.x - (int64_t)h * per_head;
  const int qt = nqt - 1 - (int)(rem / batch);
  const int seq = (int)(rem - (rem / batch) * batch);
  const int g = h / (H / Hkv);
  const int64_t row0 = (int64_t)seq * n_q + (int64_t)qt * kRows;  // first query row of the tile
  const int nr = (int)min((int64_t)kRows, n_q - (int64_t)qt * kRows);
  const int64_t pos0 = n_kv - n_q + (int64_t)qt * kRows;            // position of row 0
  const int nv = (int)((pos0 + nr - 1) / kRows) + 1;                // visible key tiles
  const uint4* mbase = masks + ((int64_t)seq * nqt + qt) * nkt * kRows;

  if (warp == kWarpMMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(bar(B_KFULL + i), 1);
      mbar_init(bar(B_KEMPTY + i), 1);
      mbar_init(bar(B_VFULL + i), 1);
      mbar_init(bar(B_VEMPTY + i), 1);
    }
    mbar_init(bar(B_QREADY), kRows);
    for (int i = 0; i < 2; ++i) mbar_init(bar(B_SFULL + i), 1);
    mbar_init(bar(B_PREADY), kRows);
    mbar_init(bar(B_PFREE), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpK || warp == kWarpV) {
    // ---------------- TMA producers: K tiles (warp 4), V tiles + masks (warp 6) ----------------
    if (lane == 0) {
      const bool is_k = warp == kWarpK;
      const CUtensorMap* map = is_k ? &map_k : &map_v;
      const int full = is_k ? B_KFULL : B_VFULL, empty = is_k ? B_KEMPTY : B_VEMPTY;
      const uint32_t base = sb + (uint32_t)(is_k ? K_OFF : V_OFF);
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
      int issued = 0;
      for (int j = 0; j < nv; ++j) {
        const int s = j % kNS;
        if (j >= kNS && !mbar_wait_or_abort(bar(empty + s), ((j / kNS) - 1) & 1, abort_flag)) {
          fail();
          break;
        }
        const uint32_t dst = base + (uint32_t)(s * kTile);
        const int z = (int)((int64_t)seq * n_kv + (int64_t)j * kRows);
        mbar_expect_tx(bar(full + s), is_k ? kTile : kTile + kMaskBytes);
        tma_load_3d(dst, map, 0, g, z, bar(full + s));
        tma_load_3d(dst + kHalf, map, 64, g, z, bar(full + s));
        if (!is_k)
          bulk_load(sb + (uint32_t)(MASK_OFF + s * kMaskBytes), mbase + (int64_t)j * kRows, kMaskBytes,
                    bar(full + s));
        issued = j + 1;
      }
      // The copies in flight land before the CTA may exit.
      for (int j = issued > kNS ? issued - kNS : 0; j < issued; ++j) mbar_wait(bar(full + j % kNS), (j / kNS) & 1);
    }
  } else if (warp == kWarpMMA) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);  // q (tensor memory), K K-major
      constexpr uint32_t kIdO = idesc_bf16(128, 128, false, true);   // P (tensor memory), V MN-major
      bool ok = mbar_wait_or_abort(bar(B_QREADY), 0, abort_flag);
      for (int j = 0; ok && j <= nv; ++j) {
        if (j < nv) {
          // Buffer j & 1 held P_{j-2}, whose output MMA was issued before this one.
          const int s = j % kNS;
          ok = mbar_wait_or_abort(bar(B_KFULL + s), (j / kNS) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kt = sb + (uint32_t)(K_OFF + s * kTile);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk)
            umma_bf16_ta(tmem + (uint32_t)((j & 1) * 128), tmem + kColQ + (uint32_t)(8 * kk),
                         desc_kmajor_sw128(kt + (kk >> 2) * kHalf + (kk & 3) * 32), kIdS, kk > 0 ? 1u : 0u);
          umma_commit(bar(B_SFULL + (j & 1)));
          umma_commit(bar(B_KEMPTY + s));
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj % kNS;
          ok = mbar_wait_or_abort(bar(B_VFULL + s), (jj / kNS) & 1, abort_flag) &&
               mbar_wait_or_abort(bar(B_PREADY), jj & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vt = sb + (uint32_t)(V_OFF + s * kTile);
          const uint32_t pt = tmem + (uint32_t)((jj & 1) * 128);
#pragma unroll
          for (int t = 0; t < 2 * (kRows / 16); ++t)  // keys 16 t' .. 16 t' + 15, t' = t mod 8: hi, then lo
            umma_bf16_ta(tmem + kColO, pt + (uint32_t)(8 * t), desc_mnmajor_sw128(vt + (t & 7) * 2048, kHalf), kIdO,
                         (jj > 0 || t > 0) ? 1u : 0u);
          umma_commit(bar(B_VEMPTY + s));
          umma_commit(bar(B_PFREE));
        }
      }
      if (!ok) fail();
      umma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0);
    }
  } else if (warp < 4) {
    // ---------------- softmax and output: warps 0-3, thread = query row ----------------
    const int r = tid;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    {
      // q of this row (zero past the last query) as bf16 pairs in columns kColQ .. kColQ + 63
      uint32_t qv[2][32];
      const uint4* qrow = reinterpret_cast<const uint4*>(q + ((row0 + r) * H + h) * (int64_t)kD);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 x = r < nr ? __ldg(qrow + c) : make_uint4(0u, 0u, 0u, 0u);
        qv[c >> 3][(c & 7) * 4 + 0] = x.x;
        qv[c >> 3][(c & 7) * 4 + 1] = x.y;
        qv[c >> 3][(c & 7) * 4 + 2] = x.z;
        qv[c >> 3][(c & 7) * 4 + 3] = x.w;
      }
      tmem_st32_issue(tl + kColQ, qv[0]);
      tmem_st32_issue(tl + kColQ + 32, qv[1]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_QREADY));
    }
    float m_run = -INFINITY;  // running max of the row's selected raw scores
    float l = 0.f;            // sum of the row's weights, relative to m_run
    const float lim = 8.f / qscale;
    bool err = false;
    for (int j = 0; j < nv; ++j) {
      const int s = j % kNS, b = j & 1;
      const bool ok = mbar_wait_or_abort(bar(B_VFULL + s), (j / kNS) & 1, abort_flag) &&
                      mbar_wait_or_abort(bar(B_SFULL + b), (j >> 1) & 1, abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        err = true;
        break;
      }
      tc_fence_after();
      float sv[kRows];
      {
        uint32_t raw[4][32];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) tmem_ld32_issue(tl + (uint32_t)(b * 128 + 32 * c4), raw[c4]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kRows; ++c) sv[c] = __uint_as_float(raw[c >> 5][c & 31]);
      }
      const uint4 mk = *reinterpret_cast<const uint4*>(smem + MASK_OFF + s * kMaskBytes + r * 16);
      const uint32_t mw[4] = {mk.x, mk.y, mk.z, mk.w};
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        sv[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? sv[c] : -INFINITY;
        tmax = fmaxf(tmax, sv[c]);
      }
      float alpha = 1.f;
      bool resc = false;
      if (tmax > m_run + lim) {  // also the first selected entry of the row (m_run = -inf)
        if (m_run != -INFINITY) {
          alpha = exp2f((m_run - tmax) * qscale);
          l *= alpha;
          resc = true;
        }
        m_run = tmax;
      }
      if (__any_sync(0xFFFFFFFFu, resc)) {  // O holds earlier tiles: rescale it once they are in
        const bool ok2 = mbar_wait_or_abort(bar(B_PFREE), (j - 1) & 1, abort_flag);
        if (!__all_sync(0xFFFFFFFFu, ok2)) {
          err = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t ov[32];
          tmem_ld32_issue(tl + kColO + 32 * c4, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32_issue(tl + kColO + 32 * c4, ov);
        }
        tmem_wait_st();
      }
      const float nmq = m_run == -INFINITY ? 0.f : -m_run * qscale;
      // Weights over the scores of buffer b: hi pairs in columns 0-63, lo pairs in 64-127.
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = fast_exp2(fmaf(sv[32 * c4 + 2 * i], qscale, nmq));  // 0 where masked
          const float p1 = fast_exp2(fmaf(sv[32 * c4 + 2 * i + 1], qscale, nmq));
          l += p0 + p1;
          hi[i] = pack_hi(p0, p1);
          lo[i] = pack_bf16(p0 - __uint_as_float(__float_as_uint(p0) & 0xFFFF0000u),
                            p1 - __uint_as_float(__float_as_uint(p1) & 0xFFFF0000u));
        }
        tmem_st16_issue(tl + (uint32_t)(b * 128 + 16 * c4), hi);
        tmem_st16_issue(tl + (uint32_t)(b * 128 + 64 + 16 * c4), lo);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PREADY));
    }
    if (!err) {
      const bool ok = mbar_wait_or_abort(bar(B_PFREE), (nv - 1) & 1, abort_flag);
      err = !__all_sync(0xFFFFFFFFu, ok);
    }
    if (!err) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* orow = o + ((row0 + r) * H + h) * (int64_t)kD;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t ov[32];
        tmem_ld32_issue(tl + kColO + 32 * c4, ov);
        tmem_wait_ld();
        if (r < nr) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(ov[8 * q4 + 0]) * inv, __uint_as_float(ov[8 * q4 + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(ov[8 * q4 + 2]) * inv, __uint_as_float(ov[8 * q4 + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(ov[8 * q4 + 4]) * inv, __uint_as_float(ov[8 * q4 + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(ov[8 * q4 + 6]) * inv, __uint_as_float(ov[8 * q4 + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + 32 * c4 + 8 * q4) = w;
          }
        }
      }
      if (r < nr && lse)
        lse[(row0 + r) * H + h] = l > 0.f ? (m_run * qscale + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
    if (err && lane == 0) fail();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

int64_t n_tiles(int64_t n) { return (n + kRows - 1) / kRows; }

}  // namespace

bool sparse_attn_qtile_eligible(const Shape& s) {
  if (!HISA_ATTN_QT || s.d != kD || s.n_q < HISA_ATTN_QT_MIN_NQ) return false;
  if ((int64_t)s.batch * s.n_kv >= ((int64_t)1 << 31) || s.n_query >= ((int64_t)1 << 31)) return false;
  if ((int64_t)s.H * n_tiles(s.n_q) * s.batch >= ((int64_t)1 << 31)) return false;
  const double avg_keys = (double)(s.n_kv - s.n_q) + 0.5 * (double)s.n_q;
  return avg_keys <= (double)HISA_ATTN_QT_RATIO * (double)s.k;
}

size_t sparse_attn_qtile_bytes(const Shape& s) {
  return (size_t)s.batch * (size_t)n_tiles(s.n_q) * (size_t)n_tiles(s.n_kv) * kMaskBytes;
}

cudaError_t launch_sparse_attn_qtile(const Shape& s, const void* q, const void* k, const void* v,
                                     const int32_t* token_idx, void* o, float* lse, int32_t* status, void* masks,
                                     cudaStream_t st) {
  if (!sparse_attn_qtile_eligible(s)) return cudaErrorNotSupported;
  CUtensorMap mk, mv;
  if (!map_bf16_rows_of_head(&mk, k, kD, (uint64_t)s.Hkv, (uint64_t)s.batch * s.n_kv, kRows) ||
      !map_bf16_rows_of_head(&mv, v, kD, (uint64_t)s.Hkv, (uint64_t)s.batch * s.n_kv, kRows))
    return cudaErrorNotSupported;
  const int nqt = (int)n_tiles(s.n_q), nkt = (int)n_tiles(s.n_kv);
  uint4* m = static_cast<uint4*>(masks);
  attn_mask_kernel<<<dim3((unsigned)nqt, (unsigned)s.batch), kRows, 0, st>>>(token_idx, m, status, s.n_q, s.n_kv, s.k,
                                                                             nqt, nkt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = ensure_smem((const void*)sparse_attn_qtile_kernel, kSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (int64_t)s.H * nqt * s.batch;
  const float qscale = s.scale * 1.4426950408889634f;
  sparse_attn_qtile_kernel<<<(unsigned)grid, kThreads, kSmem, st>>>(mk, mv, static_cast<const uint16_t*>(q), m,
                                                                    static_cast<uint16_t*>(o), lse,
                                                                    status, s.n_q, s.n_kv, s.H, s.Hkv, s.batch, nqt,
                                                                    nkt, qscale);
  return cudaGetLastError();
}

}  // namespace hisa
