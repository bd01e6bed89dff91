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
// A CTA takes TWO consecutive query tiles A and B of one head (256 queries), so
// every K/V tile it stages serves 256 queries, and their softmax work
// alternates with each other's MMAs (ping-pong).  Roles (352 threads):
//   * warps 0-3 (tile A) and 4-7 (tile B), one thread per query row (TMEM
//     lane = row, warp w reads the lanes of quarter w % 4): per key tile read
//     the row's 128 scores, mask them, raise the running max lazily (O in TMEM
//     is rescaled only when a weight would exceed 2^8), write the weights over
//     the scores, and at the end write O / l and the LSE;
//   * warp 8, one thread: TMA loads of both query tiles (once) and of the K
//     tiles into a ring of two slots, a slot refilled once both score MMAs of
//     its key tile have read it;
//   * warp 10, one thread: TMA loads of the V tiles and of both query tiles'
//     2 KB mask blocks into a ring of two slots, refilled once both output
//     MMAs of the key tile have read them;
//   * warp 9, one thread: per key tile j, O_A += P_A(j) V_j, S_A(j+1) =
//     Q_A K_{j+1}ᵀ, O_B += P_B(j) V_j, S_B(j+1) = Q_B K_{j+1}ᵀ (tcgen05.mma
//     kind::f16, M = 128 queries, N = 128; scores bf16, outputs fp16 with the
//     weights P as the A operand in tensor memory, written over the scores
//     they came from: MMAs of one thread run in issue order, so S_A(j+1)
//     overwrites P_A(j) only after O_A += P_A(j) V_j has read it).  While the
//     warps of tile A work on S_A(j), the tensor cores run tile B's MMAs, and
//     the other way round.  Tensor memory: S_A | S_B | O_A | O_B, 128 columns
//     each.
// Precision of the output MMA: the weights (at most 2^8 with the lazy max)
// are rounded to fp16, 11 significant bits, so a row's output moves by at most
// 2^-11 * max |v| (rows normalised by the fp32 sum of the unrounded weights).
// V enters as fp16 too (both operands of one MMA have one type): a pre-pass
// (attn_v_max_kernel, attn_v_half_kernel) converts it exactly, scaled per KV
// head by a power of two 2^-e that brings the head's largest |v| below 2^15;
// the output is multiplied back by 2^e.  bf16 has 8 significant bits, so the
// conversion is exact apart from values that fall below fp16's normal range,
// which lose less than 2^-25 of the head's largest |v|.
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
constexpr int kNS = 2;      // slots of the K ring and of the V ring
constexpr int kThreads = 352;
constexpr int kWarpK = 8, kWarpMMA = 9, kWarpV = 10;
constexpr uint32_t kTmemCols = 512;
// Tensor memory columns of query tile t: scores / weights at col_s(t), output at col_o(t).
__host__ __device__ constexpr uint32_t col_s(int t) { return 128u * (uint32_t)t; }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 128u * (uint32_t)t; }

constexpr int kHalf = kRows * 128;      // 64 columns of 128 rows of 16-bit values (one 128-byte swizzle span): 16 KB
constexpr int kTile = 2 * kHalf;        // a 128 x 128 tile as two column halves
constexpr int kMaskBytes = kRows * 16;  // 128 rows x 128 bits
constexpr int Q_OFF = 0;                        // query tile t at Q_OFF + t * kTile
constexpr int K_OFF = Q_OFF + 2 * kTile;        // K slot i at K_OFF + i * kTile
constexpr int V_OFF = K_OFF + kNS * kTile;      // V slot i at V_OFF + i * kTile
constexpr int MASK_OFF = V_OFF + kNS * kTile;   // masks of V slot i, query tile t at MASK_OFF + (2 i + t) * kMaskBytes
constexpr int BAR_OFF = MASK_OFF + 2 * kNS * kMaskBytes;
enum : int {
  B_KFULL = 0,
  B_KEMPTY = kNS,
  B_VFULL = 2 * kNS,
  B_VEMPTY = 3 * kNS,
  B_QFULL = 4 * kNS,
  B_SFULL,                // [2]: per query tile
  B_PREADY = B_SFULL + 2, // [2]
  B_PFREE = B_PREADY + 2, // [2]
  B_DRAIN = B_PFREE + 2,
  kNBar
};
constexpr int MISC_OFF = BAR_OFF + kNBar * 8;
constexpr int kSmem = MISC_OFF + 16 + 1024;  // + slack for the 1024-byte alignment of the swizzled tiles
static_assert(kSmem <= 227 * 1024, "shared memory budget");
static_assert(K_OFF % 1024 == 0 && V_OFF % 1024 == 0 && kTile % 1024 == 0, "swizzle atoms stay 1024-byte aligned");

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed pairs of fp32 (sm_100 f32x2 instructions): a * b + c, a + b.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
        "l"(*reinterpret_cast<uint64_t*>(&c)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t r;
  asm("add.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
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

// Largest |v| of every KV head of V [rows][Hkv][128] bf16, as the bits of |v| (which order like
// unsigned integers); blockIdx.y = KV head, 16 threads per 256-byte row slice.  hmax starts at 0.
__global__ void __launch_bounds__(256) attn_v_max_kernel(const uint16_t* __restrict__ v, int64_t rows, int Hkv,
                                                         uint32_t* __restrict__ hmax) {
  __shared__ uint32_t wmax[8];
  const int hd = blockIdx.y, c = threadIdx.x & 15;
  uint32_t m = 0;
  for (int64_t r = (int64_t)blockIdx.x * 16 + (threadIdx.x >> 4); r < rows; r += (int64_t)gridDim.x * 16) {
    const uint4 x = ld_stream_v4(v + (r * Hkv + hd) * kD + c * 8);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < 8; ++i) m = max(m, wmax[i]);
    atomicMax(hmax + hd, m);
  }
}

// Exponent e >= 0 with (largest |v| of the head) * 2^-e < 2^15, from the bf16 bits of that |v|.
__device__ __forceinline__ int v_half_shift(uint32_t vmax_bits) { return max(0, (int)((vmax_bits >> 7) & 0xFFu) - 141); }

// V [rows][Hkv][128] bf16 -> fp16 scaled by 2^-e per head (exact but for values below fp16's normal
// range); vscale[head] = 2^e.
__global__ void __launch_bounds__(256) attn_v_half_kernel(const uint16_t* __restrict__ v, uint16_t* __restrict__ vh,
                                                          int64_t rows, int Hkv, const uint32_t* __restrict__ hmax,
                                                          float* __restrict__ vscale) {
  const int hd = blockIdx.y, c = threadIdx.x & 15;
  const int e = v_half_shift(hmax[hd]);
  const float sc = __uint_as_float((uint32_t)(127 - e) << 23);
  if (blockIdx.x == 0 && threadIdx.x == 0) vscale[hd] = __uint_as_float((uint32_t)(127 + e) << 23);
  for (int64_t r = (int64_t)blockIdx.x * 16 + (threadIdx.x >> 4); r < rows; r += (int64_t)gridDim.x * 16) {
    const int64_t at = (r * Hkv + hd) * kD + c * 8;
    const uint4 x = ld_stream_v4(v + at);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 p = __floats2half2_rn(__uint_as_float(w[i] << 16) * sc, __uint_as_float(w[i] & 0xFFFF0000u) * sc);
      h[i] = *reinterpret_cast<const uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(vh + at) = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// Eleven warps put three on some SM sub-partitions, which caps a thread at 168 registers.
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_qtile_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                             const __grid_constant__ CUtensorMap map_v, const uint4* __restrict__ masks,
                             const float* __restrict__ vscale, uint16_t* __restrict__ o, float* __restrict__ lse,
                             int32_t* __restrict__ status, int64_t n_q, int64_t n_kv, int H, int Hkv, int batch,
                             int nqt, int nkt, float qscale) {
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
  // keeps), then pairs of query tiles from the longest, then sequences.
  const int npair = (nqt + 1) / 2;
  const int64_t per_head = (int64_t)npair * batch;
  const int h = (int)(blockIdx.x / per_head);
  const int64_t rem = blockIdx.x - (int64_t)h * per_head;
  const int pair = npair - 1 - (int)(rem / batch);
  const int seq = (int)(rem - (rem / batch) * batch);
  const int g = h / (H / Hkv);
  const int ntile = 2 * pair + 1 < nqt ? 2 : 1;  // query tiles of this CTA
  // Query tile t (0 or 1) of the CTA: first row, rows, visible key tiles (0 for a missing tile B).
  auto row0_of = [&](int t) { return (int64_t)seq * n_q + (int64_t)(2 * pair + t) * kRows; };
  auto nr_of = [&](int t) { return (int)min((int64_t)kRows, n_q - (int64_t)(2 * pair + t) * kRows); };
  auto nv_of = [&](int t) {
    return t < ntile ? (int)((n_kv - n_q + (int64_t)(2 * pair + t) * kRows + nr_of(t) - 1) / kRows) + 1 : 0;
  };
  const int nv0 = nv_of(0), nv1 = nv_of(1);
  const int nvx = max(nv0, nv1);  // key tiles of the CTA

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
    mbar_init(bar(B_QFULL), 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(B_SFULL + t), 1);
      mbar_init(bar(B_PREADY + t), kRows);
      mbar_init(bar(B_PFREE + t), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpK || warp == kWarpV) {
    // ---------------- TMA producers: Q and K tiles (warp 8), V tiles + masks (warp 10) ----------------
    if (lane == 0) {
      const bool is_k = warp == kWarpK;
      const CUtensorMap* map = is_k ? &map_k : &map_v;
      const int full = is_k ? B_KFULL : B_VFULL, empty = is_k ? B_KEMPTY : B_VEMPTY;
      const uint32_t base = sb + (uint32_t)(is_k ? K_OFF : V_OFF);
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
      if (is_k) {
        mbar_expect_tx(bar(B_QFULL), ntile * kTile);
        for (int t = 0; t < ntile; ++t) {
          tma_load_3d(sb + Q_OFF + t * kTile, &map_q, 0, h, (int)row0_of(t), bar(B_QFULL));
          tma_load_3d(sb + Q_OFF + t * kTile + kHalf, &map_q, 64, h, (int)row0_of(t), bar(B_QFULL));
        }
      }
      int issued = 0;
      for (int j = 0; j < nvx; ++j) {
        const int s = j % kNS;
        if (j >= kNS && !mbar_wait_or_abort(bar(empty + s), ((j / kNS) - 1) & 1, abort_flag)) {
          fail();
          break;
        }
        const uint32_t dst = base + (uint32_t)(s * kTile);
        const int z = (int)((int64_t)seq * n_kv + (int64_t)j * kRows);
        const int nmask = is_k ? 0 : (j < nv0 ? 1 : 0) + (j < nv1 ? 1 : 0);
        mbar_expect_tx(bar(full + s), kTile + nmask * kMaskBytes);
        tma_load_3d(dst, map, 0, g, z, bar(full + s));
        tma_load_3d(dst + kHalf, map, 64, g, z, bar(full + s));
        if (!is_k) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (j < (t ? nv1 : nv0)) {
              const int qt = 2 * pair + t;
              const uint4* mb = masks + (((int64_t)seq * nqt + qt) * nkt + j) * kRows;
              bulk_load(sb + (uint32_t)(MASK_OFF + (2 * s + t) * kMaskBytes), mb, kMaskBytes, bar(full + s));
            }
          }
        }
        issued = j + 1;
      }
      // The copies in flight land before the CTA may exit.
      if (is_k) mbar_wait(bar(B_QFULL), 0);
      for (int j = issued > kNS ? issued - kNS : 0; j < issued; ++j) mbar_wait(bar(full + j % kNS), (j / kNS) & 1);
    }
  } else if (warp == kWarpMMA) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);  // Q and K both K-major
      constexpr uint32_t kIdO = idesc_f16(128, 128, false, true);    // P (tensor memory), V MN-major: fp16
      // S_t(j) = Q_t K_jᵀ (K_j in its slot already)
      auto scores = [&](int t, int j) {
        const uint32_t kt = sb + (uint32_t)(K_OFF + (j % kNS) * kTile);
        const uint32_t qb = sb + (uint32_t)(Q_OFF + t * kTile);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + col_s(t), desc_kmajor_sw128(qb + h2 * kHalf + kk * 32),
                      desc_kmajor_sw128(kt + h2 * kHalf + kk * 32), kIdS, (h2 | kk) ? 1u : 0u);
        umma_commit(bar(B_SFULL + t));
      };
      bool ok = mbar_wait_or_abort(bar(B_QFULL), 0, abort_flag) && mbar_wait_or_abort(bar(B_KFULL), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        if (nv0 > 0) scores(0, 0);
        if (nv1 > 0) scores(1, 0);
        umma_commit(bar(B_KEMPTY));
      }
      for (int j = 0; ok && j < nvx; ++j) {
        const int s = j % kNS;
        ok = mbar_wait_or_abort(bar(B_VFULL + s), (j / kNS) & 1, abort_flag);
        const bool next = j + 1 < nvx;
        bool knext = false;  // K_{j+1} waited for
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int nvt = t ? nv1 : nv0;
          if (!ok || j >= nvt) continue;
          ok = mbar_wait_or_abort(bar(B_PREADY + t), j & 1, abort_flag);
          if (!ok) continue;
          tc_fence_after();
          const uint32_t vt = sb + (uint32_t)(V_OFF + s * kTile);
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)  // keys 16 kk .. 16 kk + 15
            umma_bf16_ta(tmem + col_o(t), tmem + col_s(t) + (uint32_t)(8 * kk),
                         desc_mnmajor_sw128(vt + kk * 2048, kHalf), kIdO, (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(B_PFREE + t));
          if (j + 1 < nvt) {
            if (!knext) {
              ok = mbar_wait_or_abort(bar(B_KFULL + (j + 1) % kNS), ((j + 1) / kNS) & 1, abort_flag);
              if (!ok) continue;
              tc_fence_after();
              knext = true;
            }
            scores(t, j + 1);
          }
        }
        if (!ok) break;
        umma_commit(bar(B_VEMPTY + s));                    // V_j and its masks read by both output MMAs
        if (next) umma_commit(bar(B_KEMPTY + (j + 1) % kNS));  // K_{j+1} read by both score MMAs
      }
      if (!ok) fail();
      umma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0);
    }
  } else {
    // ---------------- softmax and output: warps 0-3 tile A, 4-7 tile B, thread = query row ----------------
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ts = tmem + lanes + col_s(t), to = tmem + lanes + col_o(t);
    const int nvt = t ? nv1 : nv0;
    const int64_t row0 = row0_of(t);
    const int nrt = nr_of(t);
    float m_run = -INFINITY;  // running max of the row's selected raw scores
    float2 l2 = {0.f, 0.f};   // sum of the row's weights, relative to m_run
    const float lim = 8.f / qscale;
    const float2 qs2 = {qscale, qscale};
    bool err = false;
    for (int j = 0; j < nvt; ++j) {
      const int s = j % kNS;
      const bool ok = mbar_wait_or_abort(bar(B_VFULL + s), (j / kNS) & 1, abort_flag) &&
                      mbar_wait_or_abort(bar(B_SFULL + t), j & 1, abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        err = true;
        break;
      }
      tc_fence_after();
      const uint4 mk = *reinterpret_cast<const uint4*>(smem + MASK_OFF + (2 * s + t) * kMaskBytes + r * 16);
      const uint32_t mw[4] = {mk.x, mk.y, mk.z, mk.w};
      // One pass, 32 columns at a time: mask the scores (-inf where the row did not keep the key),
      // take their max, and form the weights against the running max so far (kept in registers as
      // fp16 pairs; keys 2 i, 2 i + 1 -> pair i).  They stand unless this tile raises the max past
      // the lazy bound, in which case they are formed again below from the scores, which stay in
      // tensor memory until the weights are written over them.
      const float nmq0 = m_run == -INFINITY ? 0.f : -m_run * qscale;
      const float2 nmq0_2 = {nmq0, nmq0};
      uint32_t pw[64];
      float2 ls = {0.f, 0.f};
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t raw[32];
        tmem_ld32_issue(ts + (uint32_t)(32 * c4), raw);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) raw[c] = ((mw[c4] >> c) & 1u) ? raw[c] : 0xFF800000u;  // -inf
#pragma unroll
        for (int c = 0; c < 32; c += 8)
#pragma unroll
          for (int a4 = 0; a4 < 4; ++a4)
            m4[a4] = fmax3(m4[a4], __uint_as_float(raw[c + 2 * a4]), __uint_as_float(raw[c + 2 * a4 + 1]));
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 x = ffma2(make_float2(__uint_as_float(raw[2 * i]), __uint_as_float(raw[2 * i + 1])), qs2, nmq0_2);
          const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));  // 0 where masked
          ls = fadd2(ls, p);
          const __half2 ph = __floats2half2_rn(p.x, p.y);
          pw[16 * c4 + i] = *reinterpret_cast<const uint32_t*>(&ph);
        }
      }
      const float tmax = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
      const bool raise = tmax > m_run + lim;  // also the first selected entry of the row (m_run = -inf)
      if (__any_sync(0xFFFFFFFFu, raise)) {
        float alpha = 1.f;
        bool resc = false;
        if (raise) {
          if (m_run != -INFINITY) {
            alpha = exp2f((m_run - tmax) * qscale);
            l2.x *= alpha;
            l2.y *= alpha;
            resc = true;
          }
          m_run = tmax;
        }
        if (__any_sync(0xFFFFFFFFu, resc)) {  // O holds earlier tiles: rescale it once they are in
          const bool ok2 = __all_sync(0xFFFFFFFFu, mbar_wait_or_abort(bar(B_PFREE + t), (j - 1) & 1, abort_flag));
          if (!ok2) {
            err = true;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c8 = 0; c8 < 16; ++c8) {  // 8 columns at a time: the weights stay in registers
            uint32_t ov[8];
            tmem_ld<8>(to + 8 * c8, ov);
#pragma unroll
            for (int i = 0; i < 8; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st<8>(to + 8 * c8, ov);
          }
        }
        // the weights again, against the raised max (rows whose max did not move get the same values)
        const float nmq = m_run == -INFINITY ? 0.f : -m_run * qscale;
        const float2 nmq2 = {nmq, nmq};
        ls = make_float2(0.f, 0.f);
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t raw[32];
          tmem_ld32_issue(ts + (uint32_t)(32 * c4), raw);
          tmem_wait_ld();
          const uint32_t w = c4 == 0 ? mw[0] : c4 == 1 ? mw[1] : c4 == 2 ? mw[2] : mw[3];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float s0 = ((w >> (2 * i)) & 1u) ? __uint_as_float(raw[2 * i]) : -INFINITY;
            const float s1 = ((w >> (2 * i + 1)) & 1u) ? __uint_as_float(raw[2 * i + 1]) : -INFINITY;
            const float2 x = ffma2(make_float2(s0, s1), qs2, nmq2);
            const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            ls = fadd2(ls, p);
            const __half2 ph = __floats2half2_rn(p.x, p.y);
            raw[i] = *reinterpret_cast<const uint32_t*>(&ph);
          }
          // pw[16 c4 + i] = raw[i]: dynamic indexing of pw would spill it, so the pairs go to tensor
          // memory here and the store below is skipped for this tile
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = raw[i];
          tmem_st16_issue(ts + (uint32_t)(16 * c4), pk);
        }
        l2 = fadd2(l2, ls);
        tmem_wait_st();
      } else {
        l2 = fadd2(l2, ls);
        // weights over the scores: pairs 0-63 into columns 0-63 (all scores have been read)
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = pw[32 * c2 + i];
          tmem_st32_issue(ts + (uint32_t)(32 * c2), pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PREADY + t));
    }
    if (!err && nvt > 0) err = !__all_sync(0xFFFFFFFFu, mbar_wait_or_abort(bar(B_PFREE + t), (nvt - 1) & 1, abort_flag));
    if (!err && nvt > 0) {
      tc_fence_after();
      const float l = l2.x + l2.y;
      const float inv = l > 0.f ? vscale[g] / l : 0.f;  // V entered scaled by 1 / vscale
      uint16_t* orow = o + ((row0 + r) * H + h) * (int64_t)kD;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t ov[32];
        tmem_ld32_issue(to + 32 * c4, ov);
        tmem_wait_ld();
        if (r < nrt) {
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
      if (r < nrt && lse)
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
  if ((int64_t)s.H * ((n_tiles(s.n_q) + 1) / 2) * s.batch >= ((int64_t)1 << 31) || s.Hkv > 65535) return false;
  const double avg_keys = (double)(s.n_kv - s.n_q) + 0.5 * (double)s.n_q;
  return avg_keys <= (double)HISA_ATTN_QT_RATIO * (double)s.k;
}

namespace {
// Workspace of the query-tile path: masks | V in fp16 | per-head max |v| bits | per-head scale.
struct QtileLayout {
  size_t masks, vh, hmax, vscale, total;
};
QtileLayout qtile_layout(const Shape& s) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  QtileLayout L;
  L.masks = 0;
  L.vh = up((size_t)s.batch * (size_t)n_tiles(s.n_q) * (size_t)n_tiles(s.n_kv) * kMaskBytes);
  L.hmax = L.vh + up((size_t)s.batch * s.n_kv * s.Hkv * kD * 2);
  L.vscale = L.hmax + up((size_t)s.Hkv * 4);
  L.total = L.vscale + up((size_t)s.Hkv * 4);
  return L;
}
}  // namespace

size_t sparse_attn_qtile_bytes(const Shape& s) { return qtile_layout(s).total; }

cudaError_t launch_sparse_attn_qtile(const Shape& s, const void* q, const void* k, const void* v,
                                     const int32_t* token_idx, void* o, float* lse, int32_t* status, void* ws,
                                     cudaStream_t st) {
  if (!sparse_attn_qtile_eligible(s)) return cudaErrorNotSupported;
  const QtileLayout L = qtile_layout(s);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint4* m = reinterpret_cast<uint4*>(w + L.masks);
  uint16_t* vh = reinterpret_cast<uint16_t*>(w + L.vh);
  uint32_t* hmax = reinterpret_cast<uint32_t*>(w + L.hmax);
  float* vscale = reinterpret_cast<float*>(w + L.vscale);
  const int64_t rows = (int64_t)s.batch * s.n_kv;
  CUtensorMap mq, mk, mv;
  if (!map_rows_of_head(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, kD, (uint64_t)s.H, (uint64_t)s.n_query, kRows) ||
      !map_rows_of_head(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, kD, (uint64_t)s.Hkv, (uint64_t)rows, kRows) ||
      !map_rows_of_head(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, vh, kD, (uint64_t)s.Hkv, (uint64_t)rows, kRows))
    return cudaErrorNotSupported;
  const int nqt = (int)n_tiles(s.n_q), nkt = (int)n_tiles(s.n_kv);
  attn_mask_kernel<<<dim3((unsigned)nqt, (unsigned)s.batch), kRows, 0, st>>>(token_idx, m, status, s.n_q, s.n_kv, s.k,
                                                                             nqt, nkt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(hmax, 0, (size_t)s.Hkv * 4, st);
  if (e != cudaSuccess) return e;
  const int64_t want = (148 * 8 + s.Hkv - 1) / s.Hkv;  // about eight blocks per SM over all heads
  const int64_t need = (rows + 15) / 16;
  const dim3 vgrid((unsigned)(want < need ? want : need), (unsigned)s.Hkv);
  attn_v_max_kernel<<<vgrid, 256, 0, st>>>(static_cast<const uint16_t*>(v), rows, s.Hkv, hmax);
  attn_v_half_kernel<<<vgrid, 256, 0, st>>>(static_cast<const uint16_t*>(v), vh, rows, s.Hkv, hmax, vscale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = ensure_smem((const void*)sparse_attn_qtile_kernel, kSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (int64_t)s.H * ((nqt + 1) / 2) * s.batch;
  const float qscale = s.scale * 1.4426950408889634f;
  sparse_attn_qtile_kernel<<<(unsigned)grid, kThreads, kSmem, st>>>(mq, mk, mv, m, vscale, static_cast<uint16_t*>(o),
                                                                    lse, status, s.n_q, s.n_kv, s.H, s.Hkv, s.batch,
                                                                    nqt, nkt, qscale);
  return cudaGetLastError();
}

}  // namespace hisa
