// Step 4 on the 5th-generation tensor cores (prefill): token scores of the
// kept blocks.  "北大HISA稀疏注意力机制" section 1.2.2 item 1; QbitAI HISA
// article, "塊內精挑字符".
//
// A kept block is a contiguous B x d_idx tile of k_idx, and 128 consecutive
// queries keep overlapping sets of blocks.  So instead of gathering rows per
// query, a CTA takes a tile of 128 query rows of one sequence and a run of up
// to kRun key blocks at or below the tile's causal limit, and scores every
// block of the run against the whole tile with one group of tcgen05.mma
// (kind::f16, M = 128 rows, N = B, fp32 in TMEM; exact on integer-valued
// inputs).  The CTA is split by role, the roles handing work over through
// mbarriers:
//   * warp 8 (one thread): TMA of the query tile once, then of each key block
//     (B rows, 128-byte swizzle: the K-major UMMA operand) into a ring of
//     2-4 shared-memory stages;
//   * warp 9 (one thread): the MMAs of block b into TMEM accumulator b & 1,
//     once its stage has landed and that accumulator has been read out;
//   * warps 0-7, two groups of four (group g reads accumulator g, so the
//     blocks alternate between the groups): each warp reads its 32 rows back
//     (tcgen05.ld) -- only when one of its queries kept the block -- and
//     writes that query's B order-preserving keys to its slot of the key
//     buffer (0 for tokens after the query).
// With a multi-head indexer the 128 rows are 128 / H queries x H heads and
// the readout applies w_j * max(0, .) and sums a query's rows.  The slot of
// block j in each query's kept list comes from a per-CTA map built by
// scanning the lists once (same acceptance rule as the CUDA-core scorer: in
// range and above every earlier in-range entry).  The CTA holding the first
// run also zero-fills unused slots and flags malformed entries.  With no list
// (the flat indexer) slot = block id.  Waits are bounded (1 s): a role that
// gives up sets status bit 1 and an abort flag the other roles poll.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hisa {
namespace {

constexpr int kEpiWarps = 8;  // two groups of four, one per TMEM accumulator
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kTileQ = 128;
constexpr int kRun = 64;  // key blocks per CTA

// Key stages in flight per CTA (fewer stages, less shared memory: more CTAs per SM).
#ifndef HISA_TS_MAX_STAGES
#define HISA_TS_MAX_STAGES 4
#endif

// Fewest indexer heads (1 = the one-head indexer) for which B = 128 takes the token-major readout.
// Measured on the 64K prefill token stage (row readout / token-major): 1 head 4.0 / 6.2 ms,
// 2 heads 6.3 / 6.5 ms, 4 heads 8.9 / 7.5 ms.
#ifndef HISA_TS_TM_MIN_HEADS
#define HISA_TS_TM_MIN_HEADS 4
#endif

template <int D, int B>
struct TsLayout {
  static constexpr int HALVES = D / 64;
  static constexpr int Q_BYTES = HALVES * kTileQ * 128;
  static constexpr int K_BYTES = HALVES * B * 128;
  static constexpr int MAP_BYTES = kTileQ * kRun * 2;  // int16 [kTileQ][kRun]
  static constexpr int AVAIL = 227 * 1024 - 1024 - Q_BYTES - MAP_BYTES - kTileQ * 4 - 256;
  static constexpr int STAGES = AVAIL / K_BYTES >= HISA_TS_MAX_STAGES ? HISA_TS_MAX_STAGES : AVAIL / K_BYTES;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_BYTES;
  static constexpr int MAP_OFF = K_OFF + STAGES * K_BYTES;
  static constexpr int W_OFF = MAP_OFF + MAP_BYTES;  // fp32 [kTileQ] head weights of the tile rows
  static constexpr int BAR_OFF = W_OFF + kTileQ * 4;
  // mbarriers: q full | accumulator full x 2 | accumulator empty x 2 | K full x S | K empty x S
  static constexpr int B_Q = 0, B_AFULL = 1, B_AEMPTY = 3, B_KFULL = 5, B_KEMPTY = 5 + STAGES;
  static constexpr int NBAR = 5 + 2 * STAGES;
  static constexpr int MISC_OFF = BAR_OFF + 8 * NBAR;  // TMEM base, abort flag
  static constexpr int SMEM = MISC_OFF + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * B;  // two B-column accumulators
  static_assert(STAGES >= 2, "two key stages at least");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(B >> 3) << 17) |
                                    ((uint32_t)(kTileQ >> 4) << 24);
};

using namespace tc;

// HET = 0: TMEM lane = tile row (query, head), columns = the block's tokens.  HET = 8 or 16
// (token-major, B = 128): the MMA operands swap, so TMEM lane = token and columns = tile rows; a
// query's HET heads are then consecutive registers of one thread and a warp's 32 lanes write 32
// consecutive keys of a query.
template <int D, int B, int HET>
__global__ void __launch_bounds__(kThreads, 1)
    token_score_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                          const int32_t* __restrict__ block_idx, int slots, uint32_t* __restrict__ keys,
                          int32_t* __restrict__ status, int64_t n_q, int64_t n_kv, int q_tiles, int runs, int64_t q0,
                          int64_t nq, const float* __restrict__ w_idx, int HI) {
  using L = TsLayout<D, B>;
  constexpr int S = L::STAGES;
  constexpr bool kTokenMajor = HET > 0;
  static_assert(!kTokenMajor || (B == kTileQ && 32 % HET == 0), "token-major readout: B = 128, HET divides 32");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

  // Rows of the tile are (query, indexer head) pairs: QT queries x HE heads.
  const int HE = HI > 0 ? HI : 1;
  const int QT = kTileQ / HE;
  // Tiles are enumerated over the queries of the chunk [q0, q0 + nq).
  const int run = blockIdx.x % runs;
  const int64_t tile_lin = blockIdx.x / runs;
  const int64_t seq_first = q0 / n_q;
  const int64_t tile0 = (q0 % n_q) / QT;      // first tile of the first sequence touched
  const int64_t tile_abs = tile0 + tile_lin;  // tile counted from the first sequence's start
  const int64_t seq = seq_first + tile_abs / q_tiles;
  const int64_t ti = tile_abs % q_tiles;
  const int64_t tq0 = seq * n_q + ti * QT;                     // first global query of the tile
  const int64_t t_lo = max(tq0, q0);
  const int64_t t_hi = min(min(tq0 + QT, (seq + 1) * n_q), q0 + nq);  // exclusive
  if (t_lo >= t_hi) return;
  const int64_t c_max = (n_kv - n_q + (t_hi - 1 - seq * n_q)) / B;
  const int64_t jb0 = (int64_t)run * kRun;
  if (jb0 > c_max) return;
  const int nb = (int)min((int64_t)kRun, c_max + 1 - jb0);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t* sQ = smem + L::Q_OFF;
  uint8_t* sK = smem + L::K_OFF;
  int16_t* smap = reinterpret_cast<int16_t*>(smem + L::MAP_OFF);
  const uint32_t bar0 = smem_u32(smem + L::BAR_OFF);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  auto fail = [&]() {
    *abort_flag = 1;
    if (status) atomicOr(status, kStatusTimeout);
  };

  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(L::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    mbar_init(bar(L::B_Q), 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(L::B_AFULL + a), 1);
      mbar_init(bar(L::B_AEMPTY + a), 4);  // the four warps of group a
    }
    for (int st = 0; st < S; ++st) {
      mbar_init(bar(L::B_KFULL + st), 1);
      mbar_init(bar(L::B_KEMPTY + st), 1);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpTma) {
    // ---------------- producer: the query tile, then the key blocks into the stage ring ----------------
    if (lane == 0) {
      mbar_expect_tx(bar(L::B_Q), (uint32_t)L::Q_BYTES);
      for (int hh = 0; hh < L::HALVES; ++hh)
        tma_load_2d(smem_u32(sQ + hh * kTileQ * 128), &tmap_q, hh * 64, (int)(tq0 * HE), bar(L::B_Q));
      int issued = 0;
      for (int b = 0; b < nb; ++b) {
        const int st = b % S;
        if (!mbar_wait_or_abort(bar(L::B_KEMPTY + st), (uint32_t)(((b / S) & 1) ^ 1), abort_flag)) {
          fail();
          break;
        }
        mbar_expect_tx(bar(L::B_KFULL + st), (uint32_t)L::K_BYTES);
        const int krow = (int)(seq * n_kv + (jb0 + b) * B);
        for (int hh = 0; hh < L::HALVES; ++hh)
          tma_load_2d(smem_u32(sK + st * L::K_BYTES + hh * B * 128), &tmap_k, hh * 64, krow, bar(L::B_KFULL + st));
        issued = b + 1;
      }
      // copies still in flight land before the CTA exits (all of them have, unless a role gave up)
      mbar_wait(bar(L::B_Q), 0);
      for (int b = max(0, issued - S); b < issued; ++b) mbar_wait(bar(L::B_KFULL + b % S), (uint32_t)((b / S) & 1));
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer: block b into accumulator b & 1 ----------------
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
      bool ok = mbar_wait_or_abort(bar(L::B_Q), 0, abort_flag);
      int issued = 0;
      for (int b = 0; b < nb && ok; ++b) {
        const int st = b % S, a = b & 1;
        ok = mbar_wait_or_abort(bar(L::B_KFULL + st), (uint32_t)((b / S) & 1), abort_flag) &&
             mbar_wait_or_abort(bar(L::B_AEMPTY + a), (uint32_t)(((b >> 1) & 1) ^ 1), abort_flag);
        if (!ok) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t acc_col = tmem + (uint32_t)(a * B);
#pragma unroll
        for (int hh = 0; hh < L::HALVES; ++hh) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t qd = desc_kmajor_sw128(q_base + hh * kTileQ * 128 + k * 32);
            const uint64_t kd = desc_kmajor_sw128(k_base + st * L::K_BYTES + hh * B * 128 + k * 32);
            if constexpr (kTokenMajor)
              umma_bf16(acc_col, kd, qd, L::IDESC, (hh | k) ? 1u : 0u);  // D[token][row]
            else
              umma_bf16(acc_col, qd, kd, L::IDESC, (hh | k) ? 1u : 0u);  // D[row][token]
          }
        }
        umma_commit(bar(L::B_KEMPTY + st));  // the stage may be refilled once these MMAs have read it
        umma_commit(bar(L::B_AFULL + a));    // and the accumulator read out
        issued = b + 1;
      }
      if (!ok) fail();
      // every MMA issued has completed before the TMEM is released
      if (issued > 0) mbar_wait(bar(L::B_AFULL + ((issued - 1) & 1)), (uint32_t)(((issued - 1) >> 1) & 1));
    }
  } else {
    // ---------------- readout warps ----------------
    // Slot map of query tid of the tile (threads tid < QT) for blocks jb0 .. jb0+nb-1, stored
    // block-major (smap[jj * kTileQ + query]) so that a warp's 32 queries sit in consecutive halves.
    {
      uint4* m4 = reinterpret_cast<uint4*>(smap);
      for (int i = tid; i < L::MAP_BYTES / 16; i += kEpiWarps * 32) m4[i] = make_uint4(~0u, ~0u, ~0u, ~0u);
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
      const int64_t qrow = tq0 + tid;  // global query id
      const bool row_ok = tid < QT && qrow >= t_lo && qrow < t_hi;
      const int64_t p = n_kv - n_q + (qrow - seq * n_q);
      const int64_t c = p / B;
      uint32_t* krow_keys = keys + (qrow - q0) * (int64_t)slots * B;
      if (row_ok) {
        if (block_idx) {
          const int32_t* lst = block_idx + qrow * slots;
          // the list in batches of 32 entries, loaded together (16-byte loads when aligned)
          const bool vec = ((reinterpret_cast<uintptr_t>(lst) & 15) == 0);
          int mx = -1;
#pragma unroll 1
          for (int r0 = 0; r0 < slots; r0 += 32) {
            int e[32];
            if (vec && r0 + 32 <= slots) {
              const int4* l4 = reinterpret_cast<const int4*>(lst + r0);
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int4 t = l4[u];
                e[4 * u] = t.x;
                e[4 * u + 1] = t.y;
                e[4 * u + 2] = t.z;
                e[4 * u + 3] = t.w;
              }
            } else {
#pragma unroll
              for (int u = 0; u < 32; ++u) e[u] = r0 + u < slots ? lst[r0 + u] : -1;
            }
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int r = r0 + u;
              const int b = e[u];
              const bool in_range = b >= 0 && b <= c;
              const bool ok = in_range && b > mx;
              if (ok && b >= jb0 && b < jb0 + nb) smap[(b - jb0) * kTileQ + tid] = (int16_t)r;
              if (run == 0 && !ok && r < slots) {
                if (b != -1 && status) atomicOr(status, kStatusBadIndex);
                uint4* z = reinterpret_cast<uint4*>(krow_keys + (int64_t)r * B);
                for (int i = 0; i < B / 4; ++i) z[i] = make_uint4(0, 0, 0, 0);
              }
              if (in_range) mx = max(mx, b);
            }
          }
        } else {
          for (int jj = 0; jj < nb; ++jj)
            if (jb0 + jj <= c) smap[jj * kTileQ + tid] = (int16_t)(jb0 + jj);
          if (run == 0) {  // blocks after the query's own block hold no candidate
            for (int64_t r = c + 1; r < slots; ++r) {
              uint4* z = reinterpret_cast<uint4*>(krow_keys + r * B);
              for (int i = 0; i < B / 4; ++i) z[i] = make_uint4(0, 0, 0, 0);
            }
          }
        }
      }
    }
    if constexpr (kTokenMajor) {
      float* wsm = reinterpret_cast<float*>(smem + L::W_OFF);
      if (tid < kTileQ) {
        const int64_t qr = tq0 + tid / HET;
        wsm[tid] = (HI > 0 && qr >= t_lo && qr < t_hi) ? w_idx[qr * HET + tid % HET] : 0.f;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");  // the slot maps are complete

    // This thread's TMEM lane = tile row r: query tq0 + r / HE, indexer head r % HE.
    const int g = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qi = r / HE, head = r % HE;
    const int64_t qrow = tq0 + qi;
    const bool row_ok = qrow >= t_lo && qrow < t_hi;
    const int64_t p = n_kv - n_q + (qrow - seq * n_q);
    uint32_t* krow_keys = keys + (qrow - q0) * (int64_t)slots * B;
    const float wgt = (HI > 0 && row_ok) ? w_idx[qrow * HI + head] : 1.f;
    for (int b = g; b < nb; b += 2) {
      // the warp leaves together (the shuffles and TMEM loads below are warp-wide)
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_or_abort(bar(L::B_AFULL + g), (uint32_t)((b >> 1) & 1), abort_flag))) {
        if (lane == 0) fail();
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if constexpr (kTokenMajor) {
        // lane = token jb * B + quarter * 32 + lane; chunk cc holds queries cc * kQpc .. + kQpc - 1
        constexpr int kQpc = 32 / (HET > 0 ? HET : 1);
        const float* wsm = reinterpret_cast<const float*>(smem + L::W_OFF);
        const int64_t tk = (jb0 + b) * B + quarter * 32 + lane;
#pragma unroll 1
        for (int cc = 0; cc < kTileQ / 32; ++cc) {
          int sl[kQpc];
          bool any = false;
#pragma unroll
          for (int qq = 0; qq < kQpc; ++qq) {
            const int ql = cc * kQpc + qq;
            const int64_t qr = tq0 + ql;
            sl[qq] = (qr >= t_lo && qr < t_hi) ? smap[b * kTileQ + ql] : -1;  // the same in every lane
            any = any || sl[qq] >= 0;
          }
          if (!any) continue;  // warp-uniform
          uint32_t v[32];
          const uint32_t addr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(g * B + cc * 32);
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
              "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
              : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
              : "r"(addr));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int qq = 0; qq < kQpc; ++qq) {
            if (sl[qq] >= 0) {
              const int ql = cc * kQpc + qq;
              const int64_t qr = tq0 + ql;
              float sc = 0.f;
              if (HET == 1 && HI == 0) {
                sc = __uint_as_float(v[qq]);  // the one-head indexer: the plain dot product
              } else {
#pragma unroll
                for (int jh = 0; jh < HET; ++jh)
                  sc = fmaf(wsm[ql * HET + jh], fmaxf(__uint_as_float(v[qq * HET + jh]), 0.f), sc);
              }
              const int64_t pq = n_kv - n_q + (qr - seq * n_q);
              keys[(qr - q0) * (int64_t)slots * B + (int64_t)sl[qq] * B + quarter * 32 + lane] =
                  tk <= pq ? score_key(sc) : 0u;
            }
          }
        }
      } else {
        // rows whose query kept block jb0 + b
        const int slot = row_ok ? smap[b * kTileQ + qi] : -1;
        if (__any_sync(0xFFFFFFFFu, slot >= 0)) {
          const int64_t j = jb0 + b;
          const int64_t tok0 = j * B;
          uint32_t* dst = krow_keys + (int64_t)(slot < 0 ? 0 : slot) * B;
          // lane 0 holds the warp's first query: a block wholly at or before it needs no causal test
          const bool whole = tok0 + B - 1 <= __shfl_sync(0xFFFFFFFFu, p, 0);
          auto chunk = [&](int cc, const uint32_t(&v)[32]) {
            if (HI == 0) {
              if (slot >= 0) {
#pragma unroll
                for (int t = 0; t < 32; t += 4) {
                  uint4 w;
                  w.x = score_key(__uint_as_float(v[t]));
                  w.y = score_key(__uint_as_float(v[t + 1]));
                  w.z = score_key(__uint_as_float(v[t + 2]));
                  w.w = score_key(__uint_as_float(v[t + 3]));
                  if (!whole) {
                    const int64_t tk = tok0 + cc * 32 + t;
                    w.x = tk <= p ? w.x : 0u;
                    w.y = tk + 1 <= p ? w.y : 0u;
                    w.z = tk + 2 <= p ? w.z : 0u;
                    w.w = tk + 3 <= p ? w.w : 0u;
                  }
                  *reinterpret_cast<uint4*>(dst + cc * 32 + t) = w;
                }
              }
            } else {
              // Multi-head score w_j * max(0, q_j . k) per row, summed over the HE rows of a query
              // with a transposing reduction: after it, the lane of head h holds the sums of tokens
              // h * (32 / HE) .. (h + 1) * (32 / HE) - 1 of this chunk.
              float x[32];
#pragma unroll
              for (int t = 0; t < 32; ++t) x[t] = wgt * fmaxf(__uint_as_float(v[t]), 0.f);
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                if ((1 << m) < HE) {  // warp-uniform
                  constexpr int kHalfMax = 16;
                  const int half = 16 >> m;
                  const int o = HE >> (m + 1);
                  const bool up = (head & o) != 0;
#pragma unroll
                  for (int t = 0; t < kHalfMax; ++t) {
                    if (t < half) {
                      const float send = up ? x[t] : x[t + half];
                      const float keep = up ? x[t + half] : x[t];
                      x[t] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
                    }
                  }
                }
              }
              if (slot >= 0) {
                const int n = 32 / HE, t0 = head * n;
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                  if (t < n) {
                    const int64_t tk = tok0 + cc * 32 + t0 + t;
                    dst[cc * 32 + t0 + t] = tk <= p ? score_key(x[t]) : 0u;
                  }
                }
              }
            }
          };
          // 32 columns at a time, the load of the next chunk in flight while this one is converted
          const uint32_t a0 = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(g * B);
          uint32_t va[32], vb[32];
          tmem_ld32_issue(a0, va);
          tmem_wait_ld(va);
#pragma unroll
          for (int cc = 0; cc < B / 32; ++cc) {
            uint32_t(&cur)[32] = (cc & 1) ? vb : va;
            uint32_t(&nxt)[32] = (cc & 1) ? va : vb;
            if (cc + 1 < B / 32) tmem_ld32_issue(a0 + (uint32_t)((cc + 1) * 32), nxt);
            chunk(cc, cur);
            if (cc + 1 < B / 32) tmem_wait_ld(nxt);
          }
        }
      }
      // the accumulator may be overwritten once all four warps of the group have read it
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_AEMPTY + g));
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == kWarpMma) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::TMEM_COLS));
  }
}

template <int D, int B, int HET>
cudaError_t launch_ts(const Shape& s, const void* q_idx, const void* k_idx, const int32_t* block_idx, int slots,
                      uint32_t* keys, int32_t* status, int64_t q0, int64_t nq, cudaStream_t st) {
  using L = TsLayout<D, B>;
  CUtensorMap mq, mk;
  const int HE = s.HI > 0 ? s.HI : 1;
  const int QT = kTileQ / HE;
  if (!map_bf16_sw128(&mq, q_idx, D, (uint64_t)s.n_query * HE, kTileQ)) return cudaErrorNotSupported;
  if (!map_bf16_sw128(&mk, k_idx, D, (uint64_t)s.batch * s.n_kv, B)) return cudaErrorNotSupported;
  auto kern = token_score_tc_kernel<D, B, HET>;
  cudaError_t e = ensure_smem((const void*)kern, L::SMEM);
  if (e != cudaSuccess) return e;
  const int q_tiles = (int)((s.n_q + QT - 1) / QT);
  const int runs = (int)((s.n_blk + kRun - 1) / kRun);
  // tiles from the chunk's first tile to its last
  const int64_t first = (q0 / s.n_q) * q_tiles + (q0 % s.n_q) / QT;
  const int64_t lastq = q0 + nq - 1;
  const int64_t last = (lastq / s.n_q) * q_tiles + (lastq % s.n_q) / QT;
  const int64_t grid = (last - first + 1) * runs;
  if (grid > 0x7FFFFFFFLL) return cudaErrorNotSupported;
  kern<<<(unsigned)grid, kThreads, L::SMEM, st>>>(mq, mk, block_idx, slots, keys, status, s.n_q, s.n_kv, q_tiles,
                                                  runs, q0, nq, s.w_idx, s.HI);
  return cudaGetLastError();
}

}  // namespace

bool token_score_tc_eligible(const Shape& s, int slots) {
  // a query's indexer heads are consecutive rows of a warp: 1, 2, 4, 8 or 16 of them
  const bool heads_ok = s.HI == 0 || (s.HI <= 16 && (s.HI & (s.HI - 1)) == 0);
  return heads_ok && (s.d_idx == 64 || s.d_idx == 128) && (s.B == 32 || s.B == 64 || s.B == 128 || s.B == 256) &&
         s.n_q >= kTileQ && slots < 32767 && s.n_query <= 0x7FFFFFFFLL &&
         (int64_t)s.batch * s.n_kv <= 0x7FFFFFFFLL;
}

cudaError_t launch_token_score_tc(const Shape& s, const void* q_idx, const void* k_idx, const int32_t* block_idx,
                                  int slots, uint32_t* keys, int32_t* status, int64_t q0, int64_t nq, cudaStream_t st) {
  if (!token_score_tc_eligible(s, slots)) return cudaErrorNotSupported;
  // B = 128 with at least HISA_TS_TM_MIN_HEADS indexer heads: token-major readout (a query's
  // heads in one thread, coalesced key stores)
  const int he = s.HI > 0 ? s.HI : 1;
  if (s.B == 128 && he >= HISA_TS_TM_MIN_HEADS) {
#define HISA_TS_TM(DD, HH) \
  if (s.d_idx == DD && he == HH) return launch_ts<DD, 128, HH>(s, q_idx, k_idx, block_idx, slots, keys, status, q0, nq, st);
    HISA_TS_TM(64, 1) HISA_TS_TM(64, 2) HISA_TS_TM(64, 4) HISA_TS_TM(64, 8) HISA_TS_TM(64, 16)
    HISA_TS_TM(128, 1) HISA_TS_TM(128, 2) HISA_TS_TM(128, 4) HISA_TS_TM(128, 8) HISA_TS_TM(128, 16)
#undef HISA_TS_TM
  }
#define HISA_TS_CASE(DD, BB) \
  if (s.d_idx == DD && s.B == BB) return launch_ts<DD, BB, 0>(s, q_idx, k_idx, block_idx, slots, keys, status, q0, nq, st);
  HISA_TS_CASE(64, 32) HISA_TS_CASE(64, 64) HISA_TS_CASE(64, 128) HISA_TS_CASE(64, 256)
  HISA_TS_CASE(128, 32) HISA_TS_CASE(128, 64) HISA_TS_CASE(128, 128) HISA_TS_CASE(128, 256)
#undef HISA_TS_CASE
  return cudaErrorNotSupported;
}

}  // namespace hisa
