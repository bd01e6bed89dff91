// Step 4 on the 5th-generation tensor cores (prefill): token scores of the
// kept blocks.  "北大HISA稀疏注意力机制" section 1.2.2 item 1; QbitAI HISA
// article, "塊內精挑字符".
//
// A kept block is a contiguous B x d_idx tile of k_idx, and 128 consecutive
// queries keep overlapping sets of blocks.  So instead of gathering rows per
// query, a CTA takes a tile of 128 query rows of one sequence and every key
// block that some query of the tile kept (the union of their lists, a bitmap
// built once per tile), and scores each such block against the whole tile
// with one group of tcgen05.mma (kind::f16, M = 128 rows, N = B, fp32 in
// TMEM; exact on integer-valued inputs).  One CTA per tile, the tiles with the
// most visible blocks launched first; the CTA is split by role, the roles
// handing work over through mbarriers:
//   * readout warps 0 .. 4A-1, A groups of four, with A = 4 TMEM
//     accumulators of B columns (A = 2 when B = 256: 512 columns in all);
//     the blocks rotate through the groups; each warp reads its 32 rows back
//     (tcgen05.ld) -- only when one of its queries kept the block -- and
//     writes that query's B order-preserving keys to its slot of the key
//     buffer (0 for tokens after the query);
//   * warp 4A (one thread): TMA of the query tile once, then of each block of
//     the union (B rows, 128-byte swizzle: the K-major UMMA operand) into a
//     ring of 2-4 shared-memory stages;
//   * warp 4A + 1 (one thread): the MMAs of the u-th block into accumulator
//     u % A, once its stage has landed and that accumulator has been read out.
// Four groups keep four readout warps on each scheduler: the readout, not the
// MMA, sets the pace, and more warps hide its TMEM and store latency.
// With a multi-head indexer the 128 rows are 128 / H queries x H heads and
// the readout applies w_j * max(0, .) and sums a query's rows.  Each query's
// list is accepted once per tile (same rule as the CUDA-core scorer: in range
// and above every earlier in-range entry), kept in shared memory as ascending
// (block, slot) pairs, and walked by a cursor as the blocks go by; rejected
// entries are flagged and their slots zero-filled.  With no list (the flat
// indexer) slot = block id.  Waits are bounded (1 s): a role that gives up
// sets status bit 1 and an abort flag the other roles poll.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hisa {
namespace {

constexpr int kTileQ = 128;
constexpr int kListSlots = 96;     // longest kept list a tile holds (longer lists: the CUDA-core scorer)
constexpr int kMaxBlocks = 16384;  // blocks per sequence the tile's bitmap covers

// Key stages in flight per CTA.
#ifndef HISA_TS_MAX_STAGES
#define HISA_TS_MAX_STAGES 4
#endif

// Fewest indexer heads (1 = the one-head indexer) for which B = 128 takes the token-major readout.
// Measured on the 64K prefill token stage (row readout / token-major): 1 head 4.0 / 6.2 ms,
// 2 heads 6.3 / 6.5 ms, 4 heads 8.9 / 7.5 ms.
#ifndef HISA_TS_TM_MIN_HEADS
#define HISA_TS_TM_MIN_HEADS 4
#endif

template <int D, int B, int HET>
struct TsLayout {
  static constexpr int HALVES = D / 64;
  static constexpr int Q_BYTES = HALVES * kTileQ * 128;
  static constexpr int K_BYTES = HALVES * B * 128;
  // TMEM accumulators (B columns each, 512 columns in all) and the readout groups of four warps
  // that read them, one group per accumulator; then the TMA warp and the MMA warp.
  // (the token-major readout keeps two: its register use leaves no room for four groups)
  static constexpr int NACC = HET > 0 ? 2 : (4 * B <= 512 ? 4 : 512 / B);
  static constexpr int EPI_WARPS = 4 * NACC;
  static constexpr int WARP_TMA = EPI_WARPS, WARP_MMA = EPI_WARPS + 1;
  static constexpr int THREADS = (EPI_WARPS + 2) * 32;
  // kept lists, entry = block << 16 | slot, stored [kListSlots + 1][kTileQ] (a sentinel ends each)
  static constexpr int LIST_BYTES = (kListSlots + 1) * kTileQ * 4;
  static constexpr int BITS_BYTES = kMaxBlocks / 8;
  static constexpr int SLOTB_BYTES = 2 * NACC * kTileQ * 4;  // token-major: a group's slot table, 2 buffers
  static constexpr int FIXED = 1024 + Q_BYTES + LIST_BYTES + BITS_BYTES + SLOTB_BYTES + kTileQ * 4 + 512;
  static constexpr int AVAIL = 227 * 1024 - FIXED;
  static constexpr int STAGES = AVAIL / K_BYTES >= HISA_TS_MAX_STAGES ? HISA_TS_MAX_STAGES : AVAIL / K_BYTES;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_BYTES;
  static constexpr int LIST_OFF = K_OFF + STAGES * K_BYTES;
  static constexpr int BITS_OFF = LIST_OFF + LIST_BYTES;
  static constexpr int SLOTB_OFF = BITS_OFF + BITS_BYTES;
  static constexpr int W_OFF = SLOTB_OFF + SLOTB_BYTES;  // fp32 [kTileQ] head weights of the tile rows
  static constexpr int BAR_OFF = W_OFF + kTileQ * 4;
  // mbarriers: q full | accumulator full x NACC | accumulator empty x NACC | K full x S | K empty x S
  static constexpr int B_Q = 0, B_AFULL = 1, B_AEMPTY = 1 + NACC, B_KFULL = 1 + 2 * NACC,
                       B_KEMPTY = B_KFULL + STAGES;
  static constexpr int NBAR = B_KEMPTY + STAGES;
  static constexpr int MISC_OFF = BAR_OFF + 8 * NBAR;  // TMEM base, abort flag
  static constexpr int SMEM = MISC_OFF + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = NACC * B;
  static_assert(STAGES >= 2, "two key stages at least");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(B >> 3) << 17) |
                                    ((uint32_t)(kTileQ >> 4) << 24);
};

using namespace tc;

template <int D, int B, int HET>
__global__ void __launch_bounds__(TsLayout<D, B, HET>::THREADS, 1)
    token_score_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                          const int32_t* __restrict__ block_idx, int slots, uint32_t* __restrict__ keys,
                          int32_t* __restrict__ status, int64_t n_q, int64_t n_kv, int q_tiles, int64_t n_tiles,
                          int64_t q0, int64_t nq, const float* __restrict__ w_idx, int HI, int blk_lo) {
  using L = TsLayout<D, B, HET>;
  constexpr int S = L::STAGES;
  constexpr int NACC = L::NACC, kEpiWarps = L::EPI_WARPS, kWarpTma = L::WARP_TMA, kWarpMma = L::WARP_MMA;
  constexpr bool kTokenMajor = HET > 0;
  static_assert(!kTokenMajor || (B == kTileQ && 32 % HET == 0), "token-major readout: B = 128, HET divides 32");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

  // Rows of the tile are (query, indexer head) pairs: QT queries x HE heads.
  const int HE = HI > 0 ? HI : 1;
  const int QT = kTileQ / HE;
  // One CTA per tile of the chunk [q0, q0 + nq), the last tiles (the most visible blocks) first.
  const int64_t tile_lin = n_tiles - 1 - (int64_t)blockIdx.x;
  const int64_t seq_first = q0 / n_q;
  const int64_t tile0 = (q0 % n_q) / QT;      // first tile of the first sequence touched
  const int64_t tile_abs = tile0 + tile_lin;  // tile counted from the first sequence's start
  const int64_t seq = seq_first + tile_abs / q_tiles;
  const int64_t ti = tile_abs % q_tiles;
  const int64_t tq0 = seq * n_q + ti * QT;                     // first global query of the tile
  const int64_t t_lo = max(tq0, q0);
  const int64_t t_hi = min(min(tq0 + QT, (seq + 1) * n_q), q0 + nq);  // exclusive
  if (t_lo >= t_hi) return;
  const int c_max = (int)((n_kv - n_q + (t_hi - 1 - seq * n_q)) / B);  // last block visible to the tile
  const int nwords = (c_max >> 5) + 1;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t* sQ = smem + L::Q_OFF;
  uint8_t* sK = smem + L::K_OFF;
  uint32_t* lists = reinterpret_cast<uint32_t*>(smem + L::LIST_OFF);
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L::BITS_OFF);
  int32_t* slotb = reinterpret_cast<int32_t*>(smem + L::SLOTB_OFF);
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
    for (int a = 0; a < NACC; ++a) {
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

  if (warp == kWarpTma && lane == 0) {  // the query tile, while the lists are read
    mbar_expect_tx(bar(L::B_Q), (uint32_t)L::Q_BYTES);
    for (int hh = 0; hh < L::HALVES; ++hh)
      tma_load_2d(smem_u32(sQ + hh * kTileQ * 128), &tmap_q, hh * 64, (int)(tq0 * HE), bar(L::B_Q));
  }
  if (warp < kEpiWarps) {
    // ---------------- the kept lists and the tile's block bitmap ----------------
    for (int i = tid; i < nwords; i += kEpiWarps * 32) bits[i] = 0u;
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    if (tid < QT) {
      const int64_t qrow = tq0 + tid;  // global query id
      const bool row_ok = qrow >= t_lo && qrow < t_hi;
      const int64_t p = n_kv - n_q + (qrow - seq * n_q);
      const int64_t c = p / B;
      uint32_t* krow_keys = keys + (qrow - q0) * (int64_t)slots * B;
      int cnt = 0;
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
              for (int uu = 0; uu < 8; ++uu) {
                const int4 t = l4[uu];
                e[4 * uu] = t.x;
                e[4 * uu + 1] = t.y;
                e[4 * uu + 2] = t.z;
                e[4 * uu + 3] = t.w;
              }
            } else {
#pragma unroll
              for (int uu = 0; uu < 32; ++uu) e[uu] = r0 + uu < slots ? lst[r0 + uu] : -1;
            }
#pragma unroll
            for (int uu = 0; uu < 32; ++uu) {
              const int r = r0 + uu;
              const int b = e[uu];
              const bool in_range = b >= 0 && b <= c;
              const bool ok = in_range && b > mx;
              if (ok) {
                lists[cnt * kTileQ + tid] = ((uint32_t)b << 16) | (uint32_t)r;
                ++cnt;
                atomicOr(&bits[b >> 5], 1u << (b & 31));
              } else if (r < slots) {
                if (b != -1 && status) atomicOr(status, kStatusBadIndex);
                uint4* z = reinterpret_cast<uint4*>(krow_keys + (int64_t)r * B);
                for (int i = 0; i < B / 4; ++i) z[i] = make_uint4(0, 0, 0, 0);
              }
              if (in_range) mx = max(mx, b);
            }
          }
        } else {  // slots of the window after the query's own block hold no candidate
          for (int64_t r = max((int64_t)0, c + 1 - blk_lo); r < slots; ++r) {
            uint4* z = reinterpret_cast<uint4*>(krow_keys + r * B);
            for (int i = 0; i < B / 4; ++i) z[i] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      lists[cnt * kTileQ + tid] = 0xFFFF0000u;  // sentinel: above every block
    }
    if (!block_idx) {  // the flat indexer: the window's blocks up to the tile's last
      const int hi = min(c_max, blk_lo + slots - 1);
      for (int i = tid; i < nwords; i += kEpiWarps * 32) {
        const int b0 = 32 * i;
        uint32_t m = 0u;
        if (b0 <= hi && b0 + 31 >= blk_lo) {
          m = 0xFFFFFFFFu;
          if (blk_lo > b0) m &= 0xFFFFFFFFu << (blk_lo - b0);
          if (hi < b0 + 31) m &= 0xFFFFFFFFu >> (b0 + 31 - hi);
        }
        bits[i] = m;
      }
    }
    if constexpr (kTokenMajor) {
      float* wsm = reinterpret_cast<float*>(smem + L::W_OFF);
      if (tid < kTileQ) {
        const int64_t qr = tq0 + tid / HET;
        wsm[tid] = (HI > 0 && qr >= t_lo && qr < t_hi) ? w_idx[qr * HET + tid % HET] : 0.f;
      }
    }
  }
  __syncthreads();  // lists, bitmap and head weights complete

  // the kept block after b (c_max + 1 when none): every role walks the same sequence
  auto next_blk = [&](int b) -> int {
    const int x = b + 1;
    int w = x >> 5;
    if (w >= nwords) return c_max + 1;
    uint32_t m = bits[w] & (0xFFFFFFFFu << (x & 31));
    while (m == 0u) {
      if (++w >= nwords) return c_max + 1;
      m = bits[w];
    }
    return (w << 5) + __ffs(m) - 1;
  };

  if (warp == kWarpTma) {
    // ---------------- producer: the blocks of the union into the stage ring ----------------
    if (lane == 0) {
      int issued = 0, u = 0;
      for (int b = next_blk(-1); b <= c_max; b = next_blk(b), ++u) {
        const int st = u % S;
        if (!mbar_wait_or_abort(bar(L::B_KEMPTY + st), (uint32_t)(((u / S) & 1) ^ 1), abort_flag)) {
          fail();
          break;
        }
        mbar_expect_tx(bar(L::B_KFULL + st), (uint32_t)L::K_BYTES);
        const int krow = (int)(seq * n_kv + (int64_t)b * B);
        for (int hh = 0; hh < L::HALVES; ++hh)
          tma_load_2d(smem_u32(sK + st * L::K_BYTES + hh * B * 128), &tmap_k, hh * 64, krow, bar(L::B_KFULL + st));
        issued = u + 1;
      }
      // copies still in flight land before the CTA exits (all of them have, unless a role gave up)
      mbar_wait(bar(L::B_Q), 0);
      for (int v = max(0, issued - S); v < issued; ++v) mbar_wait(bar(L::B_KFULL + v % S), (uint32_t)((v / S) & 1));
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer: the u-th block into accumulator u % NACC ----------------
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
      bool ok = mbar_wait_or_abort(bar(L::B_Q), 0, abort_flag);
      int issued = 0, u = 0;
      for (int b = next_blk(-1); b <= c_max && ok; b = next_blk(b), ++u) {
        const int st = u % S, a = u % NACC;
        ok = mbar_wait_or_abort(bar(L::B_KFULL + st), (uint32_t)((u / S) & 1), abort_flag) &&
             mbar_wait_or_abort(bar(L::B_AEMPTY + a), (uint32_t)(((u / NACC) & 1) ^ 1), abort_flag);
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
        issued = u + 1;
      }
      if (!ok) fail();
      // every MMA issued has completed before the TMEM is released
      if (issued > 0) mbar_wait(bar(L::B_AFULL + (issued - 1) % NACC), (uint32_t)(((issued - 1) / NACC) & 1));
    }
  } else {
    // ---------------- readout warps ----------------
    // This thread's TMEM lane = tile row r: query tq0 + r / HE, indexer head r % HE.
    const int g = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qi = r / HE, head = r % HE;
    const int64_t qrow = tq0 + qi;
    const bool row_ok = qrow >= t_lo && qrow < t_hi;
    const int64_t p = n_kv - n_q + (qrow - seq * n_q);
    uint32_t* krow_keys = keys + (qrow - q0) * (int64_t)slots * B;
    const float wgt = (HI > 0 && row_ok) ? w_idx[qrow * HI + head] : 1.f;
    // The slot of block b in the kept list of query lq (the row's query; in the token-major
    // readout, query r of the group's table), by a cursor that only moves forward.
    const int lq = kTokenMajor ? r : qi;
    const bool lq_ok = lq < QT && tq0 + lq >= t_lo && tq0 + lq < t_hi;
    const int64_t lq_c = (n_kv - n_q + (tq0 + lq - seq * n_q)) / B;
    int cur = 0;
    uint32_t ent = (lq_ok && block_idx) ? lists[lq] : 0xFFFF0000u;
    auto slot_of = [&](int b) -> int {
      if (!lq_ok) return -1;
      if (!block_idx) return b <= lq_c ? b - blk_lo : -1;
      while ((int)(ent >> 16) < b) {
        ++cur;
        ent = lists[cur * kTileQ + lq];
      }
      return (int)(ent >> 16) == b ? (int)(ent & 0xFFFFu) : -1;
    };
    int u = 0;
    for (int b = next_blk(-1); b <= c_max; b = next_blk(b), ++u) {
      if (u % NACC != g) continue;
      // the warp leaves together (the shuffles and TMEM loads below are warp-wide)
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait_or_abort(bar(L::B_AFULL + g), (uint32_t)((u / NACC) & 1), abort_flag))) {
        if (lane == 0) fail();
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if constexpr (kTokenMajor) {
        // this block's slot of every query of the tile, one query per thread of the group
        int32_t* tbl = slotb + ((u / NACC) & 1) * (NACC * kTileQ) + g * kTileQ;
        tbl[r] = slot_of(b);
        asm volatile("bar.sync %0, %1;" ::"r"(2 + g), "n"(128) : "memory");
        // lane = token jb * B + quarter * 32 + lane; chunk cc holds queries cc * kQpc .. + kQpc - 1
        constexpr int kQpc = 32 / (HET > 0 ? HET : 1);
        const float* wsm = reinterpret_cast<const float*>(smem + L::W_OFF);
        const int64_t tk = (int64_t)b * B + quarter * 32 + lane;
#pragma unroll 1
        for (int cc = 0; cc < kTileQ / 32; ++cc) {
          int sl[kQpc];
          bool any = false;
#pragma unroll
          for (int qq = 0; qq < kQpc; ++qq) {
            const int ql = cc * kQpc + qq;
            const int64_t qr = tq0 + ql;
            sl[qq] = (qr >= t_lo && qr < t_hi) ? tbl[ql] : -1;  // the same in every lane
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
        // rows whose query kept block b
        const int slot = slot_of(b);
        if (__any_sync(0xFFFFFFFFu, slot >= 0)) {
          const int64_t tok0 = (int64_t)b * B;
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
          // 32 columns at a time
          const uint32_t a0 = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(g * B);
#pragma unroll 1
          for (int cc = 0; cc < B / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32_issue(a0 + (uint32_t)(cc * 32), v);
            tmem_wait_ld(v);
            chunk(cc, v);
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
                      uint32_t* keys, int32_t* status, int64_t q0, int64_t nq, cudaStream_t st, int blk_lo) {
  using L = TsLayout<D, B, HET>;
  CUtensorMap mq, mk;
  const int HE = s.HI > 0 ? s.HI : 1;
  const int QT = kTileQ / HE;
  if (!map_bf16_sw128(&mq, q_idx, D, (uint64_t)s.n_query * HE, kTileQ)) return cudaErrorNotSupported;
  if (!map_bf16_sw128(&mk, k_idx, D, (uint64_t)s.batch * s.n_kv, B)) return cudaErrorNotSupported;
  auto kern = token_score_tc_kernel<D, B, HET>;
  cudaError_t e = ensure_smem((const void*)kern, L::SMEM);
  if (e != cudaSuccess) return e;
  const int q_tiles = (int)((s.n_q + QT - 1) / QT);
  // tiles from the chunk's first tile to its last
  const int64_t first = (q0 / s.n_q) * q_tiles + (q0 % s.n_q) / QT;
  const int64_t lastq = q0 + nq - 1;
  const int64_t last = (lastq / s.n_q) * q_tiles + (lastq % s.n_q) / QT;
  const int64_t grid = last - first + 1;
  if (grid > 0x7FFFFFFFLL) return cudaErrorNotSupported;
  kern<<<(unsigned)grid, L::THREADS, L::SMEM, st>>>(mq, mk, block_idx, slots, keys, status, s.n_q, s.n_kv, q_tiles,
                                                  grid, q0, nq, s.w_idx, s.HI, blk_lo);
  return cudaGetLastError();
}

}  // namespace

bool token_score_tc_eligible(const Shape& s, int slots) {
  // a query's indexer heads are consecutive rows of a warp: 1, 2, 4, 8 or 16 of them
  const bool heads_ok = s.HI == 0 || (s.HI <= 16 && (s.HI & (s.HI - 1)) == 0);
  return heads_ok && (s.d_idx == 64 || s.d_idx == 128) && (s.B == 32 || s.B == 64 || s.B == 128 || s.B == 256) &&
         s.n_q >= kTileQ && s.n_blk <= kMaxBlocks && s.n_query <= 0x7FFFFFFFLL &&
         (int64_t)s.batch * s.n_kv <= 0x7FFFFFFFLL;
}

cudaError_t launch_token_score_tc(const Shape& s, const void* q_idx, const void* k_idx, const int32_t* block_idx,
                                  int slots, uint32_t* keys, int32_t* status, int64_t q0, int64_t nq, cudaStream_t st,
                                  int blk_lo) {
  if (!token_score_tc_eligible(s, slots)) return cudaErrorNotSupported;
  if (block_idx && slots > kListSlots) return cudaErrorNotSupported;  // the CUDA-core scorer takes long lists
  // B = 128 with at least HISA_TS_TM_MIN_HEADS indexer heads: token-major readout (a query's
  // heads in one thread, coalesced key stores)
  const int he = s.HI > 0 ? s.HI : 1;
  if (s.B == 128 && he >= HISA_TS_TM_MIN_HEADS) {
#define HISA_TS_TM(DD, HH) \
  if (s.d_idx == DD && he == HH) return launch_ts<DD, 128, HH>(s, q_idx, k_idx, block_idx, slots, keys, status, q0, nq, st, blk_lo);
    HISA_TS_TM(64, 1) HISA_TS_TM(64, 2) HISA_TS_TM(64, 4) HISA_TS_TM(64, 8) HISA_TS_TM(64, 16)
    HISA_TS_TM(128, 1) HISA_TS_TM(128, 2) HISA_TS_TM(128, 4) HISA_TS_TM(128, 8) HISA_TS_TM(128, 16)
#undef HISA_TS_TM
  }
#define HISA_TS_CASE(DD, BB) \
  if (s.d_idx == DD && s.B == BB) return launch_ts<DD, BB, 0>(s, q_idx, k_idx, block_idx, slots, keys, status, q0, nq, st, blk_lo);
  HISA_TS_CASE(64, 32) HISA_TS_CASE(64, 64) HISA_TS_CASE(64, 128) HISA_TS_CASE(64, 256)
  HISA_TS_CASE(128, 32) HISA_TS_CASE(128, 64) HISA_TS_CASE(128, 128) HISA_TS_CASE(128, 256)
#undef HISA_TS_CASE
  return cudaErrorNotSupported;
}

}  // namespace hisa
