// Step 2 on the 5th-generation tensor cores (prefill): scores = Q_idx x BKᵀ.
// "北大HISA稀疏注意力机制" section 1.2.1 item 2 (block scores with the
// indexer's dot product); QbitAI HISA article, "塊級粗過濾".
//
// One CTA (one warpgroup) per tile of 128 queries x 128 blocks of one
// sequence; tiles entirely above the causal diagonal exit at once.
//   * TMA brings the 128 query rows (bf16, 128-byte swizzle: already the
//     K-major UMMA operand layout) and the 128 fp32 block keys (unswizzled
//     staging) into shared memory, completing on an mbarrier.
//   * The fp32 block keys are split into three bf16 terms,
//     x = hi + mid + lo (each term the bf16 rounding of what is left), and
//     written as three K-major swizzled B operands.  Every product of a bf16
//     query with a bf16 term is exact, so the fp32 accumulation gives the same
//     score as an fp32 dot product up to summation order -- and exactly the
//     same score on integer-valued inputs.
//   * One thread issues 3 x (d_idx / 16) tcgen05.mma (kind::f16, M=N=128,
//     fp32 accumulator in 128 TMEM columns) and commits them to an mbarrier.
//   * Each warp reads its 32 TMEM lanes (= query rows) back with tcgen05.ld
//     and stores the causally visible scores.
// With a multi-head indexer the 128 rows are 128 / H queries x H heads and the
// readout applies w_j * max(0, .) and sums a query's rows: by shuffles for 1
// or 2 heads; for 4, 8 or 16 heads the MMA operands swap (TMEM lane = block,
// columns = rows), so a query's heads are one thread's registers and a warp
// writes 32 consecutive blocks of a query's score row.
// Every wait is bounded (1 s of %globaltimer); a timeout sets status bit 1
// and the CTA skips to releasing its TMEM.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hisa {
namespace {

constexpr int kTcThreads = 128;
constexpr int kTileM = 128;  // queries per tile
constexpr int kTileN = 128;  // blocks per tile

template <int D>
struct TcLayout {
  static constexpr int HALVES = D / 64;                // 128-byte K slices
  static constexpr int A_BYTES = HALVES * kTileM * 128;
  static constexpr int B_PLANE = HALVES * kTileN * 128;
  static constexpr int B_BYTES = 3 * B_PLANE;
  static constexpr int S_BYTES = kTileN * D * 4;       // fp32 block-key staging
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = A_OFF + A_BYTES;
  static constexpr int S_OFF = B_OFF + B_BYTES;
  static constexpr int BAR_OFF = S_OFF + S_BYTES;      // 2 mbarriers + TMEM address
  static constexpr int W_OFF = BAR_OFF + 64;           // fp32 [kTileM] head weights of the tile rows
  static constexpr int SMEM = W_OFF + kTileM * 4 + 1024;  // + slack for 1024-byte alignment
};

using namespace tc;

// kind::f16 instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTileN >> 3) << 17) |
                            ((uint32_t)(kTileM >> 4) << 24);

__device__ __forceinline__ uint32_t bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return (uint32_t)(*reinterpret_cast<uint16_t*>(&h));
}

// HET = 0: TMEM lane = tile row (query, head), columns = blocks.  HET = 4, 8 or 16 (token-major):
// the MMA operands swap, so TMEM lane = block and columns = tile rows; a query's HET heads are then
// consecutive registers of one thread and a warp writes 32 consecutive blocks of a query's row.
template <int D, int HET>
__global__ void __launch_bounds__(kTcThreads, 1)
    block_score_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_bk,
                          float* __restrict__ scores, int32_t* __restrict__ status, int64_t n_q, int64_t n_kv,
                          int B, int64_t n_blk, int q_tiles, int n_tiles, const float* __restrict__ w_idx, int HI) {
  using L = TcLayout<D>;
  // Rows of the tile are (query, indexer head) pairs: QT queries x HE heads.
  const int HE = HI > 0 ? HI : 1;
  const int QT = kTileM / HE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

  const int nt = blockIdx.x % n_tiles;
  const int qt_all = blockIdx.x / n_tiles;
  const int seq = qt_all / q_tiles;
  const int qt = qt_all % q_tiles;
  const int64_t q0 = (int64_t)qt * QT;
  const int64_t q_last = min(q0 + QT, n_q) - 1;
  const int64_t c_max = (n_kv - n_q + q_last) / B;
  const int64_t j0 = (int64_t)nt * kTileN;
  if (j0 > c_max) return;  // whole tile above the causal diagonal

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t* sA = smem + L::A_OFF;
  uint8_t* sB = smem + L::B_OFF;
  const float* sS = reinterpret_cast<const float*>(smem + L::S_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::BAR_OFF + 16);
  const uint32_t bar_tma = smem_u32(&bars[0]), bar_mma = smem_u32(&bars[1]);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)kTileN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_tma));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_mma));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    const uint32_t tx = (uint32_t)(L::A_BYTES + L::S_BYTES);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_tma), "r"(tx) : "memory");
    const int32_t qrow = (int32_t)(((int64_t)seq * n_q + q0) * HE);
#pragma unroll
    for (int h = 0; h < L::HALVES; ++h) {
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
              "r"(smem_u32(sA + h * kTileM * 128)),
          "l"(reinterpret_cast<uint64_t>(&tmap_q)), "r"(h * 64), "r"(qrow), "r"(bar_tma)
          : "memory");
    }
    const int32_t brow = (int32_t)((int64_t)seq * n_blk + j0);
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(sS)),
        "l"(reinterpret_cast<uint64_t>(&tmap_bk)), "r"(0), "r"(brow), "r"(bar_tma)
        : "memory");
  }
  if constexpr (HET > 0) {
    float* wsm = reinterpret_cast<float*>(smem + L::W_OFF);
    const int64_t qr = q0 + tid / HET;
    wsm[tid] = qr < n_q ? w_idx[((int64_t)seq * n_q + qr) * HET + tid % HET] : 0.f;
  }
  bool ok = mbar_wait(bar_tma, 0);
  ok = __syncthreads_and(ok) != 0;

  if (ok) {
    // Split the fp32 block keys into three bf16 terms, each a K-major 128B-swizzled operand.
    // Warp w converts rows w, w+4, ...; lane l handles dimensions 4l..4l+3 of each 128-wide slice.
    for (int r = warp; r < kTileN; r += kTcThreads / 32) {
#pragma unroll
      for (int e0 = 0; e0 < D; e0 += 128) {
        const int e = e0 + 4 * lane;
        if (e >= D) break;
        const float4 x = *reinterpret_cast<const float4*>(sS + r * D + e);
        const float xs[4] = {x.x, x.y, x.z, x.w};
        uint32_t t[3][2];
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          uint32_t hb[2], mb[2], lb[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float v = xs[2 * pr + q];
            hb[q] = bf16_bits(v);
            const float r1 = v - __uint_as_float(hb[q] << 16);
            mb[q] = bf16_bits(r1);
            const float r2 = r1 - __uint_as_float(mb[q] << 16);
            lb[q] = bf16_bits(r2);
          }
          t[0][pr] = hb[0] | (hb[1] << 16);
          t[1][pr] = mb[0] | (mb[1] << 16);
          t[2][pr] = lb[0] | (lb[1] << 16);
        }
        const int half = e / 64;
        const int chunk = (e % 64) / 8;
        const int within = (e % 8) * 2;  // bytes
        const int off = half * kTileN * 128 + r * 128 + ((chunk ^ (r & 7)) * 16) + within;
#pragma unroll
        for (int pl = 0; pl < 3; ++pl)
          *reinterpret_cast<uint2*>(sB + pl * L::B_PLANE + off) = make_uint2(t[pl][0], t[pl][1]);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  if (ok && tid == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    int first = 1;
#pragma unroll
    for (int pl = 0; pl < 3; ++pl) {
#pragma unroll
      for (int h = 0; h < L::HALVES; ++h) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t qd = desc_kmajor_sw128(a0 + h * kTileM * 128 + s * 32);
          const uint64_t kd = desc_kmajor_sw128(b0 + pl * L::B_PLANE + h * kTileN * 128 + s * 32);
          const uint32_t acc = first ? 0u : 1u;
          // D[row][block], or D[block][row] for the token-major readout
          const uint64_t ad = HET > 0 ? kd : qd, bd = HET > 0 ? qd : kd;
          asm volatile(
              "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
              " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
              "l"(ad), "l"(bd), "r"(kIdesc), "r"(acc));
          first = 0;
        }
      }
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_mma)
                 : "memory");
  }
  bool done = ok ? mbar_wait(bar_mma, 0) : false;
  done = __syncthreads_and(done) != 0;
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  ok = done;

  if (ok && HET > 0) {
    // this thread's TMEM lane = block j0 + tid; chunk cc of the columns holds queries cc * kQpc ..
    constexpr int kQpc = 32 / (HET > 0 ? HET : 1);
    const float* wsm = reinterpret_cast<const float*>(smem + L::W_OFF);
    const int64_t j = j0 + tid;
#pragma unroll 1
    for (int cc = 0; cc < kTileM / 32; ++cc) {
      uint32_t v[32];
      const uint32_t addr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cc * 32);
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
          "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
            "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
            "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
            "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
            "=r"(v[30]), "=r"(v[31])
          : "r"(addr));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int qq = 0; qq < kQpc; ++qq) {
        const int ql = cc * kQpc + qq;
        const int64_t qi = q0 + ql;
        if (ql < QT && qi < n_q) {  // the same in every lane
          const int64_t c = (n_kv - n_q + qi) / B;
          if (j <= c) {
            float sc = 0.f;
#pragma unroll
            for (int h = 0; h < (HET > 0 ? HET : 1); ++h)
              sc = fmaf(wsm[ql * HET + h], fmaxf(__uint_as_float(v[qq * HET + h]), 0.f), sc);
            scores[((int64_t)seq * n_q + qi) * n_blk + j] = sc;
          }
        }
      }
    }
  } else if (ok) {
    // this thread's TMEM lane = tile row tid: query q0 + tid / HE (within the sequence), head tid % HE
    const int head = tid % HE;
    const int64_t qi = q0 + tid / HE;
    const bool row_ok = tid / HE < QT && qi < n_q;
    const int64_t c = row_ok ? (n_kv - n_q + qi) / B : -1;
    float* out = scores + ((int64_t)seq * n_q + qi) * n_blk;
    const float wgt = (HI > 0 && row_ok) ? w_idx[((int64_t)seq * n_q + qi) * HI + head] : 1.f;
#pragma unroll
    for (int cc = 0; cc < kTileN / 32; ++cc) {
      uint32_t v[32];
      const uint32_t addr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(cc * 32);
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
          "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
            "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
            "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
            "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
            "=r"(v[30]), "=r"(v[31])
          : "r"(addr));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      const int64_t jb = j0 + cc * 32;
      if (HI > 0) {
        // w_j * max(0, q_j . bk) per row, summed over a query's HE rows by a transposing reduction:
        // the lane of head h ends with the scores of blocks jb + h * (32 / HE) .. + 32 / HE - 1.
        float x[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) x[t] = wgt * fmaxf(__uint_as_float(v[t]), 0.f);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          if ((1 << m) < HE) {  // warp-uniform
            const int half = 16 >> m;
            const int o = HE >> (m + 1);
            const bool up = (head & o) != 0;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              if (t < half) {
                const float send = up ? x[t] : x[t + half];
                const float keep = up ? x[t + half] : x[t];
                x[t] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
              }
            }
          }
        }
        const int n = 32 / HE, t0 = head * n;
        if (row_ok) {
#pragma unroll
          for (int t = 0; t < 32; ++t)
            if (t < n && jb + t0 + t <= c) out[jb + t0 + t] = x[t];
        }
      } else if (row_ok && jb <= c) {
        if (jb + 31 <= c && (n_blk & 3) == 0) {  // 16-byte aligned rows only
#pragma unroll
          for (int t = 0; t < 32; t += 4)
            *reinterpret_cast<float4*>(out + jb + t) =
                make_float4(__uint_as_float(v[t]), __uint_as_float(v[t + 1]), __uint_as_float(v[t + 2]),
                            __uint_as_float(v[t + 3]));
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t)
            if (jb + t <= c) out[jb + t] = __uint_as_float(v[t]);
        }
      }
    }
  } else if (tid == 0 && status) {
    atomicOr(status, kStatusTimeout);
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTileN));
  }
}

template <int D>
cudaError_t launch_tc(const Shape& s, const void* q_idx, const float* bk, float* scores, int32_t* status,
                      cudaStream_t st) {
  using L = TcLayout<D>;
  CUtensorMap mq, mb;
  const int HE = s.HI > 0 ? s.HI : 1;
  const int QT = kTileM / HE;
  if (!make_map_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q_idx, D, (uint64_t)s.n_query * HE, 64, kTileM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  if (!make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, bk, D, (uint64_t)s.batch * s.n_blk, D, kTileN,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorNotSupported;
  // 4, 8 or 16 indexer heads: the token-major readout (a query's heads in one thread)
  auto kern = s.HI == 4    ? block_score_tc_kernel<D, 4>
              : s.HI == 8  ? block_score_tc_kernel<D, 8>
              : s.HI == 16 ? block_score_tc_kernel<D, 16>
                           : block_score_tc_kernel<D, 0>;
  cudaError_t e = ensure_smem((const void*)kern, L::SMEM);
  if (e != cudaSuccess) return e;
  const int q_tiles = (int)((s.n_q + QT - 1) / QT);
  const int n_tiles = (int)((s.n_blk + kTileN - 1) / kTileN);
  const int64_t grid = (int64_t)s.batch * q_tiles * n_tiles;
  if (grid > 0x7FFFFFFFLL) return cudaErrorNotSupported;
  kern<<<(unsigned)grid, kTcThreads, L::SMEM, st>>>(mq, mb, scores, status, s.n_q, s.n_kv, s.B, s.n_blk, q_tiles,
                                                    n_tiles, s.w_idx, s.HI);
  return cudaGetLastError();
}

}  // namespace

bool block_score_tc_eligible(const Shape& s) {
  // a query's indexer heads are consecutive rows of a warp: 1, 2, 4, 8 or 16 of them
  const bool heads_ok = s.HI == 0 || (s.HI <= 16 && (s.HI & (s.HI - 1)) == 0);
  return heads_ok && (s.d_idx == 64 || s.d_idx == 128) && s.n_q >= 64 &&
         s.n_query * (s.HI > 0 ? s.HI : 1) <= 0x7FFFFFFFLL &&
         (int64_t)s.batch * s.n_blk <= 0x7FFFFFFFLL;
}

size_t block_score_tc_scratch_bytes(const Shape&) { return 0; }

cudaError_t launch_block_score_tc(const Shape& s, const void* q_idx, const float* block_keys, float* scores,
                                  int32_t* status, cudaStream_t st) {
  if (!block_score_tc_eligible(s)) return cudaErrorNotSupported;
  switch (s.d_idx) {
    case 64: return launch_tc<64>(s, q_idx, block_keys, scores, status, st);
    case 128: return launch_tc<128>(s, q_idx, block_keys, scores, status, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace hisa
