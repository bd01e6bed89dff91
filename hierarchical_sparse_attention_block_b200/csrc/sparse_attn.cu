// Step 6: softmax attention of every head over the selected tokens only.
// QbitAI HISA article, "HISA的關鍵優勢在於": the indexer's output keeps the
// original format and the downstream attention is unchanged.
//
// Work item = (head, query, split), heads outermost so that the CTAs running
// at the same time gather from one head's K/V (n_kv * d * 4 B), which the L2
// then serves to many queries.  A CTA has 4 warps; each warp owns every 4th
// tile of 16 list entries and runs its own cp.async pipeline of kStages tiles
// (rows kept 2d-byte aligned, 16-byte chunks XOR-swizzled by row so the
// ldmatrix reads are bank-conflict free; invalid entries are zero-filled and
// masked).  Per tile, on the tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   * scores: [q; q; 0 ...] (16 x d) x K_tileᵀ (d x 8 tokens), twice; the
//     scores of the 16 tokens land in lanes 0-7, laid out exactly as the
//     output MMA wants its B operand, so no shuffles are needed;
//   * base-2 softmax against a running max that is raised (and the state
//     rescaled) only when a score exceeds it by more than 2^8 -- one vote per
//     tile in the common case; per-lane partial row sums;
//   * output: Oᵀ (d x 8) += V_tileᵀ (d x 16, ldmatrix.trans) x Pᵀ (16 x 8),
//     column 0 of Pᵀ = bf16(p), column 1 = bf16(p - bf16(p)), so the two
//     output columns add up to the weights carried to ~16 bits.
// The four warps' (max, sum, output) states merge through shared memory.
// When there are few queries (decode) the list is split across CTAs and a
// second kernel merges the partial states.  Out-of-range entries set bit 0 of
// the status word.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"

// Tile shape of the prefill kernel: list entries per warp tile and pipeline stages.
#ifndef HISA_ATTN_TILE
#define HISA_ATTN_TILE 16
#endif
#ifndef HISA_ATTN_STAGES
#define HISA_ATTN_STAGES 2
#endif

namespace hisa {
namespace {

#ifndef HISA_ATTN_WARPS
#define HISA_ATTN_WARPS 4
#endif
constexpr int kNW = HISA_ATTN_WARPS;  // warps per CTA

template <int D, int TT, int NS>
struct AttnCfg {
  static constexpr int kT = TT;                        // list entries per warp tile (8 or 16)
  static constexpr int kNS = NS;                       // pipeline stages per warp
  static constexpr int ROW = D * 2;                    // bytes of one K or V row
  static constexpr int CH = D / 8;                     // 16-byte chunks per row
  static constexpr int ROWS_PER_ITER = 32 / (2 * CH);  // rows (K and V) moved per warp copy step
  static constexpr int STAGE = 2 * kT * ROW;           // kT K rows, then kT V rows
  static constexpr int KSTEPS = D / 16;                // QK k-steps and PV m-tiles
  static constexpr int WARP = kNS * STAGE;
  static constexpr int IDS_OFF = kNW * WARP;           // token ids of every stage
  static constexpr int MASK_OFF = IDS_OFF + kNW * kNS * kT * 4;
  static constexpr int SMEM = MASK_OFF + kNW * kNS * 4;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// 16-byte global -> shared copy through L2 only; skip == true zero-fills and reads nothing.
__device__ __forceinline__ void cp_async16_u32(uint32_t dst, const void* src, bool skip) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.b32 q, %2, 0;\n cp.async.cg.shared.global [%0], [%1], 16, q;\n}\n" ::"r"(dst),
      "l"(src), "r"((int)skip)
      : "memory");
}

// bf16 pair of the high halves of two fp32 values (truncation), and of their exact remainders
// (rounded to nearest).  x == hi + lo up to the rounding of lo.
__device__ __forceinline__ uint32_t hi_pair(float x0, float x1) {
  return __byte_perm(__float_as_uint(x0), __float_as_uint(x1), 0x7632);
}
__device__ __forceinline__ uint32_t lo_pair(float x0, float x1) {
  const float r0 = x0 - __uint_as_float(__float_as_uint(x0) & 0xFFFF0000u);
  const float r1 = x1 - __uint_as_float(__float_as_uint(x1) & 0xFFFF0000u);
  const __nv_bfloat162 l = __floats2bfloat162_rn(r0, r1);
  return *reinterpret_cast<const uint32_t*>(&l);
}

// Unpredicated 16-byte global -> shared copy through L2 only.
__device__ __forceinline__ void cp_async16_all(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}

// 2^x on the special-function unit (the weights are re-rounded to a bf16 pair right after).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row) x B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Calls f(std::integral_constant<int, I>) for I = B .. E-1 (compile-time loop).
template <int B, int E, class F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (B < E) {
    f(std::integral_constant<int, B>{});
    static_for<B + 1, E>(f);
  }
}

// D (16x8 fp32) += A (16x8 bf16, row) x B (8x8 bf16, col)
__device__ __forceinline__ void mma_bf16_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

template <int D, int TT, int NS, int MINB>
__global__ void __launch_bounds__(kNW * 32, MINB)
    sparse_attn_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                       const uint16_t* __restrict__ v, const int32_t* __restrict__ token_idx,
                       uint16_t* __restrict__ o, float* __restrict__ lse, int32_t* __restrict__ status,
                       float* __restrict__ partial, int64_t n_q, int64_t n_kv, int H, int Hkv, int topk, int splits,
                       float qscale, int64_t n_query) {
  using C = AttnCfg<D, TT, NS>;
  constexpr int kT = C::kT, kNS = C::kNS;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_last[kNW];

  const int64_t u = blockIdx.x;
  const int64_t per_head = n_query * splits;
  const int h = (int)(u / per_head);
  const int64_t rem = u - (int64_t)h * per_head;
  const int64_t qg = rem / splits;
  const int split = (int)(rem - qg * splits);
  const int seq = (int)(qg / n_q);
  const int64_t p = n_kv - n_q + qg % n_q;
  const int g = h / (H / Hkv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int32_t* list = token_idx + qg * topk;

  // One work item per (query, head): entries past the last valid one are skipped.  A list
  // split across CTAs (few queries) is cut at fixed positions; -1 entries are masked.
  int n_use = topk;
  if (splits == 1) {
    int last = -1;
    for (int e = threadIdx.x; e < topk; e += kNW * 32)
      if (list[e] >= 0) last = e;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) last = max(last, __shfl_xor_sync(0xFFFFFFFFu, last, off));
    if (lane == 0) s_last[warp] = last;
    __syncthreads();
    n_use = -1;
#pragma unroll
    for (int w = 0; w < kNW; ++w) n_use = max(n_use, s_last[w]);
    n_use += 1;
  }

  int per = (n_use + splits - 1) / splits;
  per = (per + kT - 1) / kT * kT;
  const int e0 = min(split * per, n_use), e1 = min(e0 + per, n_use);
  const int n_tiles = (e1 - e0 + kT - 1) / kT;
  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kNW - 1) / kNW : 0;

  // q as the A operand of the score MMA, in rows 0 and 1 (rows 2..15 zero), so that the
  // scores land in lanes 0-7, which are the lanes that feed P into the output MMA.
  uint32_t qa[C::KSTEPS][2];
  {
    const uint16_t* qrow = q + (qg * H + h) * D;
#pragma unroll
    for (int s = 0; s < C::KSTEPS; ++s) {
      qa[s][0] = gid < 2 ? *reinterpret_cast<const uint32_t*>(qrow + 16 * s + 2 * tig) : 0u;
      qa[s][1] = gid < 2 ? *reinterpret_cast<const uint32_t*>(qrow + 16 * s + 2 * tig + 8) : 0u;
    }
  }

  // Copies: step i moves rows i*RPI + hi (hi = lane / (2 CH)); lanes [hi*2CH, hi*2CH + CH) copy a
  // K chunk, the next CH lanes a V chunk.  Rows keep their 2d-byte pitch; logical 16-byte chunk c
  // of row r sits at chunk c ^ (r & 7), which keeps the 8-row ldmatrix reads conflict-free.
  uint8_t* wbuf = smem + warp * C::WARP;
  const uint32_t wbase = smem_u32(wbuf);
  const int hi = lane / (2 * C::CH);    // 0 when a step moves one row (d = 128)
  const int part = (lane / C::CH) & 1;  // 0 = K, 1 = V
  const int ch = lane % C::CH;
  const uint16_t* src_base = (part ? v : k) + ((int64_t)seq * n_kv * Hkv + g) * D + ch * 8;
  const uint32_t tok_stride = (uint32_t)(Hkv * D);
  int32_t* ids_s = reinterpret_cast<int32_t*>(smem + C::IDS_OFF) + warp * kNS * kT;
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(smem + C::MASK_OFF) + warp * kNS;
  // destination of this lane's chunk of row (rc + hi) in stage 0, minus rc * ROW, per (rc & 7)
  uint32_t dxo[8];
  {
    const uint32_t lane_base = wbase + (uint32_t)(part * kT * C::ROW + hi * C::ROW);
    const int chx = ch ^ hi;  // (rc + hi) & 7 == (rc & 7) ^ hi for the even rc of two-row steps
#pragma unroll
    for (int x = 0; x < 8; ++x) dxo[x] = lane_base + (uint32_t)((chx ^ x) << 4);
  }

  auto issue = [&](int j, auto stage_c) {
    constexpr int stage = decltype(stage_c)::value;
    const int t = warp + j * kNW;
    if (t < n_tiles) {  // warp-uniform
      // entry ids: lanes l and l + kT (and so on) hold entry l & (kT - 1); invalid -> token 0 + a clear bit
      const int e = e0 + t * kT + (lane & (kT - 1));
      const int tok = e < e1 ? list[e] : -1;
      const bool ok = tok >= 0 && (int64_t)tok <= p;
      const bool bad = tok != -1 && !ok;
      if (__any_sync(0xFFFFFFFFu, bad) && bad && status) atomicOr(status, kStatusBadIndex);
      const uint32_t valid = __ballot_sync(0xFFFFFFFFu, ok) & ((1u << kT) - 1u);
      ids_s[stage * kT + (lane & (kT - 1))] = ok ? tok : 0;
      mask_s[stage] = valid;
      __syncwarp();
      int tk[kT];
#pragma unroll
      for (int i = 0; i < kT; i += 4) {
        const int4 t4 = *reinterpret_cast<const int4*>(ids_s + stage * kT + i);
        tk[i] = t4.x; tk[i + 1] = t4.y; tk[i + 2] = t4.z; tk[i + 3] = t4.w;
      }
      const uint32_t vbits = valid >> hi;
      constexpr uint32_t sofs = (uint32_t)(stage * C::STAGE);
      if (valid == (1u << kT) - 1u) {  // warp-uniform: every entry valid (the common case)
#pragma unroll
        for (int i = 0; i < kT / C::ROWS_PER_ITER; ++i) {
          const int rc = i * C::ROWS_PER_ITER;
          const int tok_r = C::ROWS_PER_ITER == 1 ? tk[rc] : (hi ? tk[rc + 1] : tk[rc]);
          cp_async16_all(dxo[rc & 7] + sofs + (uint32_t)(rc * C::ROW),
                         src_base + (uint64_t)(uint32_t)tok_r * tok_stride);
        }
      } else {
#pragma unroll
        for (int i = 0; i < kT / C::ROWS_PER_ITER; ++i) {
          const int rc = i * C::ROWS_PER_ITER;
          const int tok_r = C::ROWS_PER_ITER == 1 ? tk[rc] : (hi ? tk[rc + 1] : tk[rc]);
          cp_async16_u32(dxo[rc & 7] + sofs + (uint32_t)(rc * C::ROW),
                         src_base + (uint64_t)(uint32_t)tok_r * tok_stride, ((vbits >> rc) & 1u) == 0u);
        }
      }
    }
    cp_async_commit();
  };

  float m_run = -INFINITY, l_part = 0.f;
  float m_lim = -INFINITY, neg_mq = 0.f;  // rescale threshold and -m_run * qscale
  float acc[C::KSTEPS][4];
#pragma unroll
  for (int mt = 0; mt < C::KSTEPS; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

  // ldmatrix row addresses.  Rows keep their 2d-byte pitch; logical 16-byte chunk c of row r
  // sits at chunk c ^ (r & 7).  16-token tiles: lane supplies row (lane & 7) + 8 * (mi >> 1) of
  // logical chunk 2s + (mi & 1) -> stored at 2s ^ y with y = (mi & 1) ^ (lane & 7).  8-token
  // tiles: lane supplies row (lane & 7) of chunk 2s + mi for an even s, stored at 2s ^ y with
  // y = mi ^ (lane & 7) (no carry: 2s is a multiple of 4).
  const int mi = lane >> 3;
  const uint32_t y16 = kT == 16 ? (uint32_t)(((mi & 1) ^ (lane & 7)) << 4) : (uint32_t)((mi ^ (lane & 7)) << 4);
  const uint32_t a_k = kT == 16 ? (uint32_t)(((lane & 7) + (mi >> 1) * 8) * C::ROW) : (uint32_t)((lane & 7) * C::ROW);
  const uint32_t a_v = kT == 16 ? (uint32_t)((kT + (lane & 7) + (mi >> 1) * 8) * C::ROW)
                                : (uint32_t)((kT + (lane & 7)) * C::ROW);
  uint32_t xs[C::KSTEPS];  // per k-step / m-tile chunk offsets, swizzle applied
#pragma unroll
  for (int s = 0; s < C::KSTEPS; ++s) xs[s] = ((uint32_t)s * 32u) ^ y16;

  // One tile: wait for its copies, then scores, softmax and output on the tensor cores.
  auto compute = [&](auto stage_c) {
    constexpr int stage = decltype(stage_c)::value;
    const uint32_t sb = wbase + stage * C::STAGE;
    const uint32_t sbk = sb + a_k, sbv = sb + a_v;
    constexpr int NSC = kT / 4;  // scores per lane (lanes 0-7)

    // Scores in lanes 0-7: 16-token tiles hold tokens 2tig, 2tig+1, 8+2tig, 9+2tig; 8-token tiles
    // 2tig, 2tig+1.  Even and odd k-steps accumulate separately (shorter MMA chains).
    float sc[NSC];
    {
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, t0[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (kT == 16) {
        float s1[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < C::KSTEPS; s += 2) {
          uint32_t b0, b1, b2, b3, c0, c1, c2, c3;
          ldsm_x4(sbk + xs[s], b0, b1, b2, b3);
          ldsm_x4(sbk + xs[s + 1], c0, c1, c2, c3);
          mma_bf16(s0, qa[s][0], 0u, qa[s][1], 0u, b0, b1);
          mma_bf16(s1, qa[s][0], 0u, qa[s][1], 0u, b2, b3);
          mma_bf16(t0, qa[s + 1][0], 0u, qa[s + 1][1], 0u, c0, c1);
          mma_bf16(t1, qa[s + 1][0], 0u, qa[s + 1][1], 0u, c2, c3);
        }
        const uint32_t valid = gid < 2 ? mask_s[stage] >> (2 * tig) : 0u;
        sc[0] = (valid & 1u) ? s0[0] + t0[0] : -INFINITY;
        sc[1] = (valid & 2u) ? s0[1] + t0[1] : -INFINITY;
        sc[2 % NSC] = (valid & 0x100u) ? s1[0] + t1[0] : -INFINITY;
        sc[3 % NSC] = (valid & 0x200u) ? s1[1] + t1[1] : -INFINITY;
      } else {
#pragma unroll
        for (int s = 0; s < C::KSTEPS; s += 2) {
          uint32_t b0, b1, c0, c1;
          ldsm_x4(sbk + xs[s], b0, b1, c0, c1);
          mma_bf16(s0, qa[s][0], 0u, qa[s][1], 0u, b0, b1);
          mma_bf16(t0, qa[s + 1][0], 0u, qa[s + 1][1], 0u, c0, c1);
        }
        const uint32_t valid = gid < 2 ? mask_s[stage] >> (2 * tig) : 0u;
        sc[0] = (valid & 1u) ? s0[0] + t0[0] : -INFINITY;
        sc[1 % NSC] = (valid & 2u) ? s0[1] + t0[1] : -INFINITY;
      }
    }
    float smax = sc[0];
#pragma unroll
    for (int i = 1; i < NSC; ++i) smax = fmaxf(smax, sc[i]);
    // Scores stay unscaled (q.k); m_run is their running max.  The state is rescaled only when
    // a score passes m_run + 8 / qscale, i.e. when a weight would exceed 2^8.
    if (__any_sync(0xFFFFFFFFu, smax > m_lim)) {
      float tmax = smax;
      tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, 2));
      tmax = __shfl_sync(0xFFFFFFFFu, tmax, 0);
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = exp2f((m_run - m_new) * qscale);
      l_part *= alpha;
#pragma unroll
      for (int mt = 0; mt < C::KSTEPS; ++mt) {
        acc[mt][0] *= alpha;
        acc[mt][1] *= alpha;
        acc[mt][2] *= alpha;
        acc[mt][3] *= alpha;
      }
      m_run = m_new;
      m_lim = m_new + 8.f / qscale;
      neg_mq = -m_new * qscale;
    }
    if (m_run != -INFINITY) {
      float pv[NSC];
#pragma unroll
      for (int i = 0; i < NSC; ++i) pv[i] = fast_exp2(fmaf(sc[i], qscale, neg_mq));  // 0 for masked entries
#pragma unroll
      for (int i = 0; i < NSC; ++i) l_part += pv[i];  // only lanes 0-3 are summed at the end
      // P^T column 0 (lanes 0-3) = p truncated to bf16 (its high half); column 1 (lanes 4-7) =
      // the exact remainder rounded to bf16: together ~16 significant bits.  Other lanes hold 0.
      const uint32_t b0 = gid == 0 ? hi_pair(pv[0], pv[1 % NSC]) : lo_pair(pv[0], pv[1 % NSC]);
      if constexpr (kT == 16) {
        const uint32_t b1 = gid == 0 ? hi_pair(pv[2 % NSC], pv[3 % NSC]) : lo_pair(pv[2 % NSC], pv[3 % NSC]);
#pragma unroll
        for (int mt = 0; mt < C::KSTEPS; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(sbv + xs[mt], a0, a1, a2, a3);
          mma_bf16(acc[mt], a0, a1, a2, a3, b0, b1);
        }
      } else {
#pragma unroll
        for (int mt = 0; mt < C::KSTEPS; mt += 2) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(sbv + xs[mt], a0, a1, a2, a3);
          mma_bf16_k8(acc[mt], a0, a1, b0);
          mma_bf16_k8(acc[mt + 1], a2, a3, b0);
        }
      }
    }
    __syncwarp();
  };

  // Stages cycle with the tile index, so the loop is unrolled by the stage count and every
  // stage offset is a compile-time constant.
  static_for<0, kNS - 1>([&](auto u) { issue(decltype(u)::value, u); });
  for (int j = 0; j < my_tiles; j += kNS) {
    static_for<0, kNS>([&](auto u) {
      constexpr int U = decltype(u)::value;
      if (j + U < my_tiles) {  // warp-uniform
        issue(j + U + kNS - 1, std::integral_constant<int, (U + kNS - 1) % kNS>{});
        cp_async_wait<kNS - 1>();
        __syncwarp();
        compute(u);
      }
    });
  }
  cp_async_wait<0>();
  // per-warp row sum: lanes 0-3 hold partial sums
  l_part += __shfl_xor_sync(0xFFFFFFFFu, l_part, 1);
  l_part += __shfl_xor_sync(0xFFFFFFFFu, l_part, 2);
  __syncthreads();

  // Merge the warps' states: [kNW] max, [kNW] sum, [kNW][D] output.
  float* mg = reinterpret_cast<float*>(smem);
  if (lane == 0) {
    mg[warp] = m_run * qscale;  // == -neg_mq: the offset the weights were taken against
    mg[kNW + warp] = l_part;
  }
  if (tig == 0) {
#pragma unroll
    for (int mtile = 0; mtile < C::KSTEPS; ++mtile) {
      mg[2 * kNW + warp * D + 16 * mtile + gid] = acc[mtile][0] + acc[mtile][1];
      mg[2 * kNW + warp * D + 16 * mtile + gid + 8] = acc[mtile][2] + acc[mtile][3];
    }
  }
  __syncthreads();
  for (int dd = threadIdx.x; dd < D; dd += kNW * 32) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, mg[w]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float f = exp2f(mg[w] - M);
        L = fmaf(mg[kNW + w], f, L);
        O = fmaf(mg[2 * kNW + w * D + dd], f, O);
      }
    }
    if (splits == 1) {
      const float out = L > 0.f ? O / L : 0.f;
      __nv_bfloat16 b = __float2bfloat16_rn(out);
      o[(qg * H + h) * D + dd] = *reinterpret_cast<uint16_t*>(&b);
      if (dd == 0 && lse) lse[qg * H + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    } else {
      float* pt = partial + ((qg * H + h) * splits + split) * (D + 2);
      if (dd == 0) {
        pt[0] = M;
        pt[1] = L;
      }
      pt[2 + dd] = O;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) attn_merge_kernel(const float* __restrict__ partial, uint16_t* __restrict__ o,
                                                       float* __restrict__ lse, int splits) {
  const int64_t row = blockIdx.x;  // qg * H + h
  const float* part = partial + row * splits * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, part[s * (D + 2)]);
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float f = exp2f(part[s * (D + 2)] - M);
      L = fmaf(part[s * (D + 2) + 1], f, L);
      O = fmaf(part[s * (D + 2) + 2 + threadIdx.x], f, O);
    }
  }
  const float out = L > 0.f ? O / L : 0.f;
  __nv_bfloat16 b = __float2bfloat16_rn(out);
  o[row * D + threadIdx.x] = *reinterpret_cast<uint16_t*>(&b);
  if (threadIdx.x == 0 && lse) lse[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

#ifndef HISA_ATTN_SPLIT_STAGES
#define HISA_ATTN_SPLIT_STAGES 2
#endif

template <int D, int TT, int NS>
cudaError_t launch_tiled(const Shape& s, const void* q, const void* k, const void* v, const int32_t* token_idx,
                         void* o, float* lse, int32_t* status, int splits, float* partial, cudaStream_t st) {
  constexpr int MINB = TT == 8 ? 4 : 1;
  using C = AttnCfg<D, TT, NS>;
  auto kern = sparse_attn_kernel<D, TT, NS, MINB>;
  cudaError_t e = ensure_smem((const void*)kern, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t grid = s.n_query * s.H * splits;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  const float qscale = s.scale * 1.4426950408889634f;
  kern<<<(unsigned)grid, kNW * 32, C::SMEM, st>>>(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), token_idx,
      static_cast<uint16_t*>(o), lse, status, partial, s.n_q, s.n_kv, s.H, s.Hkv, s.k, splits, qscale, s.n_query);
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  return launch_attn_merge(s, partial, o, lse, splits, st);
}

// One work item per (query, head) (prefill) or lists split across CTAs (decode).
template <int D>
cudaError_t launch_d(const Shape& s, const void* q, const void* k, const void* v, const int32_t* token_idx, void* o,
                     float* lse, int32_t* status, int splits, float* partial, cudaStream_t st) {
  if (splits > 1)
    return launch_tiled<D, 16, HISA_ATTN_SPLIT_STAGES>(s, q, k, v, token_idx, o, lse, status, splits, partial, st);
  return launch_tiled<D, HISA_ATTN_TILE, HISA_ATTN_STAGES>(s, q, k, v, token_idx, o, lse, status, splits, partial, st);
}

}  // namespace

#ifndef HISA_ATTN_SPLIT_TARGET
#define HISA_ATTN_SPLIT_TARGET (148 * 8)
#endif

int attn_pick_splits(const Shape& s) {
  if (sparse_attn_tc_eligible(s)) {
    // Persistent CTAs, one per SM, each taking the heads of one KV group at a time: about two
    // items per CTA, every split at least two tiles of 128 entries.
    const int G = s.H / s.Hkv;
    const int64_t units = s.n_query * s.Hkv * ((G + 15) / 16);
    const int64_t target = 2 * 148;
    if (units >= target) return 1;
    int64_t sp = (target + units - 1) / units;
    const int64_t max_sp = (s.k + 255) / 256;
    if (sp > max_sp) sp = max_sp;
    return sp < 1 ? 1 : (int)sp;
  }
  const int64_t units = s.n_query * s.H;
  const int64_t target = HISA_ATTN_SPLIT_TARGET;
  if (units >= target) return 1;
  int64_t sp = (target + units - 1) / units;
  const int64_t max_sp = (s.k + 127) / 128;  // keep >= ~128 entries per split
  if (sp > max_sp) sp = max_sp;
  return sp < 1 ? 1 : (int)sp;
}

size_t attn_partial_bytes(const Shape& s, int splits) {
  if (splits <= 1) return 0;
  return (size_t)s.n_query * s.H * splits * (s.d + 2) * sizeof(float);
}

cudaError_t launch_attn_merge(const Shape& s, const float* partial, void* o, float* lse, int splits, cudaStream_t st) {
  switch (s.d) {
    case 64:
      attn_merge_kernel<64><<<(unsigned)(s.n_query * s.H), 64, 0, st>>>(partial, static_cast<uint16_t*>(o), lse, splits);
      break;
    case 128:
      attn_merge_kernel<128><<<(unsigned)(s.n_query * s.H), 128, 0, st>>>(partial, static_cast<uint16_t*>(o), lse,
                                                                          splits);
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

size_t attn_workspace_bytes(const Shape& s) {
  const size_t part = attn_partial_bytes(s, attn_pick_splits(s));
  const size_t masks = sparse_attn_qtile_eligible(s) ? sparse_attn_qtile_bytes(s) : 0;
  return part > masks ? part : masks;
}

cudaError_t launch_sparse_attn(const Shape& s, const void* q, const void* k, const void* v, const int32_t* token_idx,
                               void* o, float* lse, int32_t* status, void* ws, size_t ws_bytes, cudaStream_t st) {
  // Many queries per sequence: tiles of queries against tiles of keys.
  if (ws && sparse_attn_qtile_eligible(s) && ws_bytes >= sparse_attn_qtile_bytes(s)) {
    const cudaError_t e = launch_sparse_attn_qtile(s, q, k, v, token_idx, o, lse, status, ws, st);
    if (e != cudaErrorNotSupported) return e;
  }
  int splits = attn_pick_splits(s);
  if (splits > 1 && (!ws || ws_bytes < attn_partial_bytes(s, splits))) splits = 1;
  float* part = static_cast<float*>(ws);
  // Heads sharing K/V (GQA/MQA): the tensor-core kernel takes a KV group's heads together.
  if (sparse_attn_tc_eligible(s)) {
    const cudaError_t e = launch_sparse_attn_tc(s, q, k, v, token_idx, o, lse, status, splits, part, st);
    if (e != cudaErrorNotSupported) return e;
  }
  switch (s.d) {
    case 64: return launch_d<64>(s, q, k, v, token_idx, o, lse, status, splits, part, st);
    case 128: return launch_d<128>(s, q, k, v, token_idx, o, lse, status, splits, part, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hisa
