// Step 6: softmax attention of every head over the selected tokens only.
// QbitAI HISA article, "HISA的關鍵優勢在於": the indexer's output keeps the
// original format and the downstream attention is unchanged.
//
// Work item = (head, query, split), heads outermost so that the CTAs running
// at the same time gather from one head's K/V (n_kv * d * 4 B), which the L2
// then serves to many queries.  A CTA has 4 warps; each warp owns every 4th
// tile of 8 list entries and runs its own 4-stage cp.async pipeline (no CTA
// barriers in the main loop).  Per tile: the K and V rows of 8 tokens
// (2 x 8 x d bf16) land in the warp's shared-memory stage; 8 lanes score one
// token (16-byte conflict-free reads, 3 shuffles), the warp updates its
// running max / sum (base-2 online softmax), and every lane accumulates
// d/32 output dimensions.  The four warps' partial states merge through
// shared memory at the end.  Invalid entries are zero-filled and masked.
// When there are few queries (decode) the list is split across CTAs and a
// second kernel merges the partial (max, sum, output) triples.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace hisa {
namespace {

constexpr int kNW = 4;  // warps per CTA
constexpr int kTT = 8;  // list entries per warp tile
constexpr int kNS = 4;  // pipeline stages per warp

template <int D>
struct AttnCfg {
  static constexpr int ROW = D * 2;                   // bytes per K or V row
  static constexpr int CH = D / 8;                    // 16-byte chunks per row
  static constexpr int STAGE = kTT * 2 * ROW;         // K rows then V rows
  static constexpr int IDS = kNS * kTT * 4;           // token ids per stage
  static constexpr int WARP = kNS * STAGE + IDS;      // per-warp bytes
  static constexpr int SMEM = kNW * WARP;
  static constexpr int CPL = CH / 8;                  // chunks per lane in the score
  static constexpr int PV = D / 32;                   // output dims per lane
  static constexpr int TOK_PER_ITER = 32 / (2 * CH);  // tokens copied per warp instruction
};

template <int D>
__global__ void __launch_bounds__(kNW * 32)
    sparse_attn_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                       const uint16_t* __restrict__ v, const int32_t* __restrict__ token_idx,
                       uint16_t* __restrict__ o, float* __restrict__ lse, int32_t* __restrict__ status,
                       float* __restrict__ partial, int64_t n_q, int64_t n_kv, int H, int Hkv, int topk, int splits,
                       float qscale, int64_t n_query) {
  using C = AttnCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_nuse[kNW];

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
  const int32_t* list = token_idx + qg * topk;

  // Entries past the last valid one are skipped.
  int last = -1;
  for (int e = threadIdx.x; e < topk; e += kNW * 32)
    if (list[e] >= 0) last = e;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) last = max(last, __shfl_xor_sync(0xFFFFFFFFu, last, off));
  if (lane == 0) s_nuse[warp] = last;
  __syncthreads();
  int n_use = -1;
#pragma unroll
  for (int w = 0; w < kNW; ++w) n_use = max(n_use, s_nuse[w]);
  n_use += 1;

  int per = (n_use + splits - 1) / splits;
  per = (per + kTT - 1) / kTT * kTT;
  const int e0 = min(split * per, n_use), e1 = min(e0 + per, n_use);
  const int n_tiles = (e1 - e0 + kTT - 1) / kTT;

  // Query fragment for the score: lane `sub` of each 8-lane group holds chunks sub + 8u.
  const int grp = lane >> 3, sub = lane & 7;
  float qf[8 * C::CPL];
  {
    const uint16_t* qrow = q + (qg * H + h) * D;
#pragma unroll
    for (int uu = 0; uu < C::CPL; ++uu) {
      const uint4 w = *reinterpret_cast<const uint4*>(qrow + (sub + 8 * uu) * 8);
      qf[8 * uu + 0] = bf16_lo(w.x) * qscale; qf[8 * uu + 1] = bf16_hi(w.x) * qscale;
      qf[8 * uu + 2] = bf16_lo(w.y) * qscale; qf[8 * uu + 3] = bf16_hi(w.y) * qscale;
      qf[8 * uu + 4] = bf16_lo(w.z) * qscale; qf[8 * uu + 5] = bf16_hi(w.z) * qscale;
      qf[8 * uu + 6] = bf16_lo(w.w) * qscale; qf[8 * uu + 7] = bf16_hi(w.w) * qscale;
    }
  }

  uint8_t* wbuf = smem + warp * C::WARP;
  int32_t* ids = reinterpret_cast<int32_t*>(wbuf + kNS * C::STAGE);
  const int64_t kv_row0 = (int64_t)seq * n_kv;

  // Issue the copies of this warp's j-th tile into stage j % kNS.
  auto issue = [&](int j) {
    const int t = warp + j * kNW;
    if (t < n_tiles) {
      const int stage = j % kNS;
      uint8_t* sbuf = wbuf + stage * C::STAGE;
      const int ebase = e0 + t * kTT;
      int my_tok = -1;
      if (lane < kTT) {
        const int e = ebase + lane;
        if (e < e1) {
          const int tok = list[e];
          const bool ok = tok >= 0 && (int64_t)tok <= p;
          if (!ok && tok != -1 && status) atomicOr(status, kStatusBadIndex);
          my_tok = ok ? tok : -1;
        }
        ids[stage * kTT + lane] = my_tok;
      }
#pragma unroll
      for (int it = 0; it < kTT / C::TOK_PER_ITER; ++it) {
        const int tl = it * C::TOK_PER_ITER + lane / (2 * C::CH);
        const int part = (lane / C::CH) & 1;  // 0 = K, 1 = V
        const int ch = lane % C::CH;
        const int tok = __shfl_sync(0xFFFFFFFFu, my_tok, tl);
        const uint16_t* src = (part ? v : k) + ((kv_row0 + (tok < 0 ? 0 : tok)) * Hkv + g) * D + ch * 8;
        cp_async16(sbuf + part * kTT * C::ROW + tl * C::ROW + ch * 16, src, tok >= 0);
      }
    }
    cp_async_commit();
  };

  float m_run = -INFINITY, l_run = 0.f;
  float acc[C::PV];
#pragma unroll
  for (int e = 0; e < C::PV; ++e) acc[e] = 0.f;

  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kNW - 1) / kNW : 0;
#pragma unroll
  for (int j = 0; j < kNS - 1; ++j) issue(j);
  for (int j = 0; j < my_tiles; ++j) {
    issue(j + kNS - 1);
    cp_async_wait<kNS - 1>();
    __syncwarp();
    const int stage = j % kNS;
    const uint8_t* kb = wbuf + stage * C::STAGE;
    const uint8_t* vb = kb + kTT * C::ROW;
    // scores of tokens grp and 4 + grp
    float sc[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int tl = r * 4 + grp;
      float dot = 0.f;
#pragma unroll
      for (int uu = 0; uu < C::CPL; ++uu) {
        const uint4 w = *reinterpret_cast<const uint4*>(kb + tl * C::ROW + (sub + 8 * uu) * 16);
        const float* qq = qf + 8 * uu;
        dot = fmaf(qq[0], bf16_lo(w.x), dot); dot = fmaf(qq[1], bf16_hi(w.x), dot);
        dot = fmaf(qq[2], bf16_lo(w.y), dot); dot = fmaf(qq[3], bf16_hi(w.y), dot);
        dot = fmaf(qq[4], bf16_lo(w.z), dot); dot = fmaf(qq[5], bf16_hi(w.z), dot);
        dot = fmaf(qq[6], bf16_lo(w.w), dot); dot = fmaf(qq[7], bf16_hi(w.w), dot);
      }
      dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 4);
      dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 2);
      dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 1);
      sc[r] = ids[stage * kTT + tl] >= 0 ? dot : -INFINITY;
    }
    float mt = fmaxf(sc[0], sc[1]);
    mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 8));
    mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 16));
    const float m_new = fmaxf(m_run, mt);
    if (m_new != -INFINITY) {
      const float alpha = exp2f(m_run - m_new);
      const float p0 = exp2f(sc[0] - m_new), p1 = exp2f(sc[1] - m_new);
      float ps = p0 + p1;
      ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 8);
      ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 16);
      l_run = l_run * alpha + ps;
#pragma unroll
      for (int e = 0; e < C::PV; ++e) acc[e] *= alpha;
#pragma unroll
      for (int src = 0; src < 4; ++src) {
        const float pa = __shfl_sync(0xFFFFFFFFu, p0, src * 8);
        const float pb = __shfl_sync(0xFFFFFFFFu, p1, src * 8);
        const uint8_t* va = vb + src * C::ROW + lane * C::PV * 2;
        const uint8_t* vbb = vb + (4 + src) * C::ROW + lane * C::PV * 2;
        if constexpr (C::PV == 4) {
          const uint2 a = *reinterpret_cast<const uint2*>(va);
          const uint2 b = *reinterpret_cast<const uint2*>(vbb);
          acc[0] = fmaf(pa, bf16_lo(a.x), acc[0]); acc[1] = fmaf(pa, bf16_hi(a.x), acc[1]);
          acc[2] = fmaf(pa, bf16_lo(a.y), acc[2]); acc[3] = fmaf(pa, bf16_hi(a.y), acc[3]);
          acc[0] = fmaf(pb, bf16_lo(b.x), acc[0]); acc[1] = fmaf(pb, bf16_hi(b.x), acc[1]);
          acc[2] = fmaf(pb, bf16_lo(b.y), acc[2]); acc[3] = fmaf(pb, bf16_hi(b.y), acc[3]);
        } else {
          const uint32_t a = *reinterpret_cast<const uint32_t*>(va);
          const uint32_t b = *reinterpret_cast<const uint32_t*>(vbb);
          acc[0] = fmaf(pa, bf16_lo(a), acc[0]); acc[1] = fmaf(pa, bf16_hi(a), acc[1]);
          acc[0] = fmaf(pb, bf16_lo(b), acc[0]); acc[1] = fmaf(pb, bf16_hi(b), acc[1]);
        }
      }
      m_run = m_new;
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();

  // Merge the warps' states.
  float* mg = reinterpret_cast<float*>(smem);  // [kNW] max, [kNW] sum, [kNW][D] acc
  if (lane == 0) {
    mg[warp] = m_run;
    mg[kNW + warp] = l_run;
  }
#pragma unroll
  for (int e = 0; e < C::PV; ++e) mg[2 * kNW + warp * D + lane * C::PV + e] = acc[e];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += kNW * 32) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, mg[w]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float f = exp2f(mg[w] - M);
        L = fmaf(mg[kNW + w], f, L);
        O = fmaf(mg[2 * kNW + w * D + d], f, O);
      }
    }
    if (splits == 1) {
      const float out = L > 0.f ? O / L : 0.f;
      __nv_bfloat16 b = __float2bfloat16_rn(out);
      o[(qg * H + h) * D + d] = *reinterpret_cast<uint16_t*>(&b);
      if (d == 0 && lse) lse[qg * H + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    } else {
      float* part = partial + ((qg * H + h) * splits + split) * (D + 2);
      if (d == 0) {
        part[0] = M;
        part[1] = L;
      }
      part[2 + d] = O;
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

template <int D>
cudaError_t launch_d(const Shape& s, const void* q, const void* k, const void* v, const int32_t* token_idx, void* o,
                     float* lse, int32_t* status, int splits, float* partial, cudaStream_t st) {
  using C = AttnCfg<D>;
  auto kern = sparse_attn_kernel<D>;
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
  attn_merge_kernel<D><<<(unsigned)(s.n_query * s.H), D, 0, st>>>(partial, static_cast<uint16_t*>(o), lse, splits);
  return cudaGetLastError();
}

}  // namespace

int attn_pick_splits(const Shape& s) {
  const int64_t units = s.n_query * s.H;
  const int64_t target = 148 * 8;
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

cudaError_t launch_sparse_attn(const Shape& s, const void* q, const void* k, const void* v, const int32_t* token_idx,
                               void* o, float* lse, int32_t* status, int splits, void* partial, cudaStream_t st) {
  float* part = static_cast<float*>(partial);
  switch (s.d) {
    case 64: return launch_d<64>(s, q, k, v, token_idx, o, lse, status, splits, part, st);
    case 128: return launch_d<128>(s, q, k, v, token_idx, o, lse, status, splits, part, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hisa
