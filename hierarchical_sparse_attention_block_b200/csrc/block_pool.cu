// Step 1: mean-pool every block of B indexer keys into one fp32 block key.
// "北大HISA稀疏注意力机制" section 1.2.1 item 1; QbitAI HISA article, "塊級粗過濾".
//
// One CTA per (block, sequence).  The block's B rows (d_idx bf16 each) are
// streamed once with 16-byte loads that skip L1; each thread accumulates 8
// dimensions over a strided subset of rows in fp32, the row groups are summed
// through shared memory, and the sum is divided by the block's token count
// with one correctly rounded division.  Bound: HBM read of n_kv * d_idx * 2 B.
#include "common.cuh"
#include "internal.h"

namespace hisa {
namespace {

template <int D>
__global__ void __launch_bounds__(256) block_pool_kernel(const uint16_t* __restrict__ k_idx, float* __restrict__ bk,
                                                         int64_t n_kv, int B, int64_t b0, int64_t n_blk) {
  constexpr int NT = 256, CH = D / 8, RG = NT / CH;
  __shared__ float red[RG][D];
  const int64_t j = b0 + blockIdx.x;
  const int seq = blockIdx.y;
  const int64_t t0 = j * (int64_t)B;
  const int cnt = (int)min((int64_t)B, n_kv - t0);
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
  const uint16_t* base = k_idx + ((int64_t)seq * n_kv + t0) * D + ch * 8;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  auto add = [&](const uint4& v) {
    acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
    acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
    acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
    acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
  };
  int r = rg;
  for (; r + 3 * RG < cnt; r += 4 * RG) {
    const uint4 v0 = ld_stream_v4(base + (int64_t)(r)*D);
    const uint4 v1 = ld_stream_v4(base + (int64_t)(r + RG) * D);
    const uint4 v2 = ld_stream_v4(base + (int64_t)(r + 2 * RG) * D);
    const uint4 v3 = ld_stream_v4(base + (int64_t)(r + 3 * RG) * D);
    add(v0); add(v1); add(v2); add(v3);
  }
  for (; r < cnt; r += RG) add(ld_stream_v4(base + (int64_t)r * D));
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][ch * 8 + e] = acc[e];
  __syncthreads();
  for (int e = threadIdx.x; e < D; e += NT) {
    float sum = 0.f;
#pragma unroll 8
    for (int g = 0; g < RG; ++g) sum += red[g][e];
    bk[((int64_t)seq * n_blk + j) * D + e] = __fdiv_rn(sum, (float)cnt);
  }
}

}  // namespace

cudaError_t launch_block_pool(const Shape& s, const void* k_idx, int64_t b0, int64_t b1, float* block_keys,
                              cudaStream_t st) {
  if (b1 <= b0) return cudaSuccess;
  dim3 grid((unsigned)(b1 - b0), (unsigned)s.batch);
  const uint16_t* kp = static_cast<const uint16_t*>(k_idx);
  switch (s.d_idx) {
    case 64: block_pool_kernel<64><<<grid, 256, 0, st>>>(kp, block_keys, s.n_kv, s.B, b0, s.n_blk); break;
    case 128: block_pool_kernel<128><<<grid, 256, 0, st>>>(kp, block_keys, s.n_kv, s.B, b0, s.n_blk); break;
    case 256: block_pool_kernel<256><<<grid, 256, 0, st>>>(kp, block_keys, s.n_kv, s.B, b0, s.n_blk); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace hisa
