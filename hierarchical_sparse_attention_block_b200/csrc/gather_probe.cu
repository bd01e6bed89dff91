// Measurement helper: how fast this GPU moves gathered rows from L2 into
// shared memory with 16-byte cp.async, the copy pattern of the attention
// kernel (sparse_attn.cu) without any of its arithmetic.  The pages have no
// counterpart; it gives the attention kernel a measured ceiling, the way a
// plain copy gives HBM-bound kernels theirs.
//
// Every warp walks tiles of kRows gathers, copies the rows into its own ring
// of kStages shared-memory stages and keeps kStages - 1 tiles in flight; 4
// warps per CTA and 64 KB of shared memory per CTA, one to three CTAs per SM.  The
// row of gather e is the top bits of a multiplicative hash of e (over the
// largest power of two of rows the buffer holds), computed in registers, so
// no index read or division stands between two copies.
#include "common.cuh"
#include "hisa.h"
#include "internal.h"

namespace hisa {
namespace {

constexpr int kWarps = 4, kRows = 16, kStages = 4, kMaxRowBytes = 256;
constexpr int kSmem = kWarps * kStages * kRows * kMaxRowBytes;

template <int CHUNKS>
__global__ void __launch_bounds__(kWarps * 32) gather_probe_kernel(const uint8_t* __restrict__ rows, int row_shift,
                                                                   int64_t n_gathers, uint32_t seed,
                                                                   uint32_t* __restrict__ sink) {
  constexpr int kRowBytes = CHUNKS * 16;
  constexpr int kPerStep = 32 / CHUNKS;  // rows one warp instruction moves
  static_assert(kPerStep <= kRows && kRows % kPerStep == 0, "a copy step stays inside its tile");
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r_lane = lane / CHUNKS, c_lane = lane % CHUNKS;
  uint8_t* wb = smem + warp * kStages * kRows * kMaxRowBytes;
  const int64_t n_tiles = (n_gathers + kRows - 1) / kRows;
  const int64_t step = (int64_t)gridDim.x * kWarps;
  int stage = 0;
  for (int64_t t = blockIdx.x * (int64_t)kWarps + warp; t < n_tiles; t += step) {
#pragma unroll
    for (int r0 = 0; r0 < kRows; r0 += kPerStep) {
      const int r = r0 + r_lane;
      const int64_t e = t * kRows + r;
      const uint32_t row = (uint32_t)((uint64_t)((uint32_t)e * 0x9E3779B1u + seed) >> row_shift);
      cp_async16(wb + (stage * kRows + r) * kMaxRowBytes + c_lane * 16,
                 rows + (int64_t)row * kRowBytes + c_lane * 16, e < n_gathers);
    }
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    stage = stage + 1 == kStages ? 0 : stage + 1;
  }
  cp_async_wait<0>();
  __syncwarp();
  if (lane == 0) atomicAdd(sink, *reinterpret_cast<const uint32_t*>(wb));
}

template <int CHUNKS>
cudaError_t launch_chunks(const void* rows, int row_shift, int64_t n_gathers, uint32_t seed, uint32_t* sink,
                          int ctas_per_sm, cudaStream_t st) {
  auto kern = gather_probe_kernel<CHUNKS>;
  cudaError_t e = ensure_smem((const void*)kern, kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kern<<<(unsigned)(ctas_per_sm * sms), kWarps * 32, kSmem, st>>>(static_cast<const uint8_t*>(rows), row_shift, n_gathers, seed,
                                                        sink);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather_probe(const void* rows, int64_t n_rows, int row_bytes, int64_t n_gathers, uint32_t seed,
                                uint32_t* sink, int ctas_per_sm, cudaStream_t st) {
  int bits = 0;  // rows used: the largest power of two <= n_rows
  while (bits < 31 && ((int64_t)2 << bits) <= n_rows) ++bits;
  const int shift = 32 - bits;  // 32 (one row) leaves row 0
  switch (row_bytes / 16) {
    case 16: return launch_chunks<16>(rows, shift, n_gathers, seed, sink, ctas_per_sm, st);
    case 8: return launch_chunks<8>(rows, shift, n_gathers, seed, sink, ctas_per_sm, st);
    case 4: return launch_chunks<4>(rows, shift, n_gathers, seed, sink, ctas_per_sm, st);
    case 2: return launch_chunks<2>(rows, shift, n_gathers, seed, sink, ctas_per_sm, st);
    default: return cudaErrorInvalidValue;
  }
}

// One warp instruction moves 32 / (row_bytes / 16) rows, at most a tile (kRows): rows of 32 to 256 bytes.
bool gather_probe_row_bytes_ok(int row_bytes) {
  return row_bytes >= 32 && row_bytes <= kMaxRowBytes && row_bytes % 16 == 0 && 32 % (row_bytes / 16) == 0;
}

}  // namespace hisa
