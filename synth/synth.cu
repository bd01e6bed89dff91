// Device half of the seeded input generator (the host half is synth/__init__.py).
//
// SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) used as a counter-based stream:
// output i of stream (seed, tensor) is mix64(base + (i + 1) * GAMMA) with
// base = mix64(seed * GAMMA + tensor).  Values are mapped exactly as on the
// host, so both halves produce identical bf16 bit patterns.  Nothing here is
// part of the attention method.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ inline uint64_t stream_base(uint64_t seed, uint32_t tensor) {
  return mix64(seed * kGamma + (uint64_t)tensor);
}

__device__ inline uint16_t bf16_bits_rn(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

__global__ void fill_int_kernel(uint16_t* __restrict__ out, int64_t count, uint64_t base, int64_t start) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t u = mix64(base + (uint64_t)(start + i + 1) * kGamma);
    int v = (int)(((u >> 32) * 9ull) >> 32) - 4;
    out[i] = bf16_bits_rn((float)v);
  }
}

__global__ void fill_normal_kernel(uint16_t* __restrict__ out, int64_t count, uint64_t base, int64_t start) {
  const float scale = __uint_as_float(0x37DDB3D7u);  // fp32(sqrt(3 / (2^32 - 1)))
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t u = mix64(base + (uint64_t)(start + i + 1) * kGamma);
    int64_t s = (int64_t)(u & 0xFFFF) + (int64_t)((u >> 16) & 0xFFFF) + (int64_t)((u >> 32) & 0xFFFF) +
                (int64_t)(u >> 48);
    float c = (float)(s - 131070);  // exact
    out[i] = bf16_bits_rn(__fmul_rn(c, scale));
  }
}

// keys of every token in a needle block: k <- clamp(k + 2 * sign(q_probe), -4, 4)
__global__ void plant_kernel(uint16_t* __restrict__ k_idx, int64_t n_kv, int32_t d_idx, int32_t block,
                             const int32_t* __restrict__ needles, int32_t n_needle,
                             const int8_t* __restrict__ signs) {
  const int seq = blockIdx.y;
  const int nd = blockIdx.x;
  const int64_t t0 = (int64_t)needles[(int64_t)seq * n_needle + nd] * block;
  const int64_t t1 = min(t0 + block, n_kv);
  const int8_t* sg = signs + (int64_t)seq * d_idx;
  for (int64_t e = threadIdx.x; e < (t1 - t0) * d_idx; e += blockDim.x) {
    int64_t t = t0 + e / d_idx;
    int dim = (int)(e % d_idx);
    uint16_t* p = k_idx + ((int64_t)seq * n_kv + t) * d_idx + dim;
    float v = __uint_as_float((uint32_t)(*p) << 16);
    int iv = (int)v + 2 * (int)sg[dim];
    iv = iv < -4 ? -4 : (iv > 4 ? 4 : iv);
    *p = bf16_bits_rn((float)iv);
  }
}

inline int grid_for(int64_t count) {
  int64_t g = (count + 255) / 256;
  return (int)(g < 148 * 32 ? (g < 1 ? 1 : g) : 148 * 32);
}

}  // namespace

extern "C" {

// Fill out[0:count) with outputs [start, start+count) of stream (seed, tensor) mapped to
// integer bf16 values in {-4..4}.  out: device pointer.  Returns a cudaError_t value.
int synth_fill_int_bf16(void* out, int64_t count, uint64_t seed, uint32_t tensor, int64_t start,
                        cudaStream_t stream) {
  if (count <= 0) return 0;
  fill_int_kernel<<<grid_for(count), 256, 0, stream>>>((uint16_t*)out, count, stream_base(seed, tensor), start);
  return (int)cudaGetLastError();
}

// Same, mapped to unit-variance Irwin-Hall bf16 values.
int synth_fill_normal_bf16(void* out, int64_t count, uint64_t seed, uint32_t tensor, int64_t start,
                           cudaStream_t stream) {
  if (count <= 0) return 0;
  fill_normal_kernel<<<grid_for(count), 256, 0, stream>>>((uint16_t*)out, count, stream_base(seed, tensor),
                                                          start);
  return (int)cudaGetLastError();
}

// Apply the needle shift in place.  needles: device int32 [batch][n_needle] block ids in
// [1, n_blk-2]; signs: device int8 [batch][d_idx] in {-1,0,1}.
int synth_plant_needles(void* k_idx, int32_t batch, int64_t n_kv, int32_t d_idx, int32_t block,
                        const int32_t* needles, int32_t n_needle, const int8_t* signs, cudaStream_t stream) {
  if (batch <= 0 || n_needle <= 0) return 0;
  dim3 grid(n_needle, batch);
  plant_kernel<<<grid, 256, 0, stream>>>((uint16_t*)k_idx, n_kv, d_idx, block, needles, n_needle, signs);
  return (int)cudaGetLastError();
}

// Host-side reference of one raw output, for cross-checking the two halves.
uint64_t synth_raw_u64(uint64_t seed, uint32_t tensor, int64_t index) {
  return mix64(stream_base(seed, tensor) + (uint64_t)(index + 1) * kGamma);
}

}  // extern "C"
