// hisa_token_topk_noalloc: the token stage (steps 4-5) for callers that
// cannot allocate device memory.
//
// Some callers only ever hand a library the buffers they already own: an
// inference engine that plans all of its device memory up front and gives
// plugins no allocator, code that must not make a (synchronizing) cudaMalloc
// call in a latency-critical loop, or a host language binding that can pass
// pointers but not manage a scratch buffer's lifetime.  hisa_token_topk needs
// a caller workspace for the candidate keys; this variant needs none.  Its
// scratch is a fixed, file-scope device array of kNoAllocScratchBytes that
// every GPU which loads this part of the library holds until the process
// exits.  Queries are processed in chunks that fit the array, so any size is
// accepted as long as ONE query's candidates (top_m * block keys of 4 bytes)
// fit; larger requests are rejected with HISA_ERR_UNSUPPORTED.
//
// Set-up: the first call on each device looks up the array's device address
// (cudaGetSymbolAddress, with that device current) and keeps it together with
// the id of the device's current context; make that first call before any
// stream capture.  A later call checks the context id (two driver queries, no
// synchronization) and looks the address up again only if the context was
// replaced (cudaDeviceReset, or the primary context released and retained
// anew), so the kept address never outlives the context it belongs to.  Every call shares the one array and
// it keeps the last call's contents: nothing in it needs to start at zero,
// because the scoring kernel of a call writes every key that the selection
// kernel of the same call reads.  Calls whose work overlaps on the GPU (other
// streams, other host threads) race on the array; serialize them.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "hisa.h"
#include "internal.h"

namespace hisa {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_token_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];  // id of the context the address belongs to

// Id of the calling thread's current context (unique for the life of the process), 0 if unknown.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device: looked up once per device and
// context (the runtime makes the device's context current first).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = g_scratch_ptr[dev] ? current_context_id() : 0;
  if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_token_scratch);  // also makes the device's primary context current
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace hisa

extern "C" hisa_status_t hisa_token_topk_noalloc(const hisa_params_t* params, const void* q_idx,
                                                 const float* idx_weights, const void* k_idx,
                                                 const int32_t* block_idx, int32_t* token_idx, float* token_scores,
                                                 int32_t* dev_status, cudaStream_t stream) {
  using namespace hisa;
  // Same argument rules as hisa_token_topk.
  size_t one_query = 0, preferred = 0;
  hisa_status_t rc = hisa_token_topk_workspace_size(params, &one_query, &preferred);
  if (rc != HISA_OK) return rc;
  Shape s;
  rc = make_shape(params, true, false, &s);
  if (rc == HISA_OK) rc = set_idx_weights(&s, idx_weights);
  if (rc != HISA_OK) return rc;
  if (one_query > kNoAllocScratchBytes) return HISA_ERR_UNSUPPORTED;
  if (!q_idx || !k_idx || !block_idx || !token_idx) return HISA_ERR_INVALID_ARG;
  const void* ptrs[] = {q_idx, k_idx, block_idx, token_idx};
  for (const void* p : ptrs)
    if (((uintptr_t)p & 15u) != 0) return HISA_ERR_INVALID_ARG;
  if (token_scores && ((uintptr_t)token_scores & 15u) != 0) return HISA_ERR_INVALID_ARG;

  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    g_last_cuda_error = (int32_t)e;
    return HISA_ERR_CUDA;
  }
  // Queries in chunks that fit the array.
  const int64_t chunk = (int64_t)(kNoAllocScratchBytes / one_query);
  uint32_t* keys = static_cast<uint32_t*>(scratch);
  for (int64_t q0 = 0; q0 < s.n_query; q0 += chunk) {
    const int64_t nq = s.n_query - q0 < chunk ? s.n_query - q0 : chunk;
    e = launch_token_score(s, q_idx, k_idx, block_idx, s.m, keys, dev_status, q0, nq, stream);
    if (e == cudaSuccess)
      e = launch_token_select(s, keys, block_idx, s.m, token_idx, token_scores, q0, nq, stream);
    if (e != cudaSuccess) {
      g_last_cuda_error = (int32_t)e;
      return HISA_ERR_CUDA;
    }
  }
  return HISA_OK;
}
