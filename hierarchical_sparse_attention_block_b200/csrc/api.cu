// C ABI (include/hisa.h): argument validation, workspace sizing and the
// order of launches.  Every step of the path runs in the kernels of this
// library; this file only checks arguments and enqueues them.
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "hisa.h"
#include "internal.h"

namespace hisa {

thread_local int32_t g_last_cuda_error = 0;

namespace {

hisa_status_t cuda_fail(cudaError_t e) {
  if (e == cudaSuccess) return HISA_OK;
  g_last_cuda_error = (int32_t)e;
  return HISA_ERR_CUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

}  // namespace

// Validation shared by every call.  need_attn: the attention fields matter.
hisa_status_t make_shape(const hisa_params_t* p, bool need_indexer, bool need_attn, Shape* s) {
  if (!p) return HISA_ERR_INVALID_ARG;
  if (p->flags != 0) return HISA_ERR_INVALID_ARG;
  if (p->batch < 1 || p->batch > 65535) return HISA_ERR_INVALID_ARG;
  if (p->n_kv < 1 || p->n_kv > 0x7FFFFFFFLL) return HISA_ERR_INVALID_ARG;
  if (p->n_q < 1 || p->n_q > p->n_kv) return HISA_ERR_INVALID_ARG;
  if (p->top_k < 1) return HISA_ERR_INVALID_ARG;
  s->batch = p->batch;
  s->n_q = p->n_q;
  s->n_kv = p->n_kv;
  s->d_idx = p->d_idx;
  s->B = p->block;
  s->m = p->top_m;
  s->k = p->top_k;
  s->H = p->n_heads;
  s->Hkv = p->n_kv_heads;
  s->d = p->d_head;
  s->n_query = (int64_t)p->batch * p->n_q;
  if (need_indexer) {
    if (p->block < 1 || !pow2(p->block) || p->block > 4096) return p->block < 1 ? HISA_ERR_INVALID_ARG : HISA_ERR_UNSUPPORTED;
    if (p->top_m < 2) return HISA_ERR_INVALID_ARG;
    if (p->d_idx != 64 && p->d_idx != 128 && p->d_idx != 256) return p->d_idx < 1 ? HISA_ERR_INVALID_ARG : HISA_ERR_UNSUPPORTED;
    s->n_blk = (p->n_kv + p->block - 1) / p->block;
    if ((int64_t)p->top_m * p->block > (int64_t)1 << 24) return HISA_ERR_UNSUPPORTED;
    if (p->n_idx_heads < 0) return HISA_ERR_INVALID_ARG;
    if (p->n_idx_heads > 16) return HISA_ERR_UNSUPPORTED;
    s->HI = p->n_idx_heads;
  } else {
    s->n_blk = p->block >= 1 ? (p->n_kv + p->block - 1) / p->block : 0;
  }
  if (need_attn) {
    if (p->n_heads < 1 || p->n_kv_heads < 1 || p->n_heads % p->n_kv_heads != 0) return HISA_ERR_INVALID_ARG;
    if (p->d_head != 64 && p->d_head != 128) return p->d_head < 1 ? HISA_ERR_INVALID_ARG : HISA_ERR_UNSUPPORTED;
    if (!(p->scale == p->scale) || isinf(p->scale)) return HISA_ERR_INVALID_ARG;
    s->scale = p->scale > 0.f ? p->scale : (float)(1.0 / sqrt((double)p->d_head));
  } else {
    s->scale = 0.f;
  }
  return HISA_OK;
}

hisa_status_t set_idx_weights(Shape* s, const float* idx_weights) {
  if ((s->HI == 0) != (idx_weights == nullptr)) return HISA_ERR_INVALID_ARG;
  if (idx_weights && ((uintptr_t)idx_weights & 3u) != 0) return HISA_ERR_INVALID_ARG;
  s->w_idx = idx_weights;
  return HISA_OK;
}

namespace {

size_t topm_ws(const Shape& s) {
  size_t b = align_up((size_t)s.n_query * s.n_blk * sizeof(float));
  if (block_score_tc_eligible(s)) b += align_up(block_score_tc_scratch_bytes(s));
  return b;
}

size_t token_keys_per_query(const Shape& s, int slots) { return (size_t)slots * s.B * sizeof(uint32_t); }

constexpr size_t kKeysCap = (size_t)4 << 30;  // preferred key buffer cap: 4 GiB

size_t keys_preferred(const Shape& s, int slots) {
  const size_t per = token_keys_per_query(s, slots);
  const size_t all = per * (size_t)s.n_query;
  if (all <= kKeysCap) return all;
  size_t nq = kKeysCap / per;
  if (nq < 1) nq = 1;
  return nq * per;
}

// Token stage over all queries, in as few chunks as the key buffer allows.
hisa_status_t run_token_stage(const Shape& s, const void* q_idx, const void* k_idx, const int32_t* block_idx,
                              int slots, int32_t* token_idx, float* token_scores, int32_t* status, void* keys_buf,
                              size_t keys_bytes, cudaStream_t st) {
  const size_t per = token_keys_per_query(s, slots);
  const int64_t chunk = (int64_t)(keys_bytes / per);
  if (chunk < 1) return HISA_ERR_WORKSPACE;
  uint32_t* keys = static_cast<uint32_t*>(keys_buf);
  for (int64_t q0 = 0; q0 < s.n_query; q0 += chunk) {
    const int64_t nq = s.n_query - q0 < chunk ? s.n_query - q0 : chunk;
    cudaError_t e = launch_token_score(s, q_idx, k_idx, block_idx, slots, keys, status, q0, nq, st);
    if (e == cudaSuccess) e = launch_token_select(s, keys, block_idx, slots, token_idx, token_scores, q0, nq, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return HISA_OK;
}

hisa_status_t run_block_stage(const Shape& s, const void* q_idx, const float* block_keys, int32_t* block_idx,
                              float* block_scores, int32_t* status, void* ws, cudaStream_t st) {
  float* scores = static_cast<float*>(ws);
  cudaError_t e = cudaErrorNotSupported;
  if (block_score_tc_eligible(s)) e = launch_block_score_tc(s, q_idx, block_keys, scores, status, st);
  if (e == cudaErrorNotSupported) e = launch_block_score(s, q_idx, block_keys, scores, st);
  if (e == cudaSuccess) e = launch_block_topm(s, scores, block_idx, block_scores, st);
  return cuda_fail(e);
}

}  // namespace

cudaError_t ensure_smem(const void* func, int bytes, int static_bytes) {
  if (bytes + static_bytes <= 48 * 1024) return cudaSuccess;  // within the default limit
  static std::mutex mu;
  static const void* done_f[64][64];
  static int done_b[64][64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64) {
    for (int i = 0; i < 64; ++i)
      if (done_f[dev][i] == func && done_b[dev][i] >= bytes) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) {
    for (int i = 0; i < 64; ++i) {
      if (done_f[dev][i] == nullptr || done_f[dev][i] == func) {
        done_f[dev][i] = func;
        done_b[dev][i] = bytes;
        break;
      }
    }
  }
  return cudaSuccess;
}

}  // namespace hisa

using hisa::Shape;

extern "C" {

const char* hisa_status_string(hisa_status_t status) {
  switch (status) {
    case HISA_OK: return "ok";
    case HISA_ERR_INVALID_ARG: return "invalid argument";
    case HISA_ERR_UNSUPPORTED: return "unsupported size";
    case HISA_ERR_WORKSPACE: return "workspace missing or too small";
    case HISA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

int32_t hisa_last_cuda_error(void) { return hisa::g_last_cuda_error; }

const char* hisa_version(void) { return "hisa-b200 0.1.0"; }

hisa_status_t hisa_block_pool(const hisa_params_t* params, const void* k_idx, int64_t blk_begin, int64_t blk_end,
                              float* block_keys, cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, false, &s);
  if (rc != HISA_OK) return rc;
  if (!k_idx || !block_keys || !hisa::aligned16(k_idx) || !hisa::aligned16(block_keys)) return HISA_ERR_INVALID_ARG;
  if (blk_end < 0) blk_end = s.n_blk;
  if (blk_begin < 0 || blk_begin > blk_end || blk_end > s.n_blk) return HISA_ERR_INVALID_ARG;
  return hisa::cuda_fail(hisa::launch_block_pool(s, k_idx, blk_begin, blk_end, block_keys, stream));
}

hisa_status_t hisa_block_topm_workspace_size(const hisa_params_t* params, size_t* bytes) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, false, &s);
  if (rc != HISA_OK) return rc;
  if (!bytes) return HISA_ERR_INVALID_ARG;
  *bytes = hisa::topm_ws(s);
  return HISA_OK;
}

hisa_status_t hisa_block_topm(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                              const float* block_keys, int32_t* block_idx, float* block_scores, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, false, &s);
  if (rc == HISA_OK) rc = hisa::set_idx_weights(&s, idx_weights);
  if (rc != HISA_OK) return rc;
  if (!q_idx || !block_keys || !block_idx) return HISA_ERR_INVALID_ARG;
  if (!hisa::aligned16(q_idx) || !hisa::aligned16(block_keys) || !hisa::aligned16(block_idx)) return HISA_ERR_INVALID_ARG;
  if (block_scores && !hisa::aligned16(block_scores)) return HISA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < hisa::topm_ws(s) || !hisa::aligned16(workspace)) return HISA_ERR_WORKSPACE;
  return hisa::run_block_stage(s, q_idx, block_keys, block_idx, block_scores, dev_status, workspace, stream);
}

hisa_status_t hisa_token_topk_workspace_size(const hisa_params_t* params, size_t* min_bytes, size_t* preferred_bytes) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, false, &s);
  if (rc != HISA_OK) return rc;
  if (!min_bytes && !preferred_bytes) return HISA_ERR_INVALID_ARG;
  if (min_bytes) *min_bytes = hisa::token_keys_per_query(s, s.m);
  if (preferred_bytes) *preferred_bytes = hisa::keys_preferred(s, s.m);
  return HISA_OK;
}

hisa_status_t hisa_token_topk(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                              const void* k_idx, const int32_t* block_idx, int32_t* token_idx, float* token_scores,
                              int32_t* dev_status, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, false, &s);
  if (rc == HISA_OK) rc = hisa::set_idx_weights(&s, idx_weights);
  if (rc != HISA_OK) return rc;
  if (!q_idx || !k_idx || !block_idx || !token_idx) return HISA_ERR_INVALID_ARG;
  if (!hisa::aligned16(q_idx) || !hisa::aligned16(k_idx) || !hisa::aligned16(block_idx) || !hisa::aligned16(token_idx))
    return HISA_ERR_INVALID_ARG;
  if (token_scores && !hisa::aligned16(token_scores)) return HISA_ERR_INVALID_ARG;
  if (!workspace || !hisa::aligned16(workspace)) return HISA_ERR_WORKSPACE;
  return hisa::run_token_stage(s, q_idx, k_idx, block_idx, s.m, token_idx, token_scores, dev_status, workspace,
                               workspace_bytes, stream);
}

hisa_status_t hisa_sparse_attn_workspace_size(const hisa_params_t* params, size_t* bytes) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, false, true, &s);
  if (rc != HISA_OK) return rc;
  if (!bytes) return HISA_ERR_INVALID_ARG;
  *bytes = hisa::attn_workspace_bytes(s);
  return HISA_OK;
}

hisa_status_t sparse_attn_fwd(const hisa_params_t* params, const void* q, const void* k, const void* v,
                              const int32_t* token_idx, void* o, float* lse, int32_t* dev_status, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, false, true, &s);
  if (rc != HISA_OK) return rc;
  if (!q || !k || !v || !token_idx || !o) return HISA_ERR_INVALID_ARG;
  if (!hisa::aligned16(q) || !hisa::aligned16(k) || !hisa::aligned16(v) || !hisa::aligned16(token_idx) ||
      !hisa::aligned16(o))
    return HISA_ERR_INVALID_ARG;
  if (lse && !hisa::aligned16(lse)) return HISA_ERR_INVALID_ARG;
  if (workspace && !hisa::aligned16(workspace)) return HISA_ERR_WORKSPACE;
  return hisa::cuda_fail(hisa::launch_sparse_attn(s, q, k, v, token_idx, o, lse, dev_status, workspace,
                                                  workspace ? workspace_bytes : 0, stream));
}

hisa_status_t hisa_sparse_attn_kernel(const hisa_params_t* params, size_t workspace_bytes, int32_t* kind) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, false, true, &s);
  if (rc != HISA_OK) return rc;
  if (!kind) return HISA_ERR_INVALID_ARG;
  *kind = hisa::sparse_attn_qtile_eligible(s) && workspace_bytes >= hisa::sparse_attn_qtile_bytes(s) ? 1 : 0;
  return HISA_OK;
}

// Workspace of hisa_forward: block keys | block stage | block_idx | token_idx | attention partials | token keys.
namespace {
struct FwdLayout {
  size_t bk, blk_stage, block_idx, token_idx, attn, keys, total;
};
FwdLayout fwd_layout(const Shape& s) {
  FwdLayout L;
  size_t off = 0;
  L.bk = off;
  off += hisa::align_up((size_t)s.batch * s.n_blk * s.d_idx * sizeof(float));
  L.blk_stage = off;
  off += hisa::topm_ws(s);
  L.block_idx = off;
  off += hisa::align_up((size_t)s.n_query * s.m * sizeof(int32_t));
  L.token_idx = off;
  off += hisa::align_up((size_t)s.n_query * s.k * sizeof(int32_t));
  L.attn = off;
  off += hisa::align_up(hisa::attn_workspace_bytes(s));
  L.keys = off;
  off += hisa::align_up(hisa::keys_preferred(s, s.m));
  L.total = off;
  return L;
}
}  // namespace

hisa_status_t hisa_forward_workspace_size(const hisa_params_t* params, size_t* bytes) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, true, &s);
  if (rc != HISA_OK) return rc;
  if (!bytes) return HISA_ERR_INVALID_ARG;
  *bytes = fwd_layout(s).total;
  return HISA_OK;
}

namespace {
// Steps 1-6; block keys in bk, pooled for blocks [refresh_begin, n_blk).
hisa_status_t forward_impl(const Shape& s, const FwdLayout& L, const void* q_idx, const void* k_idx, float* bk,
                           int64_t refresh_begin, const void* q, const void* k, const void* v, void* o, float* lse,
                           int32_t* block_idx_out, int32_t* token_idx_out, int32_t* dev_status, uint8_t* ws,
                           size_t workspace_bytes, cudaStream_t stream) {
  int32_t* blk = block_idx_out ? block_idx_out : reinterpret_cast<int32_t*>(ws + L.block_idx);
  int32_t* tok = token_idx_out ? token_idx_out : reinterpret_cast<int32_t*>(ws + L.token_idx);
  cudaError_t e = hisa::launch_block_pool(s, k_idx, refresh_begin, s.n_blk, bk, stream);
  if (e != cudaSuccess) return hisa::cuda_fail(e);
  hisa_status_t rc = hisa::run_block_stage(s, q_idx, bk, blk, nullptr, dev_status, ws + L.blk_stage, stream);
  if (rc != HISA_OK) return rc;
  rc = hisa::run_token_stage(s, q_idx, k_idx, blk, s.m, tok, nullptr, dev_status, ws + L.keys,
                             workspace_bytes - L.keys, stream);
  if (rc != HISA_OK) return rc;
  return hisa::cuda_fail(hisa::launch_sparse_attn(s, q, k, v, tok, o, lse, dev_status, ws + L.attn,
                                                  hisa::attn_workspace_bytes(s), stream));
}

hisa_status_t check_forward_args(const void* q_idx, const void* k_idx, const void* q, const void* k, const void* v,
                                 void* o, float* lse, int32_t* block_idx_out, int32_t* token_idx_out) {
  const void* ptrs[] = {q_idx, k_idx, q, k, v, o};
  for (const void* p : ptrs)
    if (!p || !hisa::aligned16(p)) return HISA_ERR_INVALID_ARG;
  if ((lse && !hisa::aligned16(lse)) || (block_idx_out && !hisa::aligned16(block_idx_out)) ||
      (token_idx_out && !hisa::aligned16(token_idx_out)))
    return HISA_ERR_INVALID_ARG;
  return HISA_OK;
}
}  // namespace

hisa_status_t hisa_forward(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                           const void* k_idx, const void* q, const void* k, const void* v, void* o, float* lse,
                           int32_t* block_idx_out, int32_t* token_idx_out, int32_t* dev_status, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, true, &s);
  if (rc == HISA_OK) rc = hisa::set_idx_weights(&s, idx_weights);
  if (rc != HISA_OK) return rc;
  rc = check_forward_args(q_idx, k_idx, q, k, v, o, lse, block_idx_out, token_idx_out);
  if (rc != HISA_OK) return rc;
  const FwdLayout L = fwd_layout(s);
  if (!workspace || !hisa::aligned16(workspace) || workspace_bytes < L.total) return HISA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return forward_impl(s, L, q_idx, k_idx, reinterpret_cast<float*>(ws + L.bk), 0, q, k, v, o, lse, block_idx_out,
                      token_idx_out, dev_status, ws, workspace_bytes, stream);
}

hisa_status_t hisa_forward_cached(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                                  const void* k_idx, float* block_keys, int64_t refresh_begin, const void* q,
                                  const void* k, const void* v, void* o, float* lse, int32_t* block_idx_out,
                                  int32_t* token_idx_out, int32_t* dev_status, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, true, &s);
  if (rc == HISA_OK) rc = hisa::set_idx_weights(&s, idx_weights);
  if (rc != HISA_OK) return rc;
  rc = check_forward_args(q_idx, k_idx, q, k, v, o, lse, block_idx_out, token_idx_out);
  if (rc != HISA_OK) return rc;
  if (!block_keys || !hisa::aligned16(block_keys)) return HISA_ERR_INVALID_ARG;
  if (refresh_begin < 0 || refresh_begin > s.n_blk) return HISA_ERR_INVALID_ARG;
  const FwdLayout L = fwd_layout(s);
  if (!workspace || !hisa::aligned16(workspace) || workspace_bytes < L.total) return HISA_ERR_WORKSPACE;
  return forward_impl(s, L, q_idx, k_idx, block_keys, refresh_begin, q, k, v, o, lse, block_idx_out, token_idx_out,
                      dev_status, static_cast<uint8_t*>(workspace), workspace_bytes, stream);
}

namespace {
// hisa_forward_host: the queries are taken in units whose attention can start as soon as the
// unit's rows are on the device.  A long sequence (n_q > kHostChunk) is cut into query chunks of
// at least kHostChunk queries, at most kHostMaxChunks per sequence: chunk [i0, i1) needs the K/V
// rows [0, n_kv - n_q + i1) only, so each chunk copies just the rows the earlier ones did not.
// Short sequences (decode) go in up to kHostGroups groups of whole sequences.
#ifndef HISA_HOST_CHUNK
#define HISA_HOST_CHUNK 8192
#endif
constexpr int64_t kHostChunk = HISA_HOST_CHUNK;
constexpr int64_t kHostMaxChunks = 16;
constexpr int kHostGroups = 8;

struct HostUnit {
  int s0, s1;      // sequences [s0, s1)
  int64_t i0, i1;  // queries [i0, i1) of each of them
  int64_t kv0;     // first K/V row of the sequence this unit copies (query chunks only)
};

std::vector<HostUnit> host_units(const Shape& s) {
  std::vector<HostUnit> u;
  if (s.n_q > kHostChunk) {
    const int64_t len = std::max(kHostChunk, (s.n_q + kHostMaxChunks - 1) / kHostMaxChunks);
    for (int seq = 0; seq < s.batch; ++seq)
      for (int64_t i0 = 0; i0 < s.n_q; i0 += len)
        u.push_back({seq, seq + 1, i0, std::min(i0 + len, s.n_q), i0 == 0 ? 0 : s.n_kv - s.n_q + i0});
  } else {
    const int g = std::min(s.batch, kHostGroups);
    for (int j = 0; j < g; ++j) u.push_back({s.batch * j / g, s.batch * (j + 1) / g, 0, s.n_q, 0});
  }
  return u;
}

// The attention problem of a unit: its sequences and queries, positions as in the full problem
// (p = n_kv - n_q + i), keys the prefix [0, n_kv - n_q + i1) of each sequence.  A query chunk is
// one sequence, so the shorter key range changes no stride.
Shape unit_shape(const Shape& s, const HostUnit& u) {
  Shape c = s;
  c.batch = u.s1 - u.s0;
  c.n_q = u.i1 - u.i0;
  if (u.i0 > 0 || u.i1 < s.n_q) c.n_kv = s.n_kv - s.n_q + u.i1;
  c.n_query = (int64_t)c.batch * c.n_q;
  c.n_blk = (c.n_kv + s.B - 1) / s.B;
  return c;
}

struct HostFwdLayout {
  FwdLayout f;
  size_t part[2], q_idx, w, k_idx, q, k, v, o, lse, total;
};

HostFwdLayout host_fwd_layout(const Shape& s) {
  HostFwdLayout L;
  L.f = fwd_layout(s);
  size_t part = 0;
  for (const HostUnit& u : host_units(s)) {
    const Shape c = unit_shape(s, u);
    part = std::max(part, hisa::attn_workspace_bytes(c));
  }
  size_t off = L.f.total;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += hisa::align_up(bytes);
    return at;
  };
  const int64_t he = s.HI > 0 ? s.HI : 1;
  L.part[0] = take(part);  // the attention workspace of even units and of odd units
  L.part[1] = take(part);
  L.q_idx = take((size_t)s.n_query * he * s.d_idx * 2);
  L.w = take(s.HI > 0 ? (size_t)s.n_query * s.HI * sizeof(float) : 0);
  L.k_idx = take((size_t)s.batch * s.n_kv * s.d_idx * 2);
  L.q = take((size_t)s.n_query * s.H * s.d * 2);
  L.k = take((size_t)s.batch * s.n_kv * s.Hkv * s.d * 2);
  L.v = take((size_t)s.batch * s.n_kv * s.Hkv * s.d * 2);
  L.o = take((size_t)s.n_query * s.H * s.d * 2);
  L.lse = take((size_t)s.n_query * s.H * sizeof(float));
  L.total = off;
  return L;
}

bool is_device_memory(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();  // an unknown host pointer: not device memory
    return false;
  }
  return a.type == cudaMemoryTypeDevice;
}

// Events of one call, destroyed when it returns (a pending event is released once it completes).
struct EventSet {
  std::vector<cudaEvent_t> ev;
  cudaError_t make(cudaEvent_t* e) {
    const cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
    if (r == cudaSuccess) ev.push_back(*e);
    return r;
  }
  ~EventSet() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
};
}  // namespace

hisa_status_t hisa_forward_host_workspace_size(const hisa_params_t* params, size_t* bytes) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, true, &s);
  if (rc != HISA_OK) return rc;
  if (!bytes) return HISA_ERR_INVALID_ARG;
  *bytes = host_fwd_layout(s).total;
  return HISA_OK;
}

hisa_status_t hisa_forward_host(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                                const void* k_idx, const void* q, const void* k, const void* v, void* o, float* lse,
                                int32_t* dev_status, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                                cudaStream_t copy_stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, true, &s);
  if (rc != HISA_OK) return rc;
  if ((s.HI == 0) != (idx_weights == nullptr)) return HISA_ERR_INVALID_ARG;
  if (!q_idx || !k_idx || !q || !k || !v || !o) return HISA_ERR_INVALID_ARG;
  const HostFwdLayout L = host_fwd_layout(s);
  if (!workspace || !hisa::aligned16(workspace) || workspace_bytes < L.total) return HISA_ERR_WORKSPACE;
  const void* host_ptrs[] = {q_idx, idx_weights, k_idx, q, k, v, o, lse};
  for (const void* p : host_ptrs)
    if (p && is_device_memory(p)) return HISA_ERR_INVALID_ARG;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* d_q_idx = ws + L.q_idx;
  float* d_w = s.HI > 0 ? reinterpret_cast<float*>(ws + L.w) : nullptr;
  uint8_t* d_k_idx = ws + L.k_idx;
  uint8_t* d_q = ws + L.q;
  uint8_t* d_k = ws + L.k;
  uint8_t* d_v = ws + L.v;
  uint8_t* d_o = ws + L.o;
  float* d_lse = reinterpret_cast<float*>(ws + L.lse);
  float* bk = reinterpret_cast<float*>(ws + L.f.bk);
  int32_t* blk = reinterpret_cast<int32_t*>(ws + L.f.block_idx);
  int32_t* tok = reinterpret_cast<int32_t*>(ws + L.f.token_idx);
  rc = hisa::set_idx_weights(&s, d_w);
  if (rc != HISA_OK) return rc;

  const bool overlap = copy_stream != nullptr && copy_stream != stream;
  cudaStream_t cs = overlap ? copy_stream : stream;
  EventSet events;
  // With copies on their own stream, units alternate between `stream` and a second compute stream
  // of the call, each with its own workspace part, so that a unit starts on the SMs the previous
  // unit's last wave leaves idle.
  cudaStream_t s2 = nullptr;
  if (overlap && cudaStreamCreateWithFlags(&s2, cudaStreamNonBlocking) != cudaSuccess) {
    (void)cudaGetLastError();
    s2 = nullptr;
  }
  struct StreamGuard {
    cudaStream_t st;
    ~StreamGuard() {
      if (st) cudaStreamDestroy(st);
    }
  } s2_guard{s2};
  // Everything enqueued (on success or after an error) completes before the call returns, so
  // the host buffers and the events are free afterwards.
  auto enqueue = [&]() -> hisa_status_t {
    cudaError_t e = cudaSuccess;
    auto ok = [&](cudaError_t r) {
      if (e == cudaSuccess) e = r;
      return e == cudaSuccess;
    };
    // the copy stream starts after the caller's earlier work on stream (which may use the workspace)
    if (overlap) {
      cudaEvent_t start;
      if (!ok(events.make(&start)) || !ok(cudaEventRecord(start, stream)) || !ok(cudaStreamWaitEvent(cs, start, 0)))
        return hisa::cuda_fail(e);
    }

    // Indexer inputs first (ahead of the attention inputs on the copy stream, so that they have
    // the link to themselves), then steps 1-5 on stream while the attention inputs stream in.
    const int64_t he = s.HI > 0 ? s.HI : 1;
    const size_t qrow = (size_t)s.H * s.d * 2, kvrow = (size_t)s.Hkv * s.d * 2;
    ok(cudaMemcpyAsync(d_q_idx, q_idx, (size_t)s.n_query * he * s.d_idx * 2, cudaMemcpyHostToDevice, cs));
    if (d_w) ok(cudaMemcpyAsync(d_w, idx_weights, (size_t)s.n_query * s.HI * sizeof(float), cudaMemcpyHostToDevice,
                                cs));
    ok(cudaMemcpyAsync(d_k_idx, k_idx, (size_t)s.batch * s.n_kv * s.d_idx * 2, cudaMemcpyHostToDevice, cs));
    if (overlap) {
      cudaEvent_t idx_in;
      if (ok(events.make(&idx_in)) && ok(cudaEventRecord(idx_in, cs))) ok(cudaStreamWaitEvent(stream, idx_in, 0));
    }
    if (e != cudaSuccess) return hisa::cuda_fail(e);
    if (!ok(hisa::launch_block_pool(s, d_k_idx, 0, s.n_blk, bk, stream))) return hisa::cuda_fail(e);
    rc = hisa::run_block_stage(s, d_q_idx, bk, blk, nullptr, dev_status, ws + L.f.blk_stage, stream);
    if (rc != HISA_OK) return rc;
    rc = hisa::run_token_stage(s, d_q_idx, d_k_idx, blk, s.m, tok, nullptr, dev_status, ws + L.f.keys,
                               L.f.total - L.f.keys, stream);
    if (rc != HISA_OK) return rc;

    const std::vector<HostUnit> units = host_units(s);
    std::vector<cudaEvent_t> in(units.size()), done(units.size());
    auto h2d = [&](uint8_t* dst, const void* src, size_t off, size_t bytes) {
      return ok(cudaMemcpyAsync(dst + off, static_cast<const uint8_t*>(src) + off, bytes, cudaMemcpyHostToDevice, cs));
    };
    for (size_t j = 0; j < units.size() && e == cudaSuccess; ++j) {
      const HostUnit& u = units[j];
      const Shape c = unit_shape(s, u);
      // K/V rows [kv0, c.n_kv) of each of the unit's sequences; its Q rows
      for (int seq = u.s0; seq < u.s1; ++seq) {
        const size_t off = ((size_t)seq * s.n_kv + u.kv0) * kvrow, bytes = (size_t)(c.n_kv - u.kv0) * kvrow;
        h2d(d_k, k, off, bytes);
        h2d(d_v, v, off, bytes);
      }
      if (u.i0 == 0 && u.i1 == s.n_q)
        h2d(d_q, q, (size_t)u.s0 * s.n_q * qrow, (size_t)(u.s1 - u.s0) * s.n_q * qrow);
      else
        h2d(d_q, q, ((size_t)u.s0 * s.n_q + u.i0) * qrow, (size_t)(u.i1 - u.i0) * qrow);
      if (overlap && ok(events.make(&in[j]))) ok(cudaEventRecord(in[j], cs));
    }
    if (e != cudaSuccess) return hisa::cuda_fail(e);

    // Step 6 per unit, as soon as its rows are in; odd units on the second compute stream (after
    // the token stage, and after the unit two before it, which used the same workspace part).
    if (s2) {
      cudaEvent_t idx_done;
      if (!ok(events.make(&idx_done)) || !ok(cudaEventRecord(idx_done, stream)) ||
          !ok(cudaStreamWaitEvent(s2, idx_done, 0)))
        return hisa::cuda_fail(e);
    }
    for (size_t j = 0; j < units.size(); ++j) {
      const HostUnit& u = units[j];
      const Shape c = unit_shape(s, u);
      const int part = s2 ? (int)(j & 1) : 0;
      cudaStream_t us = part ? s2 : stream;
      if (overlap && !ok(cudaStreamWaitEvent(us, in[j], 0))) return hisa::cuda_fail(e);
      const size_t q0 = (size_t)u.s0 * s.n_q + u.i0;  // first query row of the unit
      const size_t kv_off = (size_t)u.s0 * s.n_kv * kvrow;
      if (!ok(hisa::launch_sparse_attn(c, d_q + q0 * qrow, d_k + kv_off, d_v + kv_off, tok + q0 * s.k, d_o + q0 * qrow,
                                       d_lse + q0 * s.H, dev_status, ws + L.part[part], hisa::attn_workspace_bytes(c),
                                       us)))
        return hisa::cuda_fail(e);
      if (overlap && ok(events.make(&done[j]))) ok(cudaEventRecord(done[j], us));
      if (e != cudaSuccess) return hisa::cuda_fail(e);
    }
    if (s2 && units.size() > 1) {  // stream waits for the second stream's last unit
      const size_t last_odd = ((units.size() - 1) & 1) ? units.size() - 1 : units.size() - 2;
      if (!ok(cudaStreamWaitEvent(stream, done[last_odd], 0))) return hisa::cuda_fail(e);
    }

    // O and LSE of each unit back to the host once its attention is done.
    for (size_t j = 0; j < units.size() && e == cudaSuccess; ++j) {
      const HostUnit& u = units[j];
      const size_t q0 = (size_t)u.s0 * s.n_q + u.i0;
      const size_t rows = (size_t)(u.s1 - u.s0) * (u.i1 - u.i0);  // contiguous: several sequences only whole
      if (overlap) ok(cudaStreamWaitEvent(cs, done[j], 0));
      ok(cudaMemcpyAsync(static_cast<uint8_t*>(o) + q0 * qrow, d_o + q0 * qrow, rows * qrow, cudaMemcpyDeviceToHost,
                         cs));
      if (lse)
        ok(cudaMemcpyAsync(lse + q0 * s.H, d_lse + q0 * s.H, rows * s.H * sizeof(float), cudaMemcpyDeviceToHost, cs));
    }
    // The outputs are in host memory when the call returns: stream waits for the copies back and
    // is synchronised (the events of the call are then complete before they are destroyed).
    if (overlap && e == cudaSuccess) {
      cudaEvent_t end;
      if (ok(events.make(&end)) && ok(cudaEventRecord(end, cs))) ok(cudaStreamWaitEvent(stream, end, 0));
    }
    return hisa::cuda_fail(e);
  };
  const hisa_status_t st = enqueue();
  if (s2) (void)cudaStreamSynchronize(s2);
  if (overlap) (void)cudaStreamSynchronize(cs);
  const cudaError_t se = cudaStreamSynchronize(stream);
  if (st != HISA_OK) return st;
  return hisa::cuda_fail(se);
}

namespace hisa {
namespace {

// The flat indexer's window: 8192 candidate tokens (k rounded up to blocks if more), in blocks.
int flat_window(const Shape& s) {
  int64_t w = 8192 / s.B;
  if (w < 1) w = 1;
  if (w * s.B < s.k) w = (s.k + s.B - 1) / s.B;
  if (w > s.n_blk) w = s.n_blk;
  return (int)w;
}

// Bytes per query row processed at once: the window's keys and four k-entry arrays (two running
// lists, ids and scores each).
size_t flat_row_bytes(const Shape& s) {
  return (size_t)flat_window(s) * s.B * sizeof(uint32_t) + 4 * (size_t)s.k * 4;
}

constexpr size_t kFlatCap = (size_t)8 << 30;

}  // namespace
}  // namespace hisa

hisa_status_t hisa_flat_topk_workspace_size(const hisa_params_t* params, size_t* min_bytes, size_t* preferred_bytes) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, false, &s);
  if (rc != HISA_OK) return rc;
  if (!min_bytes && !preferred_bytes) return HISA_ERR_INVALID_ARG;
  if (s.n_blk > 50000 || s.k >= 32768) return HISA_ERR_UNSUPPORTED;
  const size_t per = hisa::flat_row_bytes(s) + 5 * hisa::kAlign;
  size_t rows = hisa::kFlatCap / per;
  if (rows < 1) rows = 1;
  if (rows > (size_t)s.n_query) rows = (size_t)s.n_query;
  if (min_bytes) *min_bytes = per;
  if (preferred_bytes) *preferred_bytes = rows * per;
  return HISA_OK;
}

hisa_status_t hisa_flat_topk(const hisa_params_t* params, const void* q_idx, const float* idx_weights,
                             const void* k_idx, int32_t* token_idx, float* token_scores, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(params, true, false, &s);
  if (rc == HISA_OK) rc = hisa::set_idx_weights(&s, idx_weights);
  if (rc != HISA_OK) return rc;
  if (!q_idx || !k_idx || !token_idx) return HISA_ERR_INVALID_ARG;
  if (!hisa::aligned16(q_idx) || !hisa::aligned16(k_idx) || !hisa::aligned16(token_idx)) return HISA_ERR_INVALID_ARG;
  if (token_scores && !hisa::aligned16(token_scores)) return HISA_ERR_INVALID_ARG;
  if (!workspace || !hisa::aligned16(workspace)) return HISA_ERR_WORKSPACE;
  if (s.n_blk > 50000 || s.k >= 32768) return HISA_ERR_UNSUPPORTED;
  const int W = hisa::flat_window(s);
  const int64_t k = s.k, WB = (int64_t)W * s.B;
  // rows per chunk: the window's keys, then running lists 0 and 1
  const size_t per = hisa::flat_row_bytes(s) + 5 * hisa::kAlign;
  int64_t R = (int64_t)(workspace_bytes / per);
  if (R < 1) return HISA_ERR_WORKSPACE;
  if (R > s.n_query) R = s.n_query;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base + off;
    off += hisa::align_up(bytes);
    return p;
  };
  uint32_t* keys = reinterpret_cast<uint32_t*>(take((size_t)R * WB * 4));
  int32_t* ids[2];
  float* sc[2];
  for (int i = 0; i < 2; ++i) {
    ids[i] = reinterpret_cast<int32_t*>(take((size_t)R * k * 4));
    sc[i] = reinterpret_cast<float*>(take((size_t)R * k * 4));
  }
  // the select writes row q at out + q * k: shift a chunk buffer so that global row g0 lands first
  auto at_row = [&](auto* buf, int64_t g0) {
    return reinterpret_cast<decltype(buf)>(reinterpret_cast<uintptr_t>(buf) - (uintptr_t)(g0 * k * 4));
  };
  const int64_t off_kv = s.n_kv - s.n_q;  // position of query 0
  // Window j covers blocks [j W, (j + 1) W); query i (position off_kv + i) takes part in windows
  // 0 .. its own, and its list is final after that one: rows that end at window j write the output,
  // the rest carry a running list (buffers cur / nxt in turn) to window j + 1.
  auto first_row = [&](int64_t j, int64_t a) {  // first row of the chunk taking part in window j
    const int64_t r = j * WB - off_kv;
    return r > a ? r : a;
  };
  // When every query sees every window (decode; or sequences whose first query lies past the last
  // window's start), whole sequences share each window's launches: G of them per group.
  const int64_t n_win = (s.n_blk + W - 1) / W;
  const bool all_see = (n_win - 1) * WB <= off_kv;
  const int64_t G = (all_see && R >= s.n_q) ? R / s.n_q : 1;
  for (int64_t seq0 = 0; seq0 < s.batch; seq0 += G) {
    const int64_t nseq = G < s.batch - seq0 ? G : s.batch - seq0;
    for (int64_t a = 0; a < s.n_q; a += (nseq > 1 ? s.n_q : R)) {
      const int64_t b = nseq > 1 ? s.n_q : (a + R < s.n_q ? a + R : s.n_q);
      const int64_t g0 = seq0 * s.n_q + a;  // global query of the chunk's row 0
      int cur = 0, nxt = 1;
      for (int64_t j = 0; j < n_win; ++j) {
        const int64_t qa = first_row(j, a);
        if (qa >= b) break;
        const int64_t qe = j + 1 < n_win ? (first_row(j + 1, a) < b ? first_row(j + 1, a) : b) : b;
        // per sequence, rows [qa, qe) end here and rows [qe, b) go on; as chunk rows (with several
        // sequences, qa = a = 0 and qe is 0 or n_q, so the ranges cover whole sequences)
        const int64_t ra = (qa - a) * nseq, re = (qe - a) * nseq, rb = (b - a) * nseq;
        const int blo = (int)(j * W);
        cudaError_t e =
            hisa::launch_token_score(s, q_idx, k_idx, nullptr, W, keys, nullptr, g0 + ra, rb - ra, stream, blo);
        const uint32_t* keys_go = keys + (re - ra) * WB;  // key rows of the rows that go on
        if (j == 0) {
          if (e == cudaSuccess && re > ra)
            e = hisa::launch_token_select(s, keys, nullptr, W, token_idx, token_scores, g0 + ra, re - ra, stream, blo);
          if (e == cudaSuccess && rb > re)
            e = hisa::launch_token_select(s, keys_go, nullptr, W, at_row(ids[cur], g0), at_row(sc[cur], g0), g0 + re,
                                          rb - re, stream, blo);
        } else {
          const int64_t tok0 = (int64_t)blo * s.B;
          if (e == cudaSuccess && re > ra)
            e = hisa::launch_flat_select(keys, (int)WB, ids[cur] + ra * k, sc[cur] + ra * k, (int)k, tok0, re - ra,
                                         token_idx + (g0 + ra) * k,
                                         token_scores ? token_scores + (g0 + ra) * k : nullptr, stream);
          if (e == cudaSuccess && rb > re)
            e = hisa::launch_flat_select(keys_go, (int)WB, ids[cur] + re * k, sc[cur] + re * k, (int)k, tok0, rb - re,
                                         ids[nxt] + re * k, sc[nxt] + re * k, stream);
          const int t = cur;
          cur = nxt;
          nxt = t;
        }
        if (e != cudaSuccess) return hisa::cuda_fail(e);
      }
    }
  }
  return HISA_OK;
}

hisa_status_t hisa_block_candidates_workspace_size(const hisa_params_t* local, size_t* bytes) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(local, true, false, &s);
  if (rc != HISA_OK) return rc;
  if (!bytes) return HISA_ERR_INVALID_ARG;
  *bytes = (size_t)s.n_query * s.n_blk * sizeof(float);
  return HISA_OK;
}

hisa_status_t hisa_block_candidates(const hisa_params_t* local, int64_t n_kv_global, int64_t first_block,
                                    const void* q_idx, const float* idx_weights, const float* block_keys,
                                    float* cand_scores, int32_t* cand_ids, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream) {
  Shape s;
  hisa_status_t rc = hisa::make_shape(local, true, false, &s);
  if (rc == HISA_OK) rc = hisa::set_idx_weights(&s, idx_weights);
  if (rc != HISA_OK) return rc;
  if (s.n_q != 1) return HISA_ERR_UNSUPPORTED;  // decode: the query is the newest token of the whole context
  if (first_block < 0 || n_kv_global < 1 || first_block * s.B + s.n_kv > n_kv_global) return HISA_ERR_INVALID_ARG;
  if (!q_idx || !block_keys || !cand_scores || !cand_ids) return HISA_ERR_INVALID_ARG;
  if (!hisa::aligned16(q_idx) || !hisa::aligned16(block_keys)) return HISA_ERR_INVALID_ARG;
  if (!workspace || !hisa::aligned16(workspace) || workspace_bytes < (size_t)s.n_query * s.n_blk * sizeof(float))
    return HISA_ERR_WORKSPACE;
  float* scores = static_cast<float*>(workspace);
  cudaError_t e = hisa::launch_block_score(s, q_idx, block_keys, scores, stream);
  if (e != cudaSuccess) return hisa::cuda_fail(e);
  const int64_t c = (n_kv_global - 1) / s.B;
  return hisa::cuda_fail(
      hisa::launch_block_candidates(s, scores, first_block, c, s.m - 2, cand_scores, cand_ids, stream));
}

hisa_status_t hisa_topk_merge(const float* scores, const int32_t* ids, int32_t n_parts, int64_t rows, int32_t n_per,
                              int32_t k, int32_t* out_ids, float* out_scores, cudaStream_t stream) {
  if (!scores || !ids || !out_ids || n_parts < 1 || rows < 0 || rows > 0x7FFFFFFFLL || n_per < 1 || k < 1)
    return HISA_ERR_INVALID_ARG;
  if ((int64_t)n_parts * n_per > (1 << 24)) return HISA_ERR_UNSUPPORTED;
  if (rows == 0) return HISA_OK;
  return hisa::cuda_fail(hisa::launch_topk_merge(scores, ids, n_parts, rows, n_per, k, out_ids, out_scores, stream));
}

hisa_status_t hisa_remap_ids(const int32_t* in, int64_t rows, int32_t cols, int64_t lo, int64_t hi, int64_t delta,
                             int32_t* out, cudaStream_t stream) {
  if (!in || !out || rows < 0 || cols < 1 || lo > hi) return HISA_ERR_INVALID_ARG;
  if (hi + delta > 0x7FFFFFFFLL || lo + delta < 0) return HISA_ERR_INVALID_ARG;
  if (rows == 0) return HISA_OK;
  return hisa::cuda_fail(hisa::launch_remap_ids(in, rows, cols, lo, hi, delta, out, stream));
}

hisa_status_t hisa_lse_merge(const void* o_parts, const float* lse_parts, int32_t n_parts, int64_t rows, int32_t d,
                             void* o, float* lse, cudaStream_t stream) {
  if (!o_parts || !lse_parts || !o || n_parts < 1 || rows < 0 || d < 1) return HISA_ERR_INVALID_ARG;
  if (rows == 0) return HISA_OK;
  return hisa::cuda_fail(hisa::launch_lse_merge(o_parts, lse_parts, n_parts, rows, d, o, lse, stream));
}

hisa_status_t hisa_gather_probe(const void* rows, int64_t n_rows, int32_t row_bytes, int64_t n_gathers, uint32_t seed,
                                uint32_t* sink, int32_t ctas_per_sm, cudaStream_t stream) {
  if (!rows || !sink || n_rows < 1 || n_rows > 0x7FFFFFFFLL || n_gathers < 0) return HISA_ERR_INVALID_ARG;
  if (ctas_per_sm < 0 || ctas_per_sm > 3) return HISA_ERR_INVALID_ARG;
  if (!hisa::gather_probe_row_bytes_ok(row_bytes) || !hisa::aligned16(rows)) return HISA_ERR_INVALID_ARG;
  if (n_gathers == 0) return HISA_OK;
  return hisa::cuda_fail(hisa::launch_gather_probe(rows, n_rows, row_bytes, n_gathers, seed, sink,
                                                     ctas_per_sm ? ctas_per_sm : 3, stream));
}

}  // extern "C"
