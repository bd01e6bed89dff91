"""Python binding of the two-level sparse-attention library (include/hisa.h).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libhisa.so``.  PyTorch supplies device memory and the current stream.  The
library must be built (``hierarchical_sparse_attention_block_b200.build``);
importing this package without it raises ImportError -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhisa.so")

HISA_OK, HISA_ERR_INVALID_ARG, HISA_ERR_UNSUPPORTED, HISA_ERR_WORKSPACE, HISA_ERR_CUDA = range(5)
STATUS_BAD_INDEX = 1
STATUS_TIMEOUT = 2

# Every exported symbol of include/hisa.h.
EXPORTS = (
    "hisa_block_pool", "hisa_block_topm_workspace_size", "hisa_block_topm", "hisa_token_topk_workspace_size",
    "hisa_token_topk", "hisa_sparse_attn_workspace_size", "sparse_attn_fwd", "hisa_forward_workspace_size",
    "hisa_forward", "hisa_flat_topk_workspace_size", "hisa_flat_topk", "hisa_status_string",
    "hisa_last_cuda_error", "hisa_version", "hisa_token_topk_noalloc", "hisa_forward_cached", "hisa_gather_probe",
    "hisa_block_candidates_workspace_size", "hisa_block_candidates", "hisa_topk_merge", "hisa_remap_ids",
    "hisa_lse_merge", "hisa_forward_host_workspace_size", "hisa_forward_host", "hisa_sparse_attn_kernel",
)


class HisaParams(ctypes.Structure):
    """Mirror of hisa_params_t."""

    _fields_ = [
        ("batch", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("n_q", ctypes.c_int64), ("n_kv", ctypes.c_int64),
        ("block", ctypes.c_int32), ("top_m", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("d_head", ctypes.c_int32),
        ("scale", ctypes.c_float), ("flags", ctypes.c_int32), ("n_idx_heads", ctypes.c_int32),
    ]


class HisaError(RuntimeError):
    """A call of the library returned a status other than HISA_OK, or the binding refused an argument
    before the call (then ``status`` is HISA_ERR_INVALID_ARG, the status the library gives bad arguments)."""

    def __init__(self, call: str, status: int, detail: str | None = None):
        if detail is None:
            detail = _lib.hisa_status_string(status).decode()
            if status == HISA_ERR_CUDA:
                detail += f" (cudaError {_lib.hisa_last_cuda_error()})"
        super().__init__(f"{call}: {detail}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python hierarchical_sparse_attention_block_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)
    pp = ctypes.POINTER(HisaParams)
    sig = {
        "hisa_block_pool": [pp, vp, i64, i64, vp, vp],
        "hisa_block_topm_workspace_size": [pp, sz],
        "hisa_block_topm": [pp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp],
        "hisa_token_topk_workspace_size": [pp, sz, sz],
        "hisa_token_topk": [pp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp],
        "hisa_sparse_attn_workspace_size": [pp, sz],
        "sparse_attn_fwd": [pp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp],
        "hisa_forward_workspace_size": [pp, sz],
        "hisa_forward": [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp],
        "hisa_flat_topk_workspace_size": [pp, sz, sz],
        "hisa_flat_topk": [pp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp],
        "hisa_token_topk_noalloc": [pp, vp, vp, vp, vp, vp, vp, vp, vp],
        "hisa_forward_cached": [pp, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp],
        "hisa_forward_host_workspace_size": [pp, sz],
        "hisa_forward_host": [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp],
        "hisa_gather_probe": [vp, i64, ctypes.c_int32, i64, ctypes.c_uint32, vp, ctypes.c_int32, vp],
        "hisa_block_candidates_workspace_size": [pp, sz],
        "hisa_block_candidates": [pp, i64, i64, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp],
        "hisa_topk_merge": [vp, vp, ctypes.c_int32, i64, ctypes.c_int32, ctypes.c_int32, vp, vp, vp],
        "hisa_remap_ids": [vp, i64, ctypes.c_int32, i64, i64, i64, vp, vp],
        "hisa_lse_merge": [vp, vp, ctypes.c_int32, i64, ctypes.c_int32, vp, vp, vp],
        "hisa_sparse_attn_kernel": [pp, ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32)],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.hisa_status_string.argtypes = [ctypes.c_int]
    lib.hisa_status_string.restype = ctypes.c_char_p
    lib.hisa_last_cuda_error.restype = ctypes.c_int32
    lib.hisa_version.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib():
    return _lib


def params(batch, n_q, n_kv, d_idx, block, top_m, top_k, n_heads=1, n_kv_heads=None, d_head=64,
           scale=0.0, n_idx_heads=0) -> HisaParams:
    return HisaParams(batch=batch, d_idx=d_idx, n_q=n_q, n_kv=n_kv, block=block, top_m=top_m, top_k=top_k,
                      n_heads=n_heads, n_kv_heads=n_kv_heads if n_kv_heads else n_heads, d_head=d_head,
                      scale=scale, flags=0, n_idx_heads=n_idx_heads)


def params_of(w) -> HisaParams:
    """hisa_params_t of a workload description (synth.workloads.Workload or alike)."""
    return params(w.batch, w.n_q, w.n_kv, w.d_idx, w.block, w.top_m, w.top_k, w.n_heads, w.n_kv_heads, w.d_head,
                  n_idx_heads=getattr(w, "n_idx_heads", 0))


def _ptr(t):
    """Device address of a CUDA tensor (None passes through).  A CPU tensor is refused here, before
    a host address could reach a kernel."""
    if t is None:
        return None
    if not t.is_cuda:
        raise HisaError("binding", HISA_ERR_INVALID_ARG, f"expected a CUDA tensor, got one on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def _hptr(t):
    """Host address of a CPU tensor (None passes through), for the host-buffer entry point."""
    if t is None:
        return None
    if t.is_cuda:
        raise HisaError("binding", HISA_ERR_INVALID_ARG, "expected a host (CPU) tensor, got a CUDA one")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch

        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name, rc):
    if rc != HISA_OK:
        raise HisaError(name, rc)


def _size(fn, p, two=False):
    a = ctypes.c_size_t(0)
    if two:
        b = ctypes.c_size_t(0)
        _check(fn.__name__, fn(ctypes.byref(p), ctypes.byref(a), ctypes.byref(b)))
        return a.value, b.value
    _check(fn.__name__, fn(ctypes.byref(p), ctypes.byref(a)))
    return a.value


def _workspace(nbytes, device):
    import torch

    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- calls of include/hisa.h

def hisa_block_pool(p, k_idx, block_keys, blk_begin=0, blk_end=-1, stream=None):
    _check("hisa_block_pool", _lib.hisa_block_pool(ctypes.byref(p), _ptr(k_idx), blk_begin, blk_end,
                                                   _ptr(block_keys), _stream(stream)))


def hisa_block_topm_workspace_size(p) -> int:
    return _size(_lib.hisa_block_topm_workspace_size, p)


def hisa_block_topm(p, q_idx, block_keys, block_idx, block_scores=None, dev_status=None, workspace=None,
                    stream=None, idx_weights=None):
    if workspace is None:
        workspace = _workspace(hisa_block_topm_workspace_size(p), q_idx.device)
    _check("hisa_block_topm", _lib.hisa_block_topm(ctypes.byref(p), _ptr(q_idx), _ptr(idx_weights), _ptr(block_keys),
                                                   _ptr(block_idx),
                                                   _ptr(block_scores), _ptr(dev_status), _ptr(workspace),
                                                   workspace.numel(), _stream(stream)))


def hisa_token_topk_workspace_size(p):
    """(minimum, preferred) bytes."""
    return _size(_lib.hisa_token_topk_workspace_size, p, two=True)


def hisa_token_topk(p, q_idx, k_idx, block_idx, token_idx, token_scores=None, dev_status=None, workspace=None,
                    stream=None, idx_weights=None):
    if workspace is None:
        workspace = _workspace(hisa_token_topk_workspace_size(p)[1], q_idx.device)
    _check("hisa_token_topk", _lib.hisa_token_topk(ctypes.byref(p), _ptr(q_idx), _ptr(idx_weights), _ptr(k_idx),
                                                   _ptr(block_idx),
                                                   _ptr(token_idx), _ptr(token_scores), _ptr(dev_status),
                                                   _ptr(workspace), workspace.numel(), _stream(stream)))


def hisa_sparse_attn_workspace_size(p) -> int:
    return _size(_lib.hisa_sparse_attn_workspace_size, p)


def sparse_attn_fwd(p, q, k, v, token_idx, o, lse=None, dev_status=None, workspace=None, stream=None):
    if workspace is None:
        n = hisa_sparse_attn_workspace_size(p)
        workspace = _workspace(n, q.device) if n else None
    _check("sparse_attn_fwd", _lib.sparse_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(token_idx),
                                                   _ptr(o), _ptr(lse), _ptr(dev_status), _ptr(workspace),
                                                   0 if workspace is None else workspace.numel(), _stream(stream)))


ATTN_GATHER, ATTN_QTILE = 0, 1


def hisa_sparse_attn_kernel(p, workspace_bytes: int) -> int:
    """Which step-6 kernel sparse_attn_fwd runs with this workspace: ATTN_QTILE or ATTN_GATHER."""
    k = ctypes.c_int32(-1)
    _check("hisa_sparse_attn_kernel", _lib.hisa_sparse_attn_kernel(ctypes.byref(p), int(workspace_bytes),
                                                                    ctypes.byref(k)))
    return k.value


def hisa_forward_workspace_size(p) -> int:
    return _size(_lib.hisa_forward_workspace_size, p)


def hisa_forward(p, q_idx, k_idx, q, k, v, o, lse=None, block_idx_out=None, token_idx_out=None, dev_status=None,
                 workspace=None, stream=None, idx_weights=None):
    if workspace is None:
        workspace = _workspace(hisa_forward_workspace_size(p), q_idx.device)
    _check("hisa_forward", _lib.hisa_forward(ctypes.byref(p), _ptr(q_idx), _ptr(idx_weights), _ptr(k_idx), _ptr(q),
                                             _ptr(k), _ptr(v),
                                             _ptr(o), _ptr(lse), _ptr(block_idx_out), _ptr(token_idx_out),
                                             _ptr(dev_status), _ptr(workspace), workspace.numel(), _stream(stream)))


def hisa_forward_cached(p, q_idx, k_idx, block_keys, refresh_begin, q, k, v, o, lse=None, block_idx_out=None,
                        token_idx_out=None, dev_status=None, workspace=None, stream=None, idx_weights=None):
    if workspace is None:
        workspace = _workspace(hisa_forward_workspace_size(p), q_idx.device)
    _check("hisa_forward_cached",
           _lib.hisa_forward_cached(ctypes.byref(p), _ptr(q_idx), _ptr(idx_weights), _ptr(k_idx), _ptr(block_keys),
                                    int(refresh_begin),
                                    _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(block_idx_out),
                                    _ptr(token_idx_out), _ptr(dev_status), _ptr(workspace), workspace.numel(),
                                    _stream(stream)))


def hisa_forward_host_workspace_size(p):
    return _size(_lib.hisa_forward_host_workspace_size, p)


def hisa_forward_host(p, q_idx, k_idx, q, k, v, o, lse=None, dev_status=None, workspace=None, stream=None,
                      copy_stream=None, idx_weights=None):
    """Steps 1-6 with host inputs and outputs (CPU tensors, pinned for asynchronous copies) and a
    device workspace; the copies overlap the work when copy_stream is given (see include/hisa.h).
    Synchronous: returns when o and lse hold the results."""
    import torch

    if workspace is None:
        workspace = _workspace(hisa_forward_host_workspace_size(p), torch.device("cuda", torch.cuda.current_device()))
    cs = ctypes.c_void_p(copy_stream.cuda_stream) if copy_stream is not None else None
    _check("hisa_forward_host",
           _lib.hisa_forward_host(ctypes.byref(p), _hptr(q_idx), _hptr(idx_weights), _hptr(k_idx), _hptr(q),
                                  _hptr(k), _hptr(v), _hptr(o), _hptr(lse), _ptr(dev_status), _ptr(workspace),
                                  workspace.numel(), _stream(stream), cs))


def hisa_flat_topk_workspace_size(p):
    return _size(_lib.hisa_flat_topk_workspace_size, p, two=True)


def hisa_flat_topk(p, q_idx, k_idx, token_idx, token_scores=None, workspace=None, stream=None, idx_weights=None):
    if workspace is None:
        workspace = _workspace(hisa_flat_topk_workspace_size(p)[1], q_idx.device)
    _check("hisa_flat_topk", _lib.hisa_flat_topk(ctypes.byref(p), _ptr(q_idx), _ptr(idx_weights), _ptr(k_idx),
                                                 _ptr(token_idx),
                                                 _ptr(token_scores), _ptr(workspace), workspace.numel(),
                                                 _stream(stream)))


def hisa_token_topk_noalloc(p, q_idx, k_idx, block_idx, token_idx, token_scores=None, dev_status=None,
                            stream=None, idx_weights=None):
    """hisa_token_topk for callers that cannot allocate: the library's fixed device scratch
    array stands in for the workspace (see include/hisa.h)."""
    _check("hisa_token_topk_noalloc",
           _lib.hisa_token_topk_noalloc(ctypes.byref(p), _ptr(q_idx), _ptr(idx_weights), _ptr(k_idx), _ptr(block_idx),
                                        _ptr(token_idx),
                                        _ptr(token_scores), _ptr(dev_status), _stream(stream)))


def hisa_block_candidates_workspace_size(p) -> int:
    return _size(_lib.hisa_block_candidates_workspace_size, p)


def hisa_block_candidates(p_local, n_kv_global, first_block, q_idx, block_keys, cand_scores, cand_ids,
                          workspace=None, stream=None, idx_weights=None):
    """This rank's step-3 candidates (see include/hisa.h): [batch][top_m] scores and global block ids."""
    if workspace is None:
        workspace = _workspace(hisa_block_candidates_workspace_size(p_local), q_idx.device)
    _check("hisa_block_candidates",
           _lib.hisa_block_candidates(ctypes.byref(p_local), n_kv_global, first_block, _ptr(q_idx), _ptr(idx_weights),
                                      _ptr(block_keys),
                                      _ptr(cand_scores), _ptr(cand_ids), _ptr(workspace), workspace.numel(),
                                      _stream(stream)))


def hisa_topk_merge(scores, ids, k, out_ids, out_scores=None, stream=None):
    """Best k of the candidates in scores / ids [n_parts][rows][n_per] (ascending ids within a row)."""
    n_parts, rows, n_per = scores.shape
    _check("hisa_topk_merge", _lib.hisa_topk_merge(_ptr(scores), _ptr(ids), n_parts, rows, n_per, k, _ptr(out_ids),
                                                   _ptr(out_scores), _stream(stream)))


def hisa_remap_ids(ids, lo, hi, delta, out=None, stream=None):
    """Entries of each row of ids [rows][cols] inside [lo, hi), shifted by delta, compacted, -1 padded."""
    out = ids if out is None else out
    rows, cols = ids.reshape(-1, ids.shape[-1]).shape
    _check("hisa_remap_ids", _lib.hisa_remap_ids(_ptr(ids), rows, cols, lo, hi, delta, _ptr(out), _stream(stream)))
    return out


def hisa_lse_merge(o_parts, lse_parts, o, lse=None, stream=None):
    """o_parts [n_parts][rows..][d] bf16 and lse_parts [n_parts][rows..] merged into o (and lse)."""
    n_parts, d = o_parts.shape[0], o_parts.shape[-1]
    rows = lse_parts[0].numel()
    _check("hisa_lse_merge", _lib.hisa_lse_merge(_ptr(o_parts), _ptr(lse_parts), n_parts, rows, d, _ptr(o), _ptr(lse),
                                                 _stream(stream)))


def hisa_gather_probe(rows, row_bytes, n_gathers, sink, seed=1, ctas_per_sm=0, stream=None):
    """Measurement helper: n_gathers copies of hashed rows of `rows` into shared memory, the
    attention kernel's gather pattern without its arithmetic (see include/hisa.h)."""
    n_rows = rows.numel() * rows.element_size() // row_bytes
    _check("hisa_gather_probe", _lib.hisa_gather_probe(_ptr(rows), n_rows, row_bytes, n_gathers, seed, _ptr(sink),
                                                       ctas_per_sm, _stream(stream)))


def hisa_version() -> str:
    return _lib.hisa_version().decode()


# ---------------------------------------------------------------- convenience front end

def forward(p, q_idx, k_idx, q, k, v, return_indices=False, stream=None, idx_weights=None):
    """Allocate the outputs with torch and run hisa_forward; returns (o, lse[, block_idx, token_idx]).
    idx_weights: the indexer's head weights [b][n_q][n_idx_heads] when p.n_idx_heads > 0."""
    import torch

    dev = q_idx.device
    o = torch.empty((p.batch, p.n_q, p.n_heads, p.d_head), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((p.batch, p.n_q, p.n_heads), dtype=torch.float32, device=dev)
    blk = tok = None
    if return_indices:
        blk = torch.empty((p.batch, p.n_q, p.top_m), dtype=torch.int32, device=dev)
        tok = torch.empty((p.batch, p.n_q, p.top_k), dtype=torch.int32, device=dev)
    hisa_forward(p, q_idx, k_idx, q, k, v, o, lse, blk, tok, stream=stream, idx_weights=idx_weights)
    return (o, lse, blk, tok) if return_indices else (o, lse)


def n_blocks(p) -> int:
    return math.ceil(p.n_kv / p.block)
