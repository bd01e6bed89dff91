"""TEST INFRASTRUCTURE ONLY: ctypes front end of the plain CPU oracle (hisa_oracle.c).

Only ``tests/``, ``__graft_entry__.smoke()`` and the bench's CPU-baseline /
reference leg may import this package.  The product path never routes through
it.  The oracle shares no code with the CUDA library; the only thing both
sides share is the seeded input generator in ``synth``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "hisa_oracle.c")
LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = np.ctypeslib.ndpointer
_u16 = _P(dtype=np.uint16, flags="C_CONTIGUOUS")
_f64 = _P(dtype=np.float64, flags="C_CONTIGUOUS")
_i32 = _P(dtype=np.int32, flags="C_CONTIGUOUS")
_i64 = _P(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force: bool = False, out: str = LIB_PATH, defines=()) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               *[f"-D{d}" for d in defines], SRC, "-o", out, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def load(path: str = LIB_PATH):
    lib = ctypes.CDLL(path)
    i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    vp = ctypes.c_void_p
    lib.hisa_oracle_block_pool.argtypes = [_u16, i64, i32, i32, _f64]
    lib.hisa_oracle_block_pool.restype = None
    lib.hisa_oracle_block_topm.argtypes = [_u16, vp, i32, _f64, i32, i32, i64, i32, _i32, vp]
    lib.hisa_oracle_block_topm.restype = i32
    lib.hisa_oracle_token_topk.argtypes = [_u16, vp, i32, _u16, i32, i32, i64, i64, _i32, i32, i32, _i32, vp, vp]
    lib.hisa_oracle_token_topk.restype = i32
    lib.hisa_oracle_flat_topk.argtypes = [_u16, vp, i32, _u16, i32, i64, i32, _i32, vp]
    lib.hisa_oracle_flat_topk.restype = i32
    lib.hisa_oracle_sparse_attn.argtypes = [_u16, _u16, _u16, i32, i32, i32, dbl, _i32, i32, _f64, _f64]
    lib.hisa_oracle_sparse_attn.restype = None
    lib.hisa_oracle_run.argtypes = [i32, i64, i64, i32, i32, i32, i32, i32, i32, i32, dbl, i32, vp,
                                    _u16, _u16, _f64, vp, vp, vp, _i64, i64, vp, _i32, vp, vp, vp, i32]
    lib.hisa_oracle_run.restype = i32
    lib.hisa_oracle_threads.restype = i32
    lib.hisa_oracle_set_threads.argtypes = [i32]
    return lib


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load()
    return _lib


def _heads(q_row, w):
    """(q rows as [n_heads][d_idx] or [d_idx], weights as fp64 or None, n_idx_heads)."""
    q_row = np.ascontiguousarray(q_row, dtype=np.uint16)
    if w is None:
        return q_row.reshape(-1), None, 0
    w = np.ascontiguousarray(w, dtype=np.float64).reshape(-1)
    return q_row.reshape(-1), w, len(w)


class Oracle:
    """Thin numpy wrapper over one loaded oracle library (the real one or a test variant).

    The indexer calls take ``w``: None for the plain dot-product score, or the
    query's head weights [H] with ``q_row`` [H][d_idx] for the multi-head score."""

    def __init__(self, handle=None):
        self.L = handle if handle is not None else lib()

    # -- step 1
    def block_pool(self, k_idx: np.ndarray, block: int) -> np.ndarray:
        k_idx = np.ascontiguousarray(k_idx, dtype=np.uint16)
        n_kv, d = k_idx.shape
        out = np.empty((-(-n_kv // block), d), dtype=np.float64)
        self.L.hisa_oracle_block_pool(k_idx, n_kv, d, block, out)
        return out

    # -- steps 2-3
    def block_topm(self, q_row, block_keys, block: int, p: int, top_m: int, scores: bool = False, w=None):
        q_row, w, nh = _heads(q_row, w)
        bk = np.ascontiguousarray(block_keys, dtype=np.float64)
        sel = np.empty(top_m, dtype=np.int32)
        sc = np.empty(top_m, dtype=np.float64) if scores else None
        s = self.L.hisa_oracle_block_topm(q_row, w.ctypes.data if nh else None, nh, bk, bk.shape[-1], block, p,
                                          top_m, sel, sc.ctypes.data if scores else None)
        return (sel, s, sc) if scores else (sel, s)

    # -- steps 4-5
    def token_topk(self, q_row, k_idx, block: int, p: int, sel, top_k: int, scores: bool = False, w=None):
        q_row, w, nh = _heads(q_row, w)
        k_idx = np.ascontiguousarray(k_idx, dtype=np.uint16)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        tok = np.empty(top_k, dtype=np.int32)
        sc = np.empty(top_k, dtype=np.float64) if scores else None
        nc = ctypes.c_int64(0)
        k_eff = self.L.hisa_oracle_token_topk(q_row, w.ctypes.data if nh else None, nh, k_idx, k_idx.shape[1],
                                              block, k_idx.shape[0], p, sel, len(sel), top_k, tok,
                                              sc.ctypes.data if scores else None, ctypes.addressof(nc))
        return (tok, k_eff, nc.value, sc) if scores else (tok, k_eff, nc.value)

    def flat_topk(self, q_row, k_idx, p: int, top_k: int, scores: bool = False, w=None):
        q_row, w, nh = _heads(q_row, w)
        k_idx = np.ascontiguousarray(k_idx, dtype=np.uint16)
        tok = np.empty(top_k, dtype=np.int32)
        sc = np.empty(top_k, dtype=np.float64) if scores else None
        k_eff = self.L.hisa_oracle_flat_topk(q_row, w.ctypes.data if nh else None, nh, k_idx, k_idx.shape[1], p,
                                             top_k, tok, sc.ctypes.data if scores else None)
        return (tok, k_eff, sc) if scores else (tok, k_eff)

    # -- step 6
    def sparse_attn(self, q_row, k, v, tok, scale: float | None = None):
        """q_row [H][d]; k, v [n][H_kv][d] addressed by token id; returns (o [H][d], lse [H])."""
        q_row = np.ascontiguousarray(q_row, dtype=np.uint16)
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        tok = np.ascontiguousarray(tok, dtype=np.int32)
        h, d = q_row.shape
        hkv = k.shape[1]
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        o = np.empty((h, d), dtype=np.float64)
        lse = np.empty(h, dtype=np.float64)
        self.L.hisa_oracle_sparse_attn(q_row, k, v, h, hkv, d, scale, tok, len(tok), o, lse)
        return o, lse

    # -- whole path over a list of queries
    def run(self, w, inputs: dict, query_ids=None, flat: bool = False, attention: bool = True,
            block_keys=None, scale: float | None = None):
        """Oracle outputs for ``query_ids`` (seq * n_q + i) of workload ``w``.

        ``inputs`` holds uint16 bf16 arrays q_idx [b][n_q][d_idx] ([b][n_q][H_idx][d_idx] with a
        multi-head indexer, whose head weights ``w_idx`` [b][n_q][H_idx] come along), k_idx
        [b][n_kv][d_idx] and, for attention, q [b][n_q][H][d], k, v [b][n_kv][H_kv][d].
        """
        if query_ids is None:
            query_ids = np.arange(w.batch * w.n_q, dtype=np.int64)
        query_ids = np.ascontiguousarray(query_ids, dtype=np.int64)
        nq = len(query_ids)
        q_idx = np.ascontiguousarray(inputs["q_idx"], dtype=np.uint16)
        k_idx = np.ascontiguousarray(inputs["k_idx"], dtype=np.uint16)
        if block_keys is None:
            block_keys = np.stack([self.block_pool(k_idx[s], w.block) for s in range(w.batch)])
        block_keys = np.ascontiguousarray(block_keys, dtype=np.float64)
        blk = np.full((nq, w.top_m), -7, dtype=np.int32)
        tok = np.empty((nq, w.top_k), dtype=np.int32)
        ncand = np.empty(nq, dtype=np.int64)
        o = lse = None
        qa = ka = va = None
        if attention:
            qa = np.ascontiguousarray(inputs["q"], dtype=np.uint16)
            ka = np.ascontiguousarray(inputs["k"], dtype=np.uint16)
            va = np.ascontiguousarray(inputs["v"], dtype=np.uint16)
            o = np.empty((nq, w.n_heads, w.d_head), dtype=np.float64)
            lse = np.empty((nq, w.n_heads), dtype=np.float64)
        if scale is None:
            scale = 1.0 / math.sqrt(w.d_head)
        ptr = lambda a: a.ctypes.data if a is not None else None  # noqa: E731
        nh = getattr(w, "n_idx_heads", 0)
        wi = np.ascontiguousarray(inputs["w_idx"], dtype=np.float64) if nh else None
        rc = self.L.hisa_oracle_run(w.batch, w.n_q, w.n_kv, w.d_idx, w.block, w.top_m, w.top_k, w.n_heads,
                                    w.n_kv_heads, w.d_head, scale, nh, ptr(wi), q_idx, k_idx, block_keys,
                                    ptr(qa), ptr(ka),
                                    ptr(va), query_ids, nq, blk.ctypes.data, tok, ptr(o), ptr(lse),
                                    ncand.ctypes.data, 1 if flat else 0)
        if rc != 0:
            raise ValueError("hisa_oracle_run: query id out of range")
        out = {"token_idx": tok, "n_cand": ncand, "block_keys": block_keys}
        if not flat:
            out["block_idx"] = blk
        if attention:
            out["o"], out["lse"] = o, lse
        return out

    def threads(self) -> int:
        return int(self.L.hisa_oracle_threads())

    def set_threads(self, n: int):
        self.L.hisa_oracle_set_threads(int(n))
