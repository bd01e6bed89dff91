"""Build a workload's inputs directly in device memory with the device generator.

The tensors are bit-identical to the host builders in ``synth.workloads``; the
large decode caches (tens of GiB) are therefore never generated on the host.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import T_K, T_KIDX, T_Q, T_QIDX, T_V
from .workloads import Workload, needle_table, probe_signs, w_idx_rows

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth.cu")
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(src):
        cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", src, "-o", LIB_PATH]
        subprocess.run(cmd, check=True)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run synth.device.build()")
        _lib = ctypes.CDLL(LIB_PATH)
        i64, u64, u32, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_void_p
        for name in ("synth_fill_int_bf16", "synth_fill_normal_bf16"):
            f = getattr(_lib, name)
            f.argtypes = [vp, i64, u64, u32, i64, vp]
            f.restype = ctypes.c_int
        _lib.synth_plant_needles.argtypes = [vp, ctypes.c_int32, i64, ctypes.c_int32, ctypes.c_int32, vp,
                                             ctypes.c_int32, vp, vp]
        _lib.synth_plant_needles.restype = ctypes.c_int
        _lib.synth_raw_u64.argtypes = [u64, u32, i64]
        _lib.synth_raw_u64.restype = u64
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with CUDA error {rc}")


def _stream_ptr(stream) -> int:
    return int(stream.cuda_stream) if stream is not None else 0


def fill_int(t, seed: int, tensor: int, start: int = 0, stream=None):
    _check(lib().synth_fill_int_bf16(t.data_ptr(), t.numel(), seed, tensor, start, _stream_ptr(stream)),
           "synth_fill_int_bf16")


def fill_normal(t, seed: int, tensor: int, start: int = 0, stream=None):
    _check(lib().synth_fill_normal_bf16(t.data_ptr(), t.numel(), seed, tensor, start, _stream_ptr(stream)),
           "synth_fill_normal_bf16")


def device_inputs(w: Workload, device="cuda", with_attention: bool = True, stream=None) -> dict:
    """Allocate and fill q_idx, k_idx (needles planted) and, optionally, Q, K, V on ``device``."""
    import torch

    bf = torch.bfloat16
    q_shape = (w.batch, w.n_q, w.d_idx) if w.n_idx_heads == 0 else (w.batch, w.n_q, w.n_idx_heads, w.d_idx)
    out = {
        "q_idx": torch.empty(q_shape, dtype=bf, device=device),
        "k_idx": torch.empty((w.batch, w.n_kv, w.d_idx), dtype=bf, device=device),
    }
    fill_int(out["q_idx"], w.seed, T_QIDX, 0, stream)
    if w.n_idx_heads:
        # the indexer's head weights: few values, generated on the host half of the generator
        wts = np.stack([w_idx_rows(w, s, 0, w.n_q) for s in range(w.batch)])
        out["w_idx"] = torch.from_numpy(wts).to(device)
    fill_int(out["k_idx"], w.seed, T_KIDX, 0, stream)
    if w.needles > 0:
        tables = np.stack([needle_table(w, s) for s in range(w.batch)]).astype(np.int32)
        signs = np.stack([probe_signs(w, s) for s in range(w.batch)]).astype(np.int8)
        d_tab = torch.from_numpy(tables).to(device)
        d_sg = torch.from_numpy(signs).to(device)
        _check(lib().synth_plant_needles(out["k_idx"].data_ptr(), w.batch, w.n_kv, w.d_idx, w.block,
                                         d_tab.data_ptr(), tables.shape[1], d_sg.data_ptr(),
                                         _stream_ptr(stream)), "synth_plant_needles")
        out["_needles"] = tables
        torch.cuda.synchronize()
    if with_attention:
        out["q"] = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=bf, device=device)
        out["k"] = torch.empty((w.batch, w.n_kv, w.n_kv_heads, w.d_head), dtype=bf, device=device)
        out["v"] = torch.empty((w.batch, w.n_kv, w.n_kv_heads, w.d_head), dtype=bf, device=device)
        fill_normal(out["q"], w.seed, T_Q, 0, stream)
        fill_normal(out["k"], w.seed, T_K, 0, stream)
        fill_normal(out["v"], w.seed, T_V, 0, stream)
    return out
