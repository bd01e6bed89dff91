"""The five workloads (shapes, sizes, seeds) and host-side builders for their inputs.

Shapes follow the two-level indexer's problem statement: one indexer head
(``d_idx``), fixed key blocks of ``block`` tokens, ``top_m`` blocks and
``top_k`` tokens per query, and multi-head attention over the selected tokens.
Queries are the last ``n_q`` positions of each sequence (prefill: n_q = n_kv;
decode: n_q = 1).  Needle blocks stand in for the needle-in-a-haystack probes
the pages evaluate with: the keys of a few random blocks are shifted toward
the sign pattern of the probe query (the last query of each sequence).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

from . import (T_K, T_KIDX, T_Q, T_QIDX, T_V, T_WIDX, apply_needles, int_bf16, int_values, weight_values,
               needle_blocks, needle_signs, normal_bf16)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int
    n_kv: int
    d_idx: int
    block: int
    top_m: int
    top_k: int
    n_heads: int
    n_kv_heads: int
    d_head: int
    needles: int = 0
    seed: int = 0
    n_idx_heads: int = 0  # 0: one indexer head scored by a plain dot product; H >= 1: H heads, weighted ReLU

    @property
    def n_blk(self) -> int:
        return -(-self.n_kv // self.block)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_prefill_1k": Workload("tiny_prefill_1k", 1, 1024, 1024, 64, 64, 4, 128, 1, 1, 64),
    "prefill_8k": Workload("prefill_8k", 1, 8192, 8192, 128, 128, 16, 512, 8, 8, 128, needles=8),
    "prefill_64k": Workload("prefill_64k", 1, 65536, 65536, 128, 128, 64, 2048, 16, 16, 128, needles=64),
    "decode_32x128k": Workload("decode_32x128k", 32, 1, 131072, 128, 128, 64, 2048, 16, 16, 128),
    "decode_4x1m_m32": Workload("decode_4x1m_m32", 4, 1, 1048576, 128, 256, 32, 4096, 16, 16, 128, needles=256),
    "decode_4x1m_m64": Workload("decode_4x1m_m64", 4, 1, 1048576, 128, 256, 64, 4096, 16, 16, 128, needles=256),
    "decode_4x1m_m128": Workload("decode_4x1m_m128", 4, 1, 1048576, 128, 256, 128, 4096, 16, 16, 128, needles=256),
}


def q_idx_rows(w: Workload, seq: int, i0: int, count: int) -> np.ndarray:
    """bf16 bits of q_idx[seq][i0:i0+count] -> uint16 [count][d_idx] ([count][H_idx][d_idx] with a
    multi-head indexer)."""
    nh = max(1, w.n_idx_heads)
    start = (seq * w.n_q + i0) * nh * w.d_idx
    rows = int_bf16(w.seed, T_QIDX, start, count * nh * w.d_idx)
    return rows.reshape(count, w.d_idx) if w.n_idx_heads == 0 else rows.reshape(count, nh, w.d_idx)


def w_idx_rows(w: Workload, seq: int, i0: int, count: int) -> np.ndarray:
    """Indexer head weights [count][H_idx] (fp32) of queries i0 .. i0+count-1."""
    return weight_values(w.seed, T_WIDX, (seq * w.n_q + i0) * w.n_idx_heads,
                         count * w.n_idx_heads).reshape(count, w.n_idx_heads)


def probe_signs(w: Workload, seq: int) -> np.ndarray:
    q = q_idx_rows(w, seq, w.n_q - 1, 1)[0]
    return needle_signs(q if q.ndim == 1 else q[0])  # a multi-head indexer: its first head


def needle_table(w: Workload, seq: int) -> np.ndarray:
    if w.needles <= 0:
        return np.zeros(0, dtype=np.int32)
    return needle_blocks(w.seed, seq, w.n_blk, w.needles)


def k_idx_rows_int(w: Workload, seq: int, t0: int, count: int) -> np.ndarray:
    """Integer values of k_idx[seq][t0:t0+count], needles applied -> int8 [count][d_idx]."""
    start = (seq * w.n_kv + t0) * w.d_idx
    vals = int_values(w.seed, T_KIDX, start, count * w.d_idx).reshape(count, w.d_idx)
    nb = needle_table(w, seq)
    if len(nb):
        tok = np.arange(t0, t0 + count)
        hit = np.isin(tok // w.block, nb)
        if hit.any():
            vals[hit] = apply_needles(vals[hit], probe_signs(w, seq))
    return vals


def int8_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    # Small integers are exact in bf16: the fp32 bit pattern's top half.
    return (v.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def k_idx_rows(w: Workload, seq: int, t0: int, count: int) -> np.ndarray:
    return int8_to_bf16_bits(k_idx_rows_int(w, seq, t0, count))


def q_rows(w: Workload, seq: int, i0: int, count: int) -> np.ndarray:
    """bf16 bits of Q[seq][i0:i0+count] -> uint16 [count][H][d]."""
    per = w.n_heads * w.d_head
    start = (seq * w.n_q + i0) * per
    return normal_bf16(w.seed, T_Q, start, count * per).reshape(count, w.n_heads, w.d_head)


def _kv_rows(w: Workload, tensor: int, seq: int, tokens: np.ndarray) -> np.ndarray:
    per = w.n_kv_heads * w.d_head
    tokens = np.asarray(tokens, dtype=np.int64)
    out = np.empty((len(tokens), w.n_kv_heads, w.d_head), dtype=np.uint16)
    # Contiguous runs are generated in one call each.
    if len(tokens) == 0:
        return out
    order = np.argsort(tokens, kind="stable")
    st = tokens[order]
    breaks = np.nonzero(np.diff(st) != 1)[0] + 1
    for run in np.split(np.arange(len(st)), breaks):
        t0 = int(st[run[0]])
        rows = normal_bf16(w.seed, tensor, (seq * w.n_kv + t0) * per, len(run) * per)
        out[order[run]] = rows.reshape(len(run), w.n_kv_heads, w.d_head)
    return out


def k_rows(w: Workload, seq: int, tokens) -> np.ndarray:
    return _kv_rows(w, T_K, seq, tokens)


def v_rows(w: Workload, seq: int, tokens) -> np.ndarray:
    return _kv_rows(w, T_V, seq, tokens)


def full_inputs(w: Workload) -> dict:
    """All inputs of a (small) workload on the host as uint16 bf16 bit arrays."""
    q_idx = np.stack([q_idx_rows(w, s, 0, w.n_q) for s in range(w.batch)])
    k_idx = np.stack([k_idx_rows(w, s, 0, w.n_kv) for s in range(w.batch)])
    q = np.stack([q_rows(w, s, 0, w.n_q) for s in range(w.batch)])
    allt = np.arange(w.n_kv)
    k = np.stack([k_rows(w, s, allt) for s in range(w.batch)])
    v = np.stack([v_rows(w, s, allt) for s in range(w.batch)])
    out = {"q_idx": q_idx, "k_idx": k_idx, "q": q, "k": k, "v": v}
    if w.n_idx_heads:
        out["w_idx"] = np.stack([w_idx_rows(w, s, 0, w.n_q) for s in range(w.batch)])
    return out
