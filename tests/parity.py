"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and the oracle on
the same seeded inputs, and compare them."""
from __future__ import annotations

import math

import numpy as np

from synth.workloads import Workload, k_idx_rows, k_rows, q_idx_rows, q_rows, v_rows

# Attention tolerance, elementwise: |gpu - oracle| <= ATOL + RTOL * |oracle| (bf16 inputs,
# fp32 accumulation, bf16 output rounding of at most 2^-9 relative).
ATOL, RTOL = 2e-3, 1e-2


def dev_inputs(inp: dict, device="cuda") -> dict:
    """Host inputs on the device: bf16 bit arrays as bf16 tensors, the fp32 head weights as fp32."""
    import torch

    out = {}
    for k, v in inp.items():
        if k.startswith("_"):
            continue
        out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(device) if v.dtype == np.float32 else to_dev(v, device)
    return out


def to_dev(a_u16: np.ndarray, device="cuda"):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_to_f64(t) -> np.ndarray:
    import torch

    return t.float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 else t.cpu().numpy()


def assert_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bad = ~(np.abs(gpu - ref) <= ATOL + RTOL * np.abs(ref))
    both_ninf = np.isneginf(gpu) & np.isneginf(ref)
    bad &= ~both_ninf
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance, e.g. at {idx.tolist()}: "
                             f"gpu={gpu[tuple(idx[0])]} ref={ref[tuple(idx[0])]}")


def run_stages(hs, w: Workload, dev: dict, attention=True):
    """Stage-by-stage run through the C ABI.  Returns the intermediates as torch tensors."""
    import torch

    p = hs.params_of(w)
    d = dev["q_idx"].device
    bk = torch.empty((w.batch, w.n_blk, w.d_idx), dtype=torch.float32, device=d)
    hs.hisa_block_pool(p, dev["k_idx"], bk)
    status = torch.zeros(1, dtype=torch.int32, device=d)
    blk = torch.empty((w.batch, w.n_q, w.top_m), dtype=torch.int32, device=d)
    bsc = torch.empty((w.batch, w.n_q, w.top_m), dtype=torch.float32, device=d)
    wi = dev.get("w_idx")  # the indexer's head weights (multi-head indexer only)
    hs.hisa_block_topm(p, dev["q_idx"], bk, blk, bsc, status, idx_weights=wi)
    tok = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.int32, device=d)
    tsc = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.float32, device=d)
    hs.hisa_token_topk(p, dev["q_idx"], dev["k_idx"], blk, tok, tsc, status, idx_weights=wi)
    out = {"block_keys": bk, "block_idx": blk, "block_scores": bsc, "token_idx": tok, "token_scores": tsc,
           "status": status}
    if attention:
        o = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16, device=d)
        lse = torch.empty((w.batch, w.n_q, w.n_heads), dtype=torch.float32, device=d)
        hs.sparse_attn_fwd(p, dev["q"], dev["k"], dev["v"], tok, o, lse, status)
        out["o"], out["lse"] = o, lse
    torch.cuda.synchronize()
    return out


def run_forward(hs, w: Workload, dev: dict):
    import torch

    p = hs.params_of(w)
    d = dev["q_idx"].device
    o = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16, device=d)
    lse = torch.empty((w.batch, w.n_q, w.n_heads), dtype=torch.float32, device=d)
    blk = torch.empty((w.batch, w.n_q, w.top_m), dtype=torch.int32, device=d)
    tok = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.int32, device=d)
    status = torch.zeros(1, dtype=torch.int32, device=d)
    hs.hisa_forward(p, dev["q_idx"], dev["k_idx"], dev["q"], dev["k"], dev["v"], o, lse, blk, tok, status,
                    idx_weights=dev.get("w_idx"))
    torch.cuda.synchronize()
    return {"o": o, "lse": lse, "block_idx": blk, "token_idx": tok, "status": status}


class SampledOracle:
    """The oracle on single queries of a large workload, regenerating only the rows it needs."""

    def __init__(self, O, w: Workload):
        self.O, self.w = O, w
        self._seq = None

    def _load_seq(self, seq):
        if self._seq != seq:
            self.k_idx = k_idx_rows(self.w, seq, 0, self.w.n_kv)
            self.bk = self.O.block_pool(self.k_idx, self.w.block)
            self._seq = seq

    def query(self, seq: int, i: int, attention=True):
        w = self.w
        self._load_seq(seq)
        p = w.n_kv - w.n_q + i
        qi = q_idx_rows(w, seq, i, 1)[0]
        sel, s = self.O.block_topm(qi, self.bk, w.block, p, w.top_m)
        tok, k_eff, n_cand = self.O.token_topk(qi, self.k_idx, w.block, p, sel, w.top_k)
        out = {"block_idx": sel, "token_idx": tok, "k_eff": k_eff, "n_cand": n_cand}
        if attention:
            valid = tok[tok >= 0]
            kk = k_rows(w, seq, valid)
            vv = v_rows(w, seq, valid)
            remap = np.full(w.top_k, -1, dtype=np.int32)
            remap[: len(valid)] = np.arange(len(valid), dtype=np.int32)
            o, lse = self.O.sparse_attn(q_rows(w, seq, i, 1)[0], kk, vv, remap, 1.0 / math.sqrt(w.d_head))
            out["o"], out["lse"] = o, lse
        return out
