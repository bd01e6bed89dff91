"""Decode with the context split across ranks, host logic on CPU: two and three gloo ranks run
`context_parallel.decode_step` (its exchanges are real all-gathers) with per-rank phases written
here from the oracle and numpy, and must reproduce the oracle's answer for the whole context:
the same blocks and tokens, bit for bit, and the same attention output within fp64 rounding.
This pins the decomposition itself (local best -> union -> global best, log-sum-exp merge) and
the exchange order; the CUDA phases are checked against the oracle on a GPU in
test_context_parallel_gpu.py."""
import math
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

from synth.workloads import Workload, full_inputs  # noqa: E402

W = Workload("cp_decode_cpu", 2, 1, 3000, 64, 64, 6, 150, 4, 2, 64, needles=3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bf16(a):
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class OraclePhases:
    """The per-rank phases of a step, from the oracle (test infrastructure) and numpy."""

    def __init__(self, oracle, w):
        self.O, self.w = oracle, w

    def blocks(self, pl, shard, q_idx, k_idx, idx_weights=None):
        w = self.w
        m, c = w.top_m, (shard.n_kv_global - 1) // w.block
        scores = np.full((w.batch, m), np.nan, dtype=np.float32)
        ids = np.full((w.batch, m), -1, dtype=np.int32)
        for s in range(w.batch):
            bk = self.O.block_pool(k_idx[s], w.block)  # this rank's block means
            sc = bk @ _bf16(q_idx[s, 0])
            g = shard.first_block + np.arange(len(bk))
            forced = (g == 0) | (g == c)
            cand = (g >= 1) & (g < c)
            order = np.lexsort((g[cand], -sc[cand]))[: m - 2]
            keep = np.concatenate([g[forced], g[cand][order]])
            vals = np.concatenate([np.full(forced.sum(), np.inf), sc[cand][order]])
            o = np.argsort(keep)
            scores[s, : len(keep)], ids[s, : len(keep)] = vals[o], keep[o]
        return torch.from_numpy(scores), torch.from_numpy(ids)

    def merge(self, scores_all, ids_all, k):
        sc = scores_all.numpy().transpose(1, 0, 2).reshape(scores_all.shape[1], -1)
        ids = ids_all.numpy().transpose(1, 0, 2).reshape(ids_all.shape[1], -1)
        out = np.full((sc.shape[0], k), -1, dtype=np.int32)
        for r in range(sc.shape[0]):
            v = ids[r] >= 0
            order = np.lexsort((ids[r][v], -sc[r][v].astype(np.float64)))[:k]
            out[r, : len(order)] = np.sort(ids[r][v][order])
        return torch.from_numpy(out), None

    def tokens(self, pl, shard, q_idx, k_idx, block_idx, status=None, idx_weights=None):
        w = self.w
        scores = np.full((w.batch, w.top_k), np.nan, dtype=np.float32)
        ids = np.full((w.batch, w.top_k), -1, dtype=np.int32)
        for s in range(w.batch):
            g = block_idx[s].numpy()
            mine = g[(g >= shard.first_block) & (g < shard.first_block + shard.n_blk)] - shard.first_block
            tok, k_eff, _, sc = self.O.token_topk(q_idx[s, 0], k_idx[s], w.block, shard.n_loc - 1, mine, w.top_k,
                                                  scores=True)
            ids[s, :k_eff] = tok[:k_eff] + shard.t0
            scores[s, :k_eff] = sc[:k_eff]
        return torch.from_numpy(scores), torch.from_numpy(ids)

    def attention(self, pl, shard, q, k, v, token_idx, status=None):
        w = self.w
        o = np.zeros((w.batch, w.n_heads, w.d_head))
        lse = np.full((w.batch, w.n_heads), -np.inf)
        for s in range(w.batch):
            t = token_idx[s].numpy()
            t = t[(t >= shard.t0) & (t < shard.t0 + shard.n_loc)] - shard.t0
            if len(t):
                o[s], lse[s] = self.O.sparse_attn(q[s, 0], k[s], v[s], t)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def lse_merge(self, o_all, lse_all):
        o_all, lse_all = o_all.numpy(), lse_all.numpy()
        L = lse_all.max(axis=0)
        wgt = np.exp(lse_all - L)
        s = wgt.sum(axis=0)
        return (wgt[..., None] * o_all).sum(axis=0) / s[..., None], L + np.log(s)


def _rank_main(rank, world, port, out):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import hierarchical_sparse_attention_block_b200 as hs
        import hierarchical_sparse_attention_block_b200.context_parallel as cp
        from oracle import Oracle

        inp = full_inputs(W)
        sh = cp.Shard.even(W.n_kv, W.block, rank, world)
        sl = slice(sh.t0, sh.t0 + sh.n_loc)
        blk, tok, o, lse = cp.decode_step(hs.params_of(W), sh, inp["q_idx"], inp["k_idx"][:, sl], inp["k_idx"][:, sl],
                                          inp["q"], inp["k"][:, sl], inp["v"][:, sl], cp.all_gather_exchange(),
                                          phases=OraclePhases(Oracle(), W))
        out[rank] = (blk.numpy(), tok.numpy(), np.asarray(o), np.asarray(lse), sh.t0, sh.n_loc)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])  # 47 blocks: uneven shards, the last one ending on a partial block
def test_split_context_decode_matches_whole_context(world):
    from oracle import Oracle

    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    ref = Oracle().run(W, full_inputs(W))
    spans = sorted((v[4], v[5]) for v in out.values())
    assert spans[0][0] == 0 and sum(n for _, n in spans) == W.n_kv  # the ranks tile the context
    for r in range(world):
        blk, tok, o, lse = out[r][:4]
        assert np.array_equal(blk, ref["block_idx"])
        assert np.array_equal(tok, ref["token_idx"])
        assert np.allclose(o, ref["o"], rtol=1e-9, atol=1e-12)
        assert np.allclose(lse, ref["lse"], rtol=1e-12, atol=1e-12)
        assert not math.isnan(float(lse.sum()))
