"""Decode with the context split across ranks, on one GPU: G ranks run as host threads, each
calling `context_parallel.decode_step` with the CUDA phases on its slice of the caches; the
exchange stacks the ranks' tensors in rank order (what an all-gather returns).  No kernel waits
on another: the threads meet on the host only.  The result must be the oracle's for the whole
context (blocks and tokens bit for bit, attention within the parity tolerance) and the same
selections as the one-GPU path."""
import threading

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from parity import assert_close, dev_inputs, run_stages, to_dev  # noqa: E402
from synth.workloads import Workload, full_inputs  # noqa: E402


@pytest.fixture(scope="module")
def hs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as m

    return m


def _run_ranks(hs, w, inp, world):
    import hierarchical_sparse_attention_block_b200.context_parallel as cp

    p = hs.params_of(w)
    barrier = threading.Barrier(world)
    slots = [None] * world
    results, errors = [None] * world, []

    def exchange_of(r):
        def exchange(t):
            slots[r] = t
            barrier.wait()
            out = torch.stack(list(slots))
            barrier.wait()  # nobody refills a slot before everyone has stacked
            return out

        return exchange

    def worker(r):
        try:
            sh = cp.Shard.even(w.n_kv, w.block, r, world)
            sl = slice(sh.t0, sh.t0 + sh.n_loc)
            q_idx, q = to_dev(inp["q_idx"]), to_dev(inp["q"])
            k_idx, k, v = (to_dev(np.ascontiguousarray(inp[n][:, sl])) for n in ("k_idx", "k", "v"))
            pl = cp.local_params(p, sh)
            bk = torch.empty((w.batch, sh.n_blk, w.d_idx), dtype=torch.float32, device="cuda")
            hs.hisa_block_pool(pl, k_idx, bk)
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            wi = torch.from_numpy(inp["w_idx"]).cuda() if w.n_idx_heads else None
            blk, tok, o, lse = cp.decode_step(p, sh, q_idx, k_idx, bk, q, k, v, exchange_of(r), status=status,
                                              idx_weights=wi)
            torch.cuda.synchronize()
            results[r] = (blk.cpu().numpy(), tok.cpu().numpy(), o.float().cpu().numpy(), lse.cpu().numpy(),
                          int(status.item()))
        except BaseException as e:  # noqa: BLE001
            errors.append(e)
            barrier.abort()

    threads = [threading.Thread(target=worker, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errors:
        raise errors[0]
    return results


CASES = [
    # name, batch, n_q, n_kv, d_idx, block, top_m, top_k, n_heads, n_kv_heads, d_head
    (Workload("cp_mha", 2, 1, 20000, 64, 64, 8, 300, 4, 4, 128, needles=4), 3),
    (Workload("cp_gqa", 3, 1, 9000, 128, 128, 6, 500, 8, 2, 128), 2),
    (Workload("cp_all_blocks", 1, 1, 2500, 64, 64, 64, 2000, 2, 2, 64), 4),
    (Workload("cp_one_rank", 2, 1, 5000, 64, 64, 8, 300, 4, 4, 64), 1),
    (Workload("cp_multihead_indexer", 2, 1, 7000, 64, 64, 8, 300, 4, 4, 64, n_idx_heads=4), 3),
]


@pytest.mark.parametrize("w,world", CASES, ids=[c[0].name for c in CASES])
def test_split_context_decode_matches_oracle(hs, oracle_lib, w, world):
    inp = full_inputs(w)
    ref = oracle_lib.run(w, inp)
    one = run_stages(hs, w, dev_inputs(inp))
    n = w.batch
    for blk, tok, o, lse, status in _run_ranks(hs, w, inp, world):
        assert status == 0
        assert np.array_equal(blk, ref["block_idx"])
        assert np.array_equal(tok, ref["token_idx"])
        assert np.array_equal(tok, one["token_idx"].cpu().numpy().reshape(n, w.top_k))
        assert_close(o.reshape(n, w.n_heads, w.d_head), ref["o"], "o")
        assert_close(lse.reshape(n, w.n_heads), ref["lse"], "lse")
