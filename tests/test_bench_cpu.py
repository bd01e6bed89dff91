"""The bench's own accounting, on the CPU: its closed-form candidate and kept-token counts (which
set the attention kernel's algorithmic bytes and the roofline) must equal what the oracle counts
query by query, and the byte formulas must follow the tensor shapes."""
import importlib.util
import os

import numpy as np
import pytest

from synth.workloads import Workload, full_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


CASES = [
    Workload("counts_prefill", 1, 700, 700, 64, 32, 5, 100, 2, 2, 64),
    Workload("counts_context", 2, 300, 1000, 64, 64, 4, 150, 2, 1, 64),  # queries after a context prefix
    Workload("counts_all_blocks", 1, 200, 200, 64, 16, 64, 64, 1, 1, 64),  # m covers every block
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_closed_form_counts_match_the_oracle(bench, oracle_lib, w):
    inp = full_inputs(w)
    n_cand = k_eff = n_vis = 0
    for seq in range(w.batch):
        bk = oracle_lib.block_pool(inp["k_idx"][seq], w.block)
        for i in range(w.n_q):
            p = w.n_kv - w.n_q + i
            sel, _ = oracle_lib.block_topm(inp["q_idx"][seq, i], bk, w.block, p, w.top_m)
            _, ke, nc = oracle_lib.token_topk(inp["q_idx"][seq, i], inp["k_idx"][seq], w.block, p,
                                             sel[sel >= 0], w.top_k)
            n_cand += nc
            k_eff += ke
            n_vis += p // w.block + 1
    counts = bench.closed_form_counts(w)
    assert counts == {"n_cand": n_cand, "k_eff": k_eff, "n_vis": n_vis}


def test_byte_formulas(bench):
    w = Workload("bytes", 2, 300, 1000, 64, 64, 4, 150, 8, 2, 128)
    c = bench.closed_form_counts(w)
    nq = w.batch * w.n_q
    # every kept token's K and V rows once per KV head, plus Q and O rows, LSE and the index lists
    assert bench.attention_bytes(w, c) == (c["k_eff"] * 2 * 128 * 2 * 2 + nq * 8 * 128 * 2 * 2 + nq * 8 * 4
                                           + nq * 150 * 4)
    # every input once, every output once
    assert bench.compulsory_bytes(w) == (2 * 1000 * 64 * 2 + nq * 64 * 2 + 2 * 1000 * 2 * 128 * 2 * 2
                                         + nq * 8 * 128 * 2 * 2 + nq * 8 * 4)
    wm = w.with_(n_idx_heads=4)
    assert bench.compulsory_bytes(wm) - bench.compulsory_bytes(w) == nq * 3 * 64 * 2 + nq * 4 * 4


def test_workload_config_names_the_workload(bench):
    w = Workload("cfg", 2, 300, 1000, 64, 64, 4, 150, 8, 2, 128, n_idx_heads=4, needles=3)
    c = bench.workload_config(w)
    assert c == {"workload": "cfg", "batch": 2, "n_q": 300, "n_kv": 1000, "d_idx": 64, "block": 64, "top_m": 4,
                 "top_k": 150, "n_heads": 8, "n_kv_heads": 2, "d_head": 128, "n_idx_heads": 4, "needles": 3}


@pytest.mark.parametrize("shape", [(1, 300, 300), (3, 200, 777), (1, 65536, 65536), (2, 129, 1000)])
def test_qtile_flops_count_every_visible_key_tile(bench, shape):
    """The query-tile kernel's flops: 4 * 128^3 per (query tile, visible key tile, head), the visible
    key tiles of a query tile being those up to its last query's position; checked against a count
    over the queries themselves."""
    b, n_q, n_kv = shape
    w = Workload("tiles", b, n_q, n_kv, 64, 64, 4, 64, 3, 3, 128)
    fl, tiles = bench.qtile_flops(w)
    pos = n_kv - n_q + np.arange(n_q)
    last_tile = {}
    for i, p in enumerate(pos):
        last_tile[i // 128] = max(last_tile.get(i // 128, -1), p // 128)
    want = sum(t + 1 for t in last_tile.values()) * b * 3
    assert tiles == want and fl == want * 4 * 128 ** 3
