"""GPU parity of step 6 for many queries per sequence: the query-tile tensor-core kernel (tiles of
128 queries against tiles of 128 keys, the selections as bit masks) and the gather kernels it
replaces, both against the oracle's attention on the same token lists.

The lists are built here (seeded), not by the indexer, so that the cases the query-tile kernel
special-cases come up on purpose: ragged query tiles, several sequences, query positions that do
not start at a tile boundary (chunked prefill), heads sharing K/V, empty rows, rows whose scores
grow along the sequence (the running max is raised late and the accumulator rescaled), and lists
with malformed entries.  Tolerance: |gpu - oracle| <= 2e-3 + 1e-2 |oracle|.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from parity import assert_close, to_dev  # noqa: E402
from synth import T_K, T_Q, T_V, normal_bf16  # noqa: E402
from synth.workloads import Workload  # noqa: E402


@pytest.fixture(scope="module")
def hs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as m

    return m


def _inputs(w, seed=5, k_growth=0.0):
    """Q, K, V bf16 bits; with k_growth > 0 the K rows are scaled by 1 + k_growth * t / n_kv, so later
    keys score higher and the running max of a row keeps rising."""
    nq, nkv = w.batch * w.n_q, w.batch * w.n_kv
    q = normal_bf16(seed, T_Q, 0, nq * w.n_heads * w.d_head).reshape(w.batch, w.n_q, w.n_heads, w.d_head)
    k = normal_bf16(seed, T_K, 0, nkv * w.n_kv_heads * w.d_head).reshape(w.batch, w.n_kv, w.n_kv_heads, w.d_head)
    v = normal_bf16(seed, T_V, 0, nkv * w.n_kv_heads * w.d_head).reshape(w.batch, w.n_kv, w.n_kv_heads, w.d_head)
    if k_growth:
        kt = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).float()
        f = 1.0 + k_growth * torch.arange(w.n_kv, dtype=torch.float32) / w.n_kv
        kt = (kt * f.view(1, -1, 1, 1)).to(torch.bfloat16)
        k = kt.view(torch.int16).numpy().view(np.uint16)
    return q, k, v


def _lists(w, rng, density=None, empty_every=0):
    """Ascending -1-padded lists: min(k, p + 1) distinct tokens t <= p per query (fewer with
    `density`, the kept fraction), and every `empty_every`-th row empty."""
    out = np.full((w.batch, w.n_q, w.top_k), -1, dtype=np.int32)
    for s in range(w.batch):
        for i in range(w.n_q):
            if empty_every and (s * w.n_q + i) % empty_every == 3:
                continue
            p = w.n_kv - w.n_q + i
            n = min(w.top_k, p + 1)
            if density is not None:
                n = max(1, min(n, int(density * (p + 1))))
            sel = np.sort(rng.choice(p + 1, size=n, replace=False)).astype(np.int32)
            out[s, i, :n] = sel
    return out


def _run(hs, w, q, k, v, lists, qtile: bool, status=None):
    p = hs.params_of(w)
    dev = "cuda"
    o = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.n_q, w.n_heads), dtype=torch.float32, device=dev)
    tok = torch.from_numpy(lists).to(dev)
    # the query-tile kernel needs the full workspace (its masks); 16 bytes leave only the gather kernels
    ws = None if qtile else torch.empty(16, dtype=torch.uint8, device=dev)
    if qtile:
        masks = w.batch * -(-w.n_q // 128) * -(-w.n_kv // 128) * 2048
        assert hs.hisa_sparse_attn_workspace_size(p) >= masks
    hs.sparse_attn_fwd(p, to_dev(q), to_dev(k), to_dev(v), tok, o, lse, status, ws)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _check(oracle_lib, w, q, k, v, lists, o, lse, rows=None):
    scale = 1.0 / math.sqrt(w.d_head)
    if rows is None:
        rows = [(s, i) for s in range(w.batch) for i in range(w.n_q)]
    for s, i in rows:
        if not np.any(lists[s, i] >= 0):  # an empty list: o = 0, lse = -inf
            assert np.all(o[s, i] == 0) and np.all(np.isneginf(lse[s, i])), f"empty row {s},{i}"
            continue
        ro, rl = oracle_lib.sparse_attn(q[s, i], k[s], v[s], lists[s, i], scale)
        assert_close(o[s, i], ro, f"o[{s},{i}]")
        assert_close(lse[s, i], rl, f"lse[{s},{i}]")


SHAPES = [
    # name, batch, n_q, n_kv, (d_idx, B, m: unused by step 6), k, H, H_kv, d
    Workload("one_tile", 1, 128, 128, 64, 64, 2, 40, 2, 2, 128),
    Workload("ragged_tiles", 1, 300, 300, 64, 64, 2, 64, 2, 2, 128),
    Workload("batch3_chunked", 3, 200, 777, 64, 64, 2, 96, 3, 3, 128),
    Workload("gqa_4_on_2", 2, 260, 260, 64, 64, 2, 80, 4, 2, 128),
    Workload("mqa_8_on_1", 1, 384, 1000, 64, 64, 2, 200, 8, 1, 128),
    Workload("dense_k_ge_p", 1, 256, 256, 64, 64, 2, 256, 2, 2, 128),
]


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_qtile_and_gather_match_oracle(hs, oracle_lib, w):
    rng = np.random.default_rng(11)
    q, k, v = _inputs(w)
    lists = _lists(w, rng, empty_every=97)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for qtile in (True, False):
        o, lse = _run(hs, w, q, k, v, lists, qtile, status)
        _check(oracle_lib, w, q, k, v, lists, o, lse)
    assert int(status.item()) == 0


def test_qtile_rescale_of_late_maxima(hs, oracle_lib):
    """Keys grow along the sequence, so most rows raise their running max in late key tiles."""
    w = Workload("late_max", 2, 512, 1300, 64, 64, 2, 500, 2, 2, 128)
    rng = np.random.default_rng(12)
    q, k, v = _inputs(w, seed=6, k_growth=6.0)
    lists = _lists(w, rng)
    o, lse = _run(hs, w, q, k, v, lists, True)
    _check(oracle_lib, w, q, k, v, lists, o, lse)


def test_qtile_sparse_rows_and_first_tile_only(hs, oracle_lib):
    """Rows keeping very few tokens (most key tiles of a row are empty) and rows keeping only keys of
    the first tile: many tiles add nothing to a row before or after its first kept key."""
    w = Workload("sparse_rows", 1, 640, 640, 64, 64, 2, 64, 2, 2, 128)
    rng = np.random.default_rng(13)
    q, k, v = _inputs(w, seed=7)
    lists = _lists(w, rng, density=0.01)
    lists[0, 300:400] = -1
    lists[0, 300:400, :5] = np.arange(5, dtype=np.int32)
    o, lse = _run(hs, w, q, k, v, lists, True)
    _check(oracle_lib, w, q, k, v, lists, o, lse)


def test_qtile_malformed_entries_are_flagged_and_skipped(hs, oracle_lib):
    """Out-of-range entries (beyond the query's position, below -1), a repeated entry and an entry
    below an earlier one are skipped and flagged; the row then equals the attention over the
    remaining ascending in-range entries.  An empty row gives o = 0 and lse = -inf."""
    w = Workload("bad_entries", 1, 256, 256, 64, 64, 2, 16, 2, 2, 128)
    rng = np.random.default_rng(14)
    q, k, v = _inputs(w, seed=8)
    lists = _lists(w, rng)
    i = 200
    row = lists[0, i].copy()
    bad = row.copy()
    bad[1] = 230      # beyond position 200
    bad[2] = -5       # below -1
    bad[4] = row[3]   # repeats the entry before it
    bad[6] = row[0]   # below an earlier entry
    lists[0, i] = bad
    lists[0, 7] = -1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _run(hs, w, q, k, v, lists, True, status)
    assert int(status.item()) & hs.STATUS_BAD_INDEX
    kept = row.copy()
    kept[[1, 2, 4, 6]] = -1
    ro, rl = oracle_lib.sparse_attn(q[0, i], k[0], v[0], kept, 1.0 / math.sqrt(w.d_head))
    assert_close(o[0, i], ro, "o")
    assert_close(lse[0, i], rl, "lse")
    assert np.all(o[0, 7] == 0) and np.all(np.isneginf(lse[0, 7]))
    others = [(0, j) for j in range(w.n_q) if j not in (i, 7)]
    _check(oracle_lib, w, q, k, v, lists, o, lse, rows=others[::5])


def test_qtile_chunked_prefill_at_a_long_offset(hs, oracle_lib):
    """The last 256 queries of a 20000-token sequence: 157 key tiles, position offset not a multiple
    of 128 (sampled rows checked)."""
    w = Workload("long_offset", 1, 256, 20000, 64, 64, 2, 700, 4, 4, 128)
    rng = np.random.default_rng(15)
    q, k, v = _inputs(w, seed=9)
    lists = _lists(w, rng)
    o, lse = _run(hs, w, q, k, v, lists, True)
    rows = [(0, i) for i in (0, 1, 2, 100, 127, 128, 200, 254, 255)]
    _check(oracle_lib, w, q, k, v, lists, o, lse, rows=rows)
