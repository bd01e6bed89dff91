"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Indices must match bit for bit (integer-valued indexer inputs make every score
exact); attention outputs must satisfy |gpu - oracle| <= 2e-3 + 1e-2 |oracle|.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from parity import ATOL, RTOL, SampledOracle, assert_close, run_forward, run_stages, to_dev  # noqa: E402
from synth import T_K, T_KIDX, T_Q, T_QIDX, T_V, int_bf16, normal_bf16  # noqa: E402
from synth.workloads import WORKLOADS, Workload, full_inputs  # noqa: E402


@pytest.fixture(scope="module")
def hs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as m

    return m


def _dev(inp):
    return {k: to_dev(v) for k, v in inp.items() if not k.startswith("_")}


SMALL = [
    WORKLOADS["tiny_prefill_1k"],
    Workload("ragged_b16", 1, 1000, 1000, 64, 16, 5, 40, 2, 2, 64),
    Workload("chunked_prefill_b3", 3, 300, 1000, 128, 32, 6, 100, 4, 2, 128, needles=3),
    Workload("m2_k1", 2, 200, 517, 64, 8, 2, 1, 1, 1, 64),
    Workload("d256_b256", 1, 700, 1300, 256, 256, 3, 300, 2, 1, 64),
    Workload("b1_tokens", 1, 64, 64, 64, 1, 5, 7, 1, 1, 64),
    Workload("degenerate_all_blocks", 1, 600, 600, 128, 64, 10, 700, 2, 2, 128),
]


def _oracle_full(O, w, inp):
    return O.run(w, inp)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_stages_match_oracle(hs, oracle_lib, w):
    inp = full_inputs(w)
    ref = _oracle_full(oracle_lib, w, inp)
    got = run_stages(hs, w, _dev(inp))
    # step 1: block means, compared as fp32 (both are the correctly rounded mean)
    assert np.array_equal(got["block_keys"].cpu().numpy(), ref["block_keys"].astype(np.float32))
    n = w.batch * w.n_q
    blk = got["block_idx"].cpu().numpy().reshape(n, w.top_m)
    assert np.array_equal(blk, ref["block_idx"]), np.argwhere(blk != ref["block_idx"])[:5]
    tok = got["token_idx"].cpu().numpy().reshape(n, w.top_k)
    assert np.array_equal(tok, ref["token_idx"]), np.argwhere(tok != ref["token_idx"])[:5]
    assert int(got["status"].item()) == 0
    # token scores are exact integers: recompute from the inputs in int64
    q = inp["q_idx"].reshape(n, w.d_idx)
    ts = got["token_scores"].cpu().numpy().reshape(n, w.top_k)
    qf = (q.astype(np.uint32) << 16).view(np.float32).astype(np.int64)
    kf = (inp["k_idx"].astype(np.uint32) << 16).view(np.float32).astype(np.int64)
    for r in range(0, n, max(1, n // 50)):
        seq = r // w.n_q
        v = tok[r] >= 0
        exact = kf[seq][tok[r][v]] @ qf[r]
        assert np.array_equal(ts[r][v], exact.astype(np.float32))
        assert np.all(np.isnan(ts[r][~v]))
    o = got["o"].float().cpu().numpy().reshape(n, w.n_heads, w.d_head)
    assert_close(o, ref["o"], "o")
    assert_close(got["lse"].cpu().numpy().reshape(n, w.n_heads), ref["lse"], "lse")
    # block scores of the kept blocks: exact for full blocks (mean of integers over a
    # power-of-two count), within fp32 rounding for a final partial block
    bsc = got["block_scores"].cpu().numpy().reshape(n, w.top_m)
    for r in range(0, n, max(1, n // 64)):
        seq, i = divmod(r, w.n_q)
        p = w.n_kv - w.n_q + i
        sel, s_, sc = oracle_lib.block_topm(inp["q_idx"][seq, i], ref["block_keys"][seq], w.block, p, w.top_m,
                                            scores=True)
        full = (sel[:s_] + 1) * w.block <= w.n_kv
        assert np.array_equal(bsc[r][:s_][full], sc[:s_][full].astype(np.float32)), r
        assert np.allclose(bsc[r][:s_][~full], sc[:s_][~full], rtol=1e-5, atol=1e-4), r
        assert np.all(np.isnan(bsc[r][s_:]))


@pytest.mark.parametrize("w", SMALL[:3] + [WORKLOADS["prefill_8k"]], ids=lambda w: w.name)
def test_forward_matches_oracle(hs, oracle_lib, w):
    inp = full_inputs(w)
    ref = _oracle_full(oracle_lib, w, inp)
    got = run_forward(hs, w, _dev(inp))
    n = w.batch * w.n_q
    assert np.array_equal(got["block_idx"].cpu().numpy().reshape(n, w.top_m), ref["block_idx"])
    assert np.array_equal(got["token_idx"].cpu().numpy().reshape(n, w.top_k), ref["token_idx"])
    assert_close(got["o"].float().cpu().numpy().reshape(n, w.n_heads, w.d_head), ref["o"], "o")
    assert_close(got["lse"].cpu().numpy().reshape(n, w.n_heads), ref["lse"], "lse")
    assert int(got["status"].item()) == 0


@pytest.mark.parametrize("w", [WORKLOADS["tiny_prefill_1k"], SMALL[1], SMALL[2]], ids=lambda w: w.name)
def test_flat_matches_oracle_and_degeneration(hs, oracle_lib, w):
    inp = full_inputs(w)
    ref = oracle_lib.run(w, inp, flat=True, attention=False)
    dev = _dev(inp)
    p = hs.params_of(w)
    tok = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.int32, device="cuda")
    sc = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.float32, device="cuda")
    hs.hisa_flat_topk(p, dev["q_idx"], dev["k_idx"], tok, sc)
    n = w.batch * w.n_q
    flat = tok.cpu().numpy().reshape(n, w.top_k)
    assert np.array_equal(flat, ref["token_idx"])
    # short-context degeneration: m >= number of blocks gives the flat indexer's output
    wd = w.with_(top_m=w.n_blk + 1)
    got = run_stages(hs, wd, dev, attention=False)
    assert np.array_equal(got["token_idx"].cpu().numpy().reshape(n, w.top_k), flat)


def test_flat_streaming_windows_prefill(hs, oracle_lib):
    """The flat indexer over several 8192-token windows on the tensor-core scorer: a chunk whose
    queries join at different windows (the sequence starts 3000 tokens before the first query),
    window tops merged into the running top-k.  Sampled rows at window edges against the oracle's
    flat top-k, indices and scores bit for bit."""
    w = Workload("flat_windows", 1, 17000, 20000, 128, 128, 4, 700, 1, 1, 64)
    inp = full_inputs(w)
    dev = _dev(inp)
    p = hs.params_of(w)
    tok = torch.empty((1, w.n_q, w.top_k), dtype=torch.int32, device="cuda")
    sc = torch.empty((1, w.n_q, w.top_k), dtype=torch.float32, device="cuda")
    hs.hisa_flat_topk(p, dev["q_idx"], dev["k_idx"], tok, sc)
    torch.cuda.synchronize()
    tok = tok.cpu().numpy()[0]
    sc = sc.cpu().numpy()[0]
    off = w.n_kv - w.n_q
    rows = [0, 1, 5191, 5192, 5193, 8000, 13384, 13385, 16999]  # positions 8191 / 8192 / 16383 / 16384 on
    for i in rows:
        want, k_eff, wsc = oracle_lib.flat_topk(inp["q_idx"][0, i], inp["k_idx"][0], off + i, w.top_k, scores=True)
        assert np.array_equal(tok[i], want), (i, np.argwhere(tok[i] != want)[:5])
        assert np.array_equal(sc[i, :k_eff], wsc[:k_eff].astype(np.float32)), i


def test_flat_streaming_windows_decode_batch(hs, oracle_lib):
    """Decode shape (one query per sequence, each seeing every window): whole sequences share each
    window's launches.  Every sequence's row against the oracle's flat top-k."""
    w = Workload("flat_decode", 5, 1, 30000, 64, 64, 4, 300, 1, 1, 64)
    inp = full_inputs(w)
    dev = _dev(inp)
    p = hs.params_of(w)
    tok = torch.empty((w.batch, 1, w.top_k), dtype=torch.int32, device="cuda")
    sc = torch.empty((w.batch, 1, w.top_k), dtype=torch.float32, device="cuda")
    hs.hisa_flat_topk(p, dev["q_idx"], dev["k_idx"], tok, sc)
    torch.cuda.synchronize()
    tok = tok.cpu().numpy()
    sc = sc.cpu().numpy()
    for b in range(w.batch):
        want, k_eff, wsc = oracle_lib.flat_topk(inp["q_idx"][b, 0], inp["k_idx"][b], w.n_kv - 1, w.top_k, scores=True)
        assert np.array_equal(tok[b, 0], want), (b, np.argwhere(tok[b, 0] != want)[:5])
        assert np.array_equal(sc[b, 0, :k_eff], wsc[:k_eff].astype(np.float32)), b


def test_device_generator_matches_host(hs):
    import synth.device as sd
    from synth.workloads import k_idx_rows

    w = WORKLOADS["prefill_8k"]
    dev = sd.device_inputs(w)
    torch.cuda.synchronize()
    host_q = np.stack([np.asarray(int_bf16(w.seed, T_QIDX, 0, w.n_q * w.d_idx))]).reshape(1, w.n_q, w.d_idx)
    assert np.array_equal(dev["q_idx"].view(torch.int16).cpu().numpy().view(np.uint16), host_q)
    assert np.array_equal(dev["k_idx"].view(torch.int16).cpu().numpy().view(np.uint16)[0],
                          k_idx_rows(w, 0, 0, w.n_kv))
    for name, tid in (("q", T_Q), ("k", T_K), ("v", T_V)):
        flat = dev[name].view(torch.int16).reshape(-1)
        for start in (0, 12345, flat.numel() - 1000):
            got = flat[start:start + 1000].cpu().numpy().view(np.uint16)
            assert np.array_equal(got, normal_bf16(w.seed, tid, start, 1000)), name
    _ = T_KIDX


def test_invalid_indices_are_flagged_and_skipped(hs, oracle_lib):
    w = Workload("bad_idx", 1, 256, 256, 64, 16, 4, 32, 2, 2, 64)
    inp = full_inputs(w)
    dev = _dev(inp)
    p = hs.params_of(w)
    ref = oracle_lib.run(w, inp)
    # a block list with out-of-range, repeated and descending entries
    blk = torch.tensor(ref["block_idx"], dtype=torch.int32, device="cuda").reshape(1, w.n_q, w.top_m)
    i = 200  # own block 12
    good = blk[0, i].clone()
    blk[0, i] = torch.tensor([0, 99, 5, 5], dtype=torch.int32)  # 99 > own block, 5 repeated
    tok = torch.empty((1, w.n_q, w.top_k), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hs.hisa_token_topk(p, dev["q_idx"], dev["k_idx"], blk, tok, None, status)
    torch.cuda.synchronize()
    assert int(status.item()) & hs.STATUS_BAD_INDEX
    # the row behaves like the list [0, 5]
    sel = np.array([0, 5, -1, -1], dtype=np.int32)
    want, _, _ = oracle_lib.token_topk(inp["q_idx"][0, i], inp["k_idx"][0], w.block, i, sel, w.top_k)
    assert np.array_equal(tok[0, i].cpu().numpy(), want)
    blk[0, i] = good
    # attention: an index beyond the query position and one below -1 are skipped
    tlist = torch.tensor(ref["token_idx"], dtype=torch.int32, device="cuda").reshape(1, w.n_q, w.top_k)
    row = tlist[0, 100].clone()
    tlist[0, 100, 1] = 150   # > position 100
    tlist[0, 100, 2] = -5
    o = torch.empty((1, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, w.n_q, w.n_heads), dtype=torch.float32, device="cuda")
    status.zero_()
    hs.sparse_attn_fwd(p, dev["q"], dev["k"], dev["v"], tlist, o, lse, status)
    torch.cuda.synchronize()
    assert int(status.item()) & hs.STATUS_BAD_INDEX
    kept = row.cpu().numpy().copy()
    kept[1] = kept[2] = -1
    ro, rl = oracle_lib.sparse_attn(inp["q"][0, 100], inp["k"][0], inp["v"][0], kept)
    assert_close(o[0, 100].float().cpu().numpy(), ro, "o")
    assert_close(lse[0, 100].cpu().numpy(), rl, "lse")
    # an empty list gives o = 0 and lse = -inf
    tlist[0, 7] = -1
    hs.sparse_attn_fwd(p, dev["q"], dev["k"], dev["v"], tlist, o, lse, None)
    torch.cuda.synchronize()
    assert torch.all(o[0, 7] == 0) and torch.all(torch.isneginf(lse[0, 7]))


def test_block_pool_range_update(hs, oracle_lib):
    w = Workload("pool_range", 2, 1, 5000, 128, 128, 8, 64, 1, 1, 64)
    inp = full_inputs(w)
    dev = _dev(inp)
    p = hs.params_of(w)
    bk = torch.full((2, w.n_blk, w.d_idx), 123.0, dtype=torch.float32, device="cuda")
    hs.hisa_block_pool(p, dev["k_idx"], bk, 10, 20)
    torch.cuda.synchronize()
    got = bk.cpu().numpy()
    for s in range(2):
        ref = oracle_lib.block_pool(inp["k_idx"][s], w.block).astype(np.float32)
        assert np.array_equal(got[s, 10:20], ref[10:20])
        assert np.all(got[s, :10] == 123.0) and np.all(got[s, 20:] == 123.0)


# ------------------------------------------------------------------ full-size workloads

def _device_inputs(w, with_attention=True):
    import synth.device as sd

    return sd.device_inputs(w, with_attention=with_attention)


def _check_invariants(w, got):
    """Properties every query must satisfy, checked on the whole GPU output."""
    blk = got["block_idx"].reshape(-1, w.top_m).long()
    tok = got["token_idx"].reshape(-1, w.top_k).long()
    n = blk.shape[0]
    i = torch.arange(n, device=blk.device) % w.n_q
    p = w.n_kv - w.n_q + i
    c = p // w.block
    s = torch.clamp(c + 1, max=w.top_m)
    assert torch.all(blk[:, 0] == 0)
    assert torch.all(blk.gather(1, (s - 1)[:, None])[:, 0] == c)
    valid_b = blk >= 0
    assert torch.all(valid_b.sum(1) == s)
    n_cand = torch.where(s == c + 1, p + 1, (s - 1) * w.block + p % w.block + 1)
    k_eff = torch.clamp(n_cand, max=w.top_k)
    valid_t = tok >= 0
    assert torch.all(valid_t.sum(1) == k_eff)
    d = tok[:, 1:] - tok[:, :-1]
    assert torch.all((d > 0) | ~valid_t[:, 1:])
    assert torch.all(tok.max(1).values <= p)
    # every kept token lies in a kept block
    for r0 in range(0, n, 2048):
        vt = valid_t[r0:r0 + 2048]
        tb = torch.where(vt, tok[r0:r0 + 2048] // w.block, torch.full_like(tok[r0:r0 + 2048], -2))
        member = (tb[:, :, None] == blk[r0:r0 + 2048, None, :]).any(2) | ~vt
        assert torch.all(member)


@pytest.mark.slow
def test_prefill_64k_sampled(hs, oracle_lib):
    w = WORKLOADS["prefill_64k"]
    dev = _device_inputs(w)
    got = run_forward(hs, w, dev)
    assert int(got["status"].item()) == 0
    _check_invariants(w, got)
    so = SampledOracle(oracle_lib, w)
    picks = [0, 1, 127, 128, 129, 255, 1000, 8191, 8192, 20000, 32767, 40000, 50001, 65000, 65534, w.n_q - 1]
    rng = np.random.default_rng(3)
    picks += rng.integers(0, w.n_q, 16).tolist()
    blk = got["block_idx"][0].cpu().numpy()
    tok = got["token_idx"][0].cpu().numpy()
    o = got["o"][0].float().cpu().numpy()
    lse = got["lse"][0].cpu().numpy()
    for i in picks:
        ref = so.query(0, i)
        assert np.array_equal(blk[i], ref["block_idx"]), i
        assert np.array_equal(tok[i], ref["token_idx"]), i
        assert_close(o[i], ref["o"], f"o[{i}]")
        assert_close(lse[i], ref["lse"], f"lse[{i}]")


@pytest.mark.slow
def test_decode_32x128k_sampled(hs, oracle_lib):
    w = WORKLOADS["decode_32x128k"]
    dev = _device_inputs(w)
    got = run_forward(hs, w, dev)
    assert int(got["status"].item()) == 0
    _check_invariants(w, got)
    so = SampledOracle(oracle_lib, w)
    for seq in (0, 13, 31):
        ref = so.query(seq, 0)
        assert np.array_equal(got["block_idx"][seq, 0].cpu().numpy(), ref["block_idx"]), seq
        assert np.array_equal(got["token_idx"][seq, 0].cpu().numpy(), ref["token_idx"]), seq
        assert_close(got["o"][seq, 0].float().cpu().numpy(), ref["o"], f"o[{seq}]")
        assert_close(got["lse"][seq, 0].cpu().numpy(), ref["lse"], f"lse[{seq}]")


@pytest.mark.slow
def test_decode_4x1m_m_sweep_sampled(hs, oracle_lib):
    base = WORKLOADS["decode_4x1m_m64"]
    dev = _device_inputs(base)
    for m, seq in ((32, 1), (64, 2), (128, 3)):
        w = base.with_(top_m=m)
        got = run_forward(hs, w, dev)
        assert int(got["status"].item()) == 0
        _check_invariants(w, got)
        ref = SampledOracle(oracle_lib, w).query(seq, 0)
        assert np.array_equal(got["block_idx"][seq, 0].cpu().numpy(), ref["block_idx"]), m
        assert np.array_equal(got["token_idx"][seq, 0].cpu().numpy(), ref["token_idx"]), m
        assert_close(got["o"][seq, 0].float().cpu().numpy(), ref["o"], f"o m={m}")
        assert_close(got["lse"][seq, 0].cpu().numpy(), ref["lse"], f"lse m={m}")


def test_tolerance_constants():
    assert (ATOL, RTOL) == (2e-3, 1e-2)
    assert math.isclose(1 / math.sqrt(128), 0.08838834764831845)


@pytest.mark.parametrize("n_kv,block", [(1000, 64), (1025, 64), (777, 16)])
def test_forward_cached_decode_loop(hs, oracle_lib, n_kv, block):
    """hisa_forward_cached: refreshing only the block the newest token entered gives the same
    result as hisa_forward on the whole cache, and as the oracle."""
    w = Workload("decode_loop", 3, 1, n_kv, 128, block, 6, 200, 4, 2, 64, needles=2)
    inp = full_inputs(w)
    dev = _dev(inp)
    ref = run_forward(hs, w, dev)
    # block keys of the cache before the newest token (n_kv - 1 tokens), pooled once
    prev = w.with_(n_kv=n_kv - 1)
    bk = torch.full((w.batch, w.n_blk, w.d_idx), 9.0, dtype=torch.float32, device="cuda")
    k_prev = dev["k_idx"][:, : n_kv - 1].contiguous()
    tmp = torch.empty((w.batch, prev.n_blk, w.d_idx), dtype=torch.float32, device="cuda")
    hs.hisa_block_pool(hs.params_of(prev), k_prev, tmp)
    bk[:, : prev.n_blk] = tmp  # a block the newest token opens still holds 9.0 here
    p = hs.params_of(w)
    o = torch.empty_like(ref["o"])
    lse = torch.empty_like(ref["lse"])
    blk = torch.empty_like(ref["block_idx"])
    tok = torch.empty_like(ref["token_idx"])
    hs.hisa_forward_cached(p, dev["q_idx"], dev["k_idx"], bk, (n_kv - 1) // block, dev["q"], dev["k"], dev["v"], o,
                           lse, blk, tok)
    torch.cuda.synchronize()
    assert torch.equal(blk, ref["block_idx"]) and torch.equal(tok, ref["token_idx"])
    assert torch.equal(o, ref["o"]) and torch.equal(lse, ref["lse"])
    oref = oracle_lib.run(w, inp)
    assert np.array_equal(tok.cpu().numpy().reshape(w.batch, w.top_k), oref["token_idx"])
    assert_close(o.float().cpu().numpy().reshape(w.batch, w.n_heads, w.d_head), oref["o"], "o")
    # refresh from block 0 recomputes every key
    bk.fill_(5.0)
    hs.hisa_forward_cached(p, dev["q_idx"], dev["k_idx"], bk, 0, dev["q"], dev["k"], dev["v"], o, lse, blk, tok)
    torch.cuda.synchronize()
    assert torch.equal(tok, ref["token_idx"]) and torch.equal(o, ref["o"])


def test_decode_step_in_a_cuda_graph(hs, oracle_lib):
    """A decode step (newest-block refresh + steps 2-6) captured once in a CUDA graph and
    replayed gives the same outputs as the eager calls, for fresh query contents."""
    w = Workload("graph_decode", 8, 1, 3000, 128, 64, 8, 256, 4, 4, 128)
    inp = full_inputs(w)
    dev = _dev(inp)
    p = hs.params_of(w)
    bk = torch.empty((w.batch, w.n_blk, w.d_idx), dtype=torch.float32, device="cuda")
    hs.hisa_block_pool(p, dev["k_idx"], bk)
    ws = torch.empty(hs.hisa_forward_workspace_size(p), dtype=torch.uint8, device="cuda")
    o = torch.empty((w.batch, 1, w.n_heads, w.d_head), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.batch, 1, w.n_heads), dtype=torch.float32, device="cuda")
    tok = torch.empty((w.batch, 1, w.top_k), dtype=torch.int32, device="cuda")
    q_idx, q = dev["q_idx"].clone(), dev["q"].clone()

    def step():
        hs.hisa_forward_cached(p, q_idx, dev["k_idx"], bk, w.n_blk - 1, q, dev["k"], dev["v"], o, lse, None, tok,
                               None, ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up: one-time kernel attributes are set outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for trial in range(2):
        # new query contents each replay (a different sequence's queries rolled in)
        q_idx.copy_(dev["q_idx"].roll(trial + 1, dims=0))
        q.copy_(dev["q"].roll(trial + 1, dims=0))
        g.replay()
        torch.cuda.synchronize()
        got_o, got_tok = o.clone(), tok.clone()
        step()
        torch.cuda.synchronize()
        assert torch.equal(got_tok, tok) and torch.equal(got_o, o)
    del g


# Candidate lists longer than the selection kernel stages in shared memory (49152 keys): the keys
# are then read from global memory in every pass.
LONG_LISTS = [
    Workload("flat_long_lists", 1, 4, 60000, 64, 64, 8, 512, 2, 2, 64),             # flat: 60032 keys
    Workload("hier_long_lists", 2, 1, 70000, 64, 256, 200, 1024, 2, 2, 64, needles=5),  # m * B = 51200
]


@pytest.mark.parametrize("w", LONG_LISTS, ids=lambda w: w.name)
def test_selection_from_global_memory(hs, oracle_lib, w):
    inp = full_inputs(w)
    dev = _dev(inp)
    n = w.batch * w.n_q
    if w.name.startswith("flat"):
        ref = oracle_lib.run(w, inp, flat=True, attention=False)
        p = hs.params_of(w)
        tok = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.int32, device="cuda")
        hs.hisa_flat_topk(p, dev["q_idx"], dev["k_idx"], tok)
        assert np.array_equal(tok.cpu().numpy().reshape(n, w.top_k), ref["token_idx"])
    else:
        ref = oracle_lib.run(w, inp)
        got = run_stages(hs, w, dev)
        assert np.array_equal(got["block_idx"].cpu().numpy().reshape(n, w.top_m), ref["block_idx"])
        assert np.array_equal(got["token_idx"].cpu().numpy().reshape(n, w.top_k), ref["token_idx"])
        assert_close(got["o"].float().cpu().numpy().reshape(n, w.n_heads, w.d_head), ref["o"], "o")
        assert int(got["status"].item()) == 0
