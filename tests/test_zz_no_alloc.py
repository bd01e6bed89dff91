"""hisa_token_topk_noalloc: the token stage for callers that cannot allocate device memory.

Such callers (an engine that pre-plans all device memory and gives plugins no
allocator, a latency-critical loop that must not call cudaMalloc) get the same
results as hisa_token_topk without passing a workspace; the library's fixed
device scratch array is used instead.  This test calls the new entry point
through the C ABI and checks it against hisa_token_topk, twice in a row with
different inputs (the shared array keeps the previous call's contents), on a
case that fits in one chunk and on one that needs several.  It lives in its
own file so that it runs after every other test.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from parity import run_stages, to_dev  # noqa: E402
from synth.workloads import Workload, full_inputs  # noqa: E402


@pytest.fixture(scope="module")
def hs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as m

    return m


def _call_noalloc(hs, w, dev, blk):
    """Through the C ABI directly: no workspace argument exists."""
    p = hs.params_of(w)
    tok = torch.full((w.batch, w.n_q, w.top_k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((w.batch, w.n_q, w.top_k), 7.0, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = hs.lib().hisa_token_topk_noalloc(ctypes.byref(p), ctypes.c_void_p(dev["q_idx"].data_ptr()), None,
                                          ctypes.c_void_p(dev["k_idx"].data_ptr()), ctypes.c_void_p(blk.data_ptr()),
                                          ctypes.c_void_p(tok.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
                                          ctypes.c_void_p(status.data_ptr()), stream)
    torch.cuda.synchronize()
    assert rc == hs.HISA_OK, hs.lib().hisa_status_string(rc)
    return tok, sc, status


CASES = [
    # decode-like: 6 sequences x 1 query, fits the 16 MiB array in one chunk
    Workload("noalloc_decode", 6, 1, 20000, 128, 128, 16, 300, 1, 1, 64, needles=4),
    # prefill: 4096 queries x 64 slots x 128 keys x 4 B = 128 MiB of keys -> 8 chunks
    Workload("noalloc_prefill", 1, 4096, 4096, 128, 128, 64, 256, 1, 1, 64),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point(hs, w):
    for call, seed in enumerate((0, 1)):  # two calls in a row, different inputs
        ws = w.with_(seed=seed)
        dev = {k: to_dev(v) for k, v in full_inputs(ws).items()}
        ref = run_stages(hs, ws, dev, attention=False)  # hisa_block_topm + hisa_token_topk (with workspace)
        tok, sc, status = _call_noalloc(hs, ws, dev, ref["block_idx"])
        assert int(status.item()) == 0
        assert torch.equal(tok, ref["token_idx"]), f"call {call}: token indices differ"
        assert torch.equal(torch.nan_to_num(sc, nan=-1e30), torch.nan_to_num(ref["token_scores"], nan=-1e30)), \
            f"call {call}: token scores differ"
        assert not torch.equal(tok, torch.full_like(tok, -7))


def test_noalloc_rejects_a_query_larger_than_the_array(hs):
    # one query would need 4096 blocks x 2048 tokens x 4 B = 32 MiB of keys > 16 MiB
    p = hs.params(1, 1, 1 << 23, 128, 2048, 4096, 16)
    a = ctypes.c_void_p(1 << 20)
    rc = hs.lib().hisa_token_topk_noalloc(ctypes.byref(p), a, None, a, a, a, None, None, None)
    assert rc == hs.HISA_ERR_UNSUPPORTED
    _ = np
