"""hisa_forward_host: the forward pass with inputs and outputs in pinned host memory, the copies
overlapped with the work (query chunks of long sequences, groups of short ones).  Each chunk's
attention is the same per-(query, head) computation as hisa_forward's, so where both take the
list whole (one split) the outputs must be bit-identical to hisa_forward's on device copies of
the inputs; decode groups split lists differently, so there the check is the oracle's
tolerance.  The serialised form (no copy stream) must give the same bits as the overlapped one."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from parity import assert_close, dev_inputs  # noqa: E402
from synth.workloads import Workload, full_inputs  # noqa: E402


@pytest.fixture(scope="module")
def hs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as m

    return m


def _host(inp):
    out = {}
    for k, v in inp.items():
        if k.startswith("_"):
            continue
        a = np.ascontiguousarray(v)
        t = torch.from_numpy(a) if a.dtype == np.float32 else torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        out[k] = t.pin_memory()
    return out


def _run_host(hs, w, h, copy_stream):
    p = hs.params_of(w)
    o = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16).pin_memory()
    lse = torch.empty((w.batch, w.n_q, w.n_heads), dtype=torch.float32).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream()
    hs.hisa_forward_host(p, h["q_idx"], h["k_idx"], h["q"], h["k"], h["v"], o, lse, status, stream=st,
                         copy_stream=copy_stream, idx_weights=h.get("w_idx"))
    st.synchronize()
    assert int(status.item()) == 0
    return o, lse


def _run_device(hs, w, dev):
    p = hs.params_of(w)
    o = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.batch, w.n_q, w.n_heads), dtype=torch.float32, device="cuda")
    hs.hisa_forward(p, dev["q_idx"], dev["k_idx"], dev["q"], dev["k"], dev["v"], o, lse,
                    idx_weights=dev.get("w_idx"))
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


PREFILL = [
    # name, batch, n_q, n_kv, d_idx, block, top_m, top_k, n_heads, n_kv_heads, d_head
    Workload("host_prefill_chunks", 2, 20000, 20000, 64, 64, 8, 256, 2, 2, 64),  # 3 chunks per sequence
    Workload("host_context_gqa", 1, 9000, 12000, 128, 128, 8, 512, 8, 2, 128),  # prefix context, GQA
    Workload("host_multihead_indexer", 1, 9000, 9000, 64, 32, 6, 128, 2, 2, 64, n_idx_heads=4),
    Workload("host_context_batch2", 2, 9000, 11000, 64, 64, 8, 256, 2, 2, 64),  # chunks of sequence 1
]


@pytest.mark.parametrize("w", PREFILL, ids=lambda w: w.name)
def test_host_forward_equals_device_forward(hs, w):
    inp = full_inputs(w)
    ref_o, ref_lse = _run_device(hs, w, dev_inputs(inp))
    h = _host(inp)
    side = torch.cuda.Stream()
    o, lse = _run_host(hs, w, h, side)
    assert torch.equal(o.view(torch.int16), ref_o.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    o2, lse2 = _run_host(hs, w, h, None)  # serialised on one stream
    assert torch.equal(o2.view(torch.int16), o.view(torch.int16)) and torch.equal(lse2, lse)


@pytest.mark.parametrize("batch", [5, 11])  # groups of one sequence; groups of one and two
def test_host_forward_decode_groups_match_oracle(hs, oracle_lib, batch):
    w = Workload("host_decode", batch, 1, 7000, 64, 64, 8, 300, 4, 4, 64, needles=3)
    inp = full_inputs(w)
    ref = oracle_lib.run(w, inp)
    o, lse = _run_host(hs, w, _host(inp), torch.cuda.Stream())
    n = w.batch * w.n_q
    assert_close(o.float().numpy().reshape(n, w.n_heads, w.d_head), ref["o"], "o")
    assert_close(lse.numpy().reshape(n, w.n_heads), ref["lse"], "lse")


def test_host_forward_rejects_device_buffers(hs):
    w = Workload("host_reject", 1, 256, 256, 64, 64, 4, 64, 2, 2, 64)
    inp = full_inputs(w)
    h = _host(inp)
    dev = dev_inputs(inp)
    p = hs.params_of(w)
    o = torch.empty((1, 256, 2, 64), dtype=torch.bfloat16).pin_memory()
    with pytest.raises(hs.HisaError) as err:
        hs.hisa_forward_host(p, h["q_idx"], dev["k_idx"], h["q"], h["k"], h["v"], o)
    assert err.value.status == hs.HISA_ERR_INVALID_ARG
    torch.cuda.synchronize()


def test_host_forward_one_query_last_chunk(hs, oracle_lib):
    """8193 queries: the second chunk holds one query, whose 512-entry token list is split across
    CTAs (two work items only, so the list is cut in four), so it is checked against the oracle's
    tolerance; the first chunk stays bit-identical to hisa_forward."""
    w = Workload("host_one_query_chunk", 1, 8193, 8193, 64, 64, 8, 512, 2, 2, 64)
    inp = full_inputs(w)
    ref_o, ref_lse = _run_device(hs, w, dev_inputs(inp))
    o, lse = _run_host(hs, w, _host(inp), torch.cuda.Stream())
    assert torch.equal(o[:, :8192].view(torch.int16), ref_o[:, :8192].view(torch.int16))
    assert torch.equal(lse[:, :8192], ref_lse[:, :8192])
    ref = oracle_lib.run(w, inp, query_ids=np.array([8192], dtype=np.int64))
    assert_close(o[0, 8192].float().numpy().reshape(1, w.n_heads, w.d_head), ref["o"], "o")
    assert_close(lse[0, 8192].numpy().reshape(1, w.n_heads), ref["lse"], "lse")
