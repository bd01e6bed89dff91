"""Stored regression fixtures (tests/golden/, written by tests/golden/make_golden.py from the oracle
alone; the pages print no worked example of their own).  On the CPU the oracle must still produce
them exactly; on a GPU the CUDA path must select the same blocks and tokens, bit for bit, and
attend within the parity tolerance."""
import importlib.util
import os

import numpy as np
import pytest

from parity import assert_close, dev_inputs, run_stages
from synth.workloads import full_inputs

HERE = os.path.dirname(os.path.abspath(__file__))
_spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "golden", "make_golden.py"))
golden = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(golden)


def _fields(w):
    return [str(x) for x in (w.name, w.batch, w.n_q, w.n_kv, w.d_idx, w.block, w.top_m, w.top_k, w.n_heads,
                             w.n_kv_heads, w.d_head, w.n_idx_heads)]


@pytest.mark.parametrize("w,ids", golden.FIXTURES, ids=[f[0].name for f in golden.FIXTURES])
def test_oracle_reproduces_fixture(oracle_lib, w, ids):
    fields, rows = golden.read(golden.fixture_path(w))
    assert fields == _fields(w) and sorted(rows) == sorted(ids)
    out = oracle_lib.run(w, full_inputs(w), query_ids=np.array(ids, dtype=np.int64))
    for r, q in enumerate(ids):
        assert np.array_equal(out["block_idx"][r], rows[q]["blocks"])
        assert np.array_equal(out["token_idx"][r], rows[q]["tokens"])
        assert np.allclose(out["lse"][r], rows[q]["lse"], rtol=1e-13, atol=0)
        assert np.allclose(out["o"][r].reshape(-1), rows[q]["o"], rtol=1e-12, atol=1e-15)


@pytest.mark.gpu
@pytest.mark.parametrize("w,ids", golden.FIXTURES, ids=[f[0].name for f in golden.FIXTURES])
def test_gpu_matches_fixture(w, ids):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as hs

    _, rows = golden.read(golden.fixture_path(w))
    got = run_stages(hs, w, dev_inputs(full_inputs(w)))
    n = w.batch * w.n_q
    blk = got["block_idx"].cpu().numpy().reshape(n, w.top_m)
    tok = got["token_idx"].cpu().numpy().reshape(n, w.top_k)
    o = got["o"].float().cpu().numpy().reshape(n, w.n_heads * w.d_head)
    lse = got["lse"].cpu().numpy().reshape(n, w.n_heads)
    for q in ids:
        assert np.array_equal(blk[q], rows[q]["blocks"]), q
        assert np.array_equal(tok[q], rows[q]["tokens"]), q
        assert_close(o[q], rows[q]["o"], f"o[{q}]")
        assert_close(lse[q], rows[q]["lse"], f"lse[{q}]")
