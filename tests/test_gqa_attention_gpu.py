"""GPU parity of the attention when several heads share one K/V head (GQA/MQA).

The selected token list is shared by all heads of a query, so the heads of a KV
group read the same K and V rows; the tensor-core kernel takes them together
(groups of 2, 4, 8 or 16 heads, a group of 3 padded to 4, a group of 24 split
16 + 8).  Prefill shapes run one work item per (KV head, query); decode shapes
split the lists across CTAs and merge the partial states.  Same bar as the
other parity tests: indices bit for bit, |gpu - oracle| <= 2e-3 + 1e-2 |oracle|.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from parity import assert_close, run_stages, to_dev  # noqa: E402
from synth.workloads import Workload, full_inputs  # noqa: E402


@pytest.fixture(scope="module")
def hs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as m

    return m


CASES = [
    # name, batch, n_q, n_kv, d_idx, block, top_m, top_k, n_heads, n_kv_heads, d_head
    Workload("gqa2_prefill", 2, 257, 700, 64, 32, 6, 200, 4, 2, 128, needles=2),
    Workload("gqa3_prefill", 1, 300, 900, 64, 32, 6, 260, 6, 2, 128),
    Workload("mqa8_prefill", 1, 384, 384, 64, 32, 5, 130, 8, 1, 128),
    Workload("mqa16_prefill", 1, 200, 640, 64, 64, 4, 150, 16, 1, 128),
    Workload("gqa24_decode", 3, 1, 5000, 64, 64, 8, 300, 48, 2, 128),
    Workload("mqa16_decode", 4, 1, 9000, 64, 128, 10, 700, 16, 1, 128),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_shared_kv_attention_matches_oracle(hs, oracle_lib, w):
    inp = full_inputs(w)
    ref = oracle_lib.run(w, inp)
    got = run_stages(hs, w, {k: to_dev(v) for k, v in inp.items() if not k.startswith("_")})
    n = w.batch * w.n_q
    assert np.array_equal(got["token_idx"].cpu().numpy().reshape(n, w.top_k), ref["token_idx"])
    assert_close(got["o"].float().cpu().numpy().reshape(n, w.n_heads, w.d_head), ref["o"], "o")
    assert_close(got["lse"].cpu().numpy().reshape(n, w.n_heads), ref["lse"], "lse")
    assert int(got["status"].item()) == 0
