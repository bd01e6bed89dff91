"""GPU parity of step 5's selection on score patterns chosen for it: every score tied, three distinct
scores, scores that differ only in their lowest mantissa bits, and plain integer scores; each through
the 256-thread selection (many queries) and the 1024-thread one (few queries), against the oracle's
token top-k on the same block lists.

The selection resolves the threshold in wide digits of the order-preserving key and, when the keys
of the threshold digit are too many to gather, resolves the later digits over the whole row; the
tied and three-value patterns force that branch, the fine pattern needs the last digit.  The scores
are exact in fp32 by construction (at most two nonzero products, no rounding), so the selected
indices and their scores must match the oracle's bit for bit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from synth.workloads import Workload  # noqa: E402


@pytest.fixture(scope="module")
def hs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as m

    return m


def _bf16(x):
    """float values exactly representable in bf16 -> bf16 bits."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert np.all(u & 0xFFFF == 0), "not a bf16 value"
    return (u >> 16).astype(np.uint16)


def _pattern(name, rng, nq, nkv, d):
    q = np.zeros((nq, d), dtype=np.float32)
    k = np.zeros((nkv, d), dtype=np.float32)
    if name == "all_tied":  # a zero query: every score is 0
        k[:] = rng.integers(-4, 5, size=k.shape)
    elif name == "three_values":  # scores in {-1, 0, 1}
        q[:, 0] = 1.0
        k[:, 0] = rng.integers(-1, 2, size=nkv)
    elif name == "fine":  # k0 + k1 / 65536 with k0, k1 in [1, 2): bits down to 2^-23, 64 distinct values
        q[:, 0] = 1.0
        q[:, 1] = 2.0 ** -16
        k[:, 0] = 1.0 + rng.choice(rng.choice(128, 8, replace=False), nkv) / 128.0
        k[:, 1] = 1.0 + rng.choice(rng.choice(128, 8, replace=False), nkv) / 128.0
    elif name == "integer":
        q[:] = rng.integers(-4, 5, size=q.shape)
        k[:] = rng.integers(-4, 5, size=k.shape)
    else:
        raise ValueError(name)
    return _bf16(q), _bf16(k)


def _block_lists(rng, w):
    """Ascending -1-padded lists of top_m distinct blocks <= the query's own block, with blocks 0 and own."""
    out = np.full((w.batch, w.n_q, w.top_m), -1, dtype=np.int32)
    for s in range(w.batch):
        for i in range(w.n_q):
            c = (w.n_kv - w.n_q + i) // w.block
            if c + 1 <= w.top_m:
                out[s, i, :c + 1] = np.arange(c + 1)
                continue
            mid = rng.choice(np.arange(1, c), size=w.top_m - 2, replace=False) if c > 1 else []
            out[s, i] = np.sort(np.concatenate([[0, c], mid])).astype(np.int32)
    return out


SHAPES = [
    # 1024 keys per row; few queries (1024-thread selection) and many (256-thread selection)
    Workload("wide_1k", 4, 1, 4096, 64, 64, 16, 256, 1, 1, 64),
    Workload("narrow_1k", 8, 64, 4096, 64, 64, 16, 256, 1, 1, 64),
    # 8192 keys per row, the headline prefill's row length
    Workload("wide_8k", 2, 1, 16384, 128, 128, 64, 2048, 1, 1, 64),
    Workload("narrow_8k", 4, 80, 16384, 128, 128, 64, 2048, 1, 1, 64),
]
PATTERNS = ["all_tied", "three_values", "fine", "integer"]


@pytest.mark.parametrize("pattern", PATTERNS)
@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_selection_patterns_match_oracle(hs, oracle_lib, w, pattern):
    rng = np.random.default_rng(21)
    q, k = _pattern(pattern, rng, w.batch * w.n_q, w.batch * w.n_kv, w.d_idx)
    q = q.reshape(w.batch, w.n_q, w.d_idx)
    k = k.reshape(w.batch, w.n_kv, w.d_idx)
    blk = _block_lists(rng, w)
    p = hs.params_of(w)
    dq = torch.from_numpy(q.view(np.int16)).cuda()
    dk = torch.from_numpy(k.view(np.int16)).cuda()
    dblk = torch.from_numpy(blk).cuda()
    tok = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.int32, device="cuda")
    sc = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hs.hisa_token_topk(p, dq, dk, dblk, tok, sc, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    tok = tok.cpu().numpy()
    sc = sc.cpu().numpy()
    for s in range(w.batch):
        for i in range(w.n_q):
            pos = w.n_kv - w.n_q + i
            want, k_eff, _, wsc = oracle_lib.token_topk(q[s, i], k[s], w.block, pos, blk[s, i], w.top_k, scores=True)
            assert np.array_equal(tok[s, i], want), (s, i, np.argwhere(tok[s, i] != want)[:5])
            assert np.array_equal(sc[s, i, :k_eff], wsc[:k_eff].astype(np.float32)), (s, i)
            assert np.all(np.isnan(sc[s, i, k_eff:]))
