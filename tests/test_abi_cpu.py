"""The C-ABI library without a GPU: every declared symbol is exported, and the host-side
validation rejects bad arguments before anything is launched."""
import ctypes
import os
import re

import pytest

import hierarchical_sparse_attention_block_b200 as hs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hisa.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:hisa_status_t|const char\*|int32_t)\s+(\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 14, names
    lib = ctypes.CDLL(hs.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(hs.EXPORTS)


def test_status_strings_and_version():
    lib = hs.lib()
    for code in range(5):
        assert lib.hisa_status_string(code)
    assert hs.hisa_version().startswith("hisa-b200")
    assert lib.hisa_last_cuda_error() == 0


def _p(**kw):
    base = dict(batch=1, n_q=1024, n_kv=1024, d_idx=64, block=64, top_m=4, top_k=128, n_heads=1, d_head=64)
    base.update(kw)
    return hs.params(**base)


def _ws(fn, p):
    n = ctypes.c_size_t(0)
    return fn(ctypes.byref(p), ctypes.byref(n)), n.value


@pytest.mark.parametrize("kw,code", [
    (dict(n_q=2048), hs.HISA_ERR_INVALID_ARG),        # more queries than keys
    (dict(n_q=0), hs.HISA_ERR_INVALID_ARG),
    (dict(batch=0), hs.HISA_ERR_INVALID_ARG),
    (dict(block=48), hs.HISA_ERR_UNSUPPORTED),        # not a power of two
    (dict(block=0), hs.HISA_ERR_INVALID_ARG),
    (dict(d_idx=96), hs.HISA_ERR_UNSUPPORTED),
    (dict(top_m=1), hs.HISA_ERR_INVALID_ARG),         # the two forced blocks need m >= 2
    (dict(top_k=0), hs.HISA_ERR_INVALID_ARG),
])
def test_indexer_validation(kw, code):
    rc, _ = _ws(hs.lib().hisa_block_topm_workspace_size, _p(**kw))
    assert rc == code


@pytest.mark.parametrize("kw,code", [
    (dict(n_heads=3, n_kv_heads=2), hs.HISA_ERR_INVALID_ARG),
    (dict(d_head=96), hs.HISA_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), hs.HISA_ERR_INVALID_ARG),
])
def test_attention_validation(kw, code):
    rc, _ = _ws(hs.lib().hisa_sparse_attn_workspace_size, _p(**kw))
    assert rc == code


def test_flags_must_be_zero():
    p = _p()
    p.flags = 1
    rc, _ = _ws(hs.lib().hisa_forward_workspace_size, p)
    assert rc == hs.HISA_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected_before_launch():
    lib = hs.lib()
    p = _p()
    assert lib.hisa_block_pool(None, ctypes.c_void_p(256), 0, -1, ctypes.c_void_p(512), None) == hs.HISA_ERR_INVALID_ARG
    assert lib.hisa_block_pool(ctypes.byref(p), None, 0, -1, ctypes.c_void_p(512), None) == hs.HISA_ERR_INVALID_ARG
    assert lib.hisa_block_pool(ctypes.byref(p), ctypes.c_void_p(258), 0, -1, ctypes.c_void_p(512),
                               None) == hs.HISA_ERR_INVALID_ARG
    # block range outside [0, n_blk]
    assert lib.hisa_block_pool(ctypes.byref(p), ctypes.c_void_p(256), 3, 2, ctypes.c_void_p(512),
                               None) == hs.HISA_ERR_INVALID_ARG
    assert lib.hisa_block_pool(ctypes.byref(p), ctypes.c_void_p(256), 0, 17, ctypes.c_void_p(512),
                               None) == hs.HISA_ERR_INVALID_ARG


def test_workspace_checks_before_launch():
    lib = hs.lib()
    p = _p()
    a = ctypes.c_void_p(4096)
    need = hs.hisa_block_topm_workspace_size(p)
    assert need >= 1024 * 16 * 4
    assert lib.hisa_block_topm(ctypes.byref(p), a, None, a, a, None, None, a, need - 1, None) == hs.HISA_ERR_WORKSPACE
    assert lib.hisa_block_topm(ctypes.byref(p), a, None, a, a, None, None, None, need, None) == hs.HISA_ERR_WORKSPACE
    mn, pref = hs.hisa_token_topk_workspace_size(p)
    assert mn == p.top_m * p.block * 4 and pref == mn * p.n_q
    assert lib.hisa_token_topk(ctypes.byref(p), a, None, a, a, a, None, None, a, mn - 4, None) == hs.HISA_ERR_WORKSPACE
    # the flat indexer: one row = a window of min(8192 tokens, all 16 blocks) keys, four k-entry
    # arrays and the alignment slack of its five buffers; preferred = every row
    fmin, fpref = hs.hisa_flat_topk_workspace_size(p)
    assert fmin == 16 * 64 * 4 + 4 * 128 * 4 + 5 * 256 and fpref == fmin * p.n_q
    assert lib.hisa_flat_topk(ctypes.byref(p), a, None, a, a, None, a, fmin - 1, None) == hs.HISA_ERR_WORKSPACE
    need_f = hs.hisa_forward_workspace_size(p)
    assert lib.hisa_forward(ctypes.byref(p), a, None, a, a, a, a, a, None, None, None, None, a, need_f - 1,
                            None) == hs.HISA_ERR_WORKSPACE


def test_indexer_heads_and_weights_go_together():
    """n_idx_heads = 0 takes no head weights; n_idx_heads >= 1 requires them; more than 16 heads
    are outside the supported range.  All rejected on the host, before any launch."""
    lib = hs.lib()
    a = ctypes.c_void_p(4096)
    p = _p()
    need = hs.hisa_block_topm_workspace_size(p)
    assert lib.hisa_block_topm(ctypes.byref(p), a, a, a, a, None, None, a, need, None) == hs.HISA_ERR_INVALID_ARG
    p.n_idx_heads = 4
    assert lib.hisa_block_topm(ctypes.byref(p), a, None, a, a, None, None, a, need, None) == hs.HISA_ERR_INVALID_ARG
    mn, _ = hs.hisa_token_topk_workspace_size(p)
    assert lib.hisa_token_topk(ctypes.byref(p), a, None, a, a, a, None, None, a, mn, None) == hs.HISA_ERR_INVALID_ARG
    assert lib.hisa_token_topk(ctypes.byref(p), a, ctypes.c_void_p(4098), a, a, a, None, None, a, mn,
                               None) == hs.HISA_ERR_INVALID_ARG  # weights not 4-byte aligned
    p.n_idx_heads = 17
    assert lib.hisa_block_topm(ctypes.byref(p), a, a, a, a, None, None, a, need, None) == hs.HISA_ERR_UNSUPPORTED
    p.n_idx_heads = -1
    assert lib.hisa_block_topm(ctypes.byref(p), a, a, a, a, None, None, a, need, None) == hs.HISA_ERR_INVALID_ARG


def test_workspace_sizes_follow_the_shapes():
    # decode: 32 sequences x 128K keys, m = 64, k = 2048, 16 heads
    p = hs.params(32, 1, 131072, 128, 128, 64, 2048, 16, 16, 128)
    mn, pref = hs.hisa_token_topk_workspace_size(p)
    assert mn == 64 * 128 * 4 and pref == 32 * mn
    # the attention list is split across CTAs when there are few queries
    assert hs.hisa_sparse_attn_workspace_size(p) > 0
    # many queries per sequence: the query-tile kernel's masks, 128 x 128 bits per (query tile,
    # key tile), 512 x 512 tiles at 64K, then an fp16 copy of V and two words per KV head
    big = hs.params(1, 65536, 65536, 128, 128, 64, 2048, 16, 16, 128)
    assert hs.hisa_sparse_attn_workspace_size(big) == 512 * 512 * 2048 + 65536 * 16 * 128 * 2 + 2 * 256
    # d = 64 has no query-tile kernel and no split lists at this size
    big64 = hs.params(1, 65536, 65536, 128, 128, 64, 2048, 16, 16, 64)
    assert hs.hisa_sparse_attn_workspace_size(big64) == 0
    # a context much longer than the kept tokens: dense tiles would cost more than gathers
    far = hs.params(1, 4096, 1 << 20, 128, 128, 64, 2048, 16, 16, 128)
    assert hs.hisa_sparse_attn_workspace_size(far) == 0


def test_gather_probe_validation():
    """The measurement probe rejects bad arguments on the host: null or misaligned rows, row
    sizes other than 32, 64, 128 and 256 bytes, and launch shapes
    outside 0..3 CTAs per SM; zero gathers launch nothing."""
    lib = hs.lib()
    a = ctypes.c_void_p(4096)
    ok = dict(n_rows=1024, row_bytes=256, n=64, seed=1, ctas=0)

    def call(rows=a, sink=a, **kw):
        k = {**ok, **kw}
        return lib.hisa_gather_probe(rows, k["n_rows"], k["row_bytes"], k["n"], k["seed"], sink, k["ctas"], None)

    assert call(rows=None) == hs.HISA_ERR_INVALID_ARG
    assert call(sink=None) == hs.HISA_ERR_INVALID_ARG
    assert call(rows=ctypes.c_void_p(4104)) == hs.HISA_ERR_INVALID_ARG
    for rb in (0, 8, 16, 24, 48, 96, 272, 512):
        assert call(row_bytes=rb) == hs.HISA_ERR_INVALID_ARG, rb
    for c in (-1, 4):
        assert call(ctas=c) == hs.HISA_ERR_INVALID_ARG, c
    assert call(n_rows=0) == hs.HISA_ERR_INVALID_ARG
    assert call(n=-1) == hs.HISA_ERR_INVALID_ARG
    assert call(n=0) == hs.HISA_OK


def test_forward_host_validation():
    """hisa_forward_host checks its arguments on the host before any copy: every input and o
    present, head weights iff n_idx_heads > 0, a 16-byte aligned device workspace of at least
    hisa_forward_host_workspace_size bytes, which covers hisa_forward's workspace plus device
    copies of every input and output."""
    lib = hs.lib()
    p = _p()
    a = ctypes.c_void_p(4096)
    need = hs.hisa_forward_host_workspace_size(p)
    fwd = hs.hisa_forward_workspace_size(p)
    io = (p.batch * p.n_q * p.d_idx * 2 + p.batch * p.n_kv * p.d_idx * 2
          + 2 * p.batch * p.n_q * p.n_heads * p.d_head * 2 + 2 * p.batch * p.n_kv * p.n_kv_heads * p.d_head * 2
          + p.batch * p.n_q * p.n_heads * 4)
    assert need >= fwd + io

    def call(qi=a, w=None, ki=a, q=a, k=a, v=a, o=a, ws=a, nbytes=need):
        return lib.hisa_forward_host(ctypes.byref(p), qi, w, ki, q, k, v, o, None, None, ws, nbytes, None, None)

    for kw in ("qi", "ki", "q", "k", "v", "o"):
        assert call(**{kw: None}) == hs.HISA_ERR_INVALID_ARG, kw
    assert call(w=a) == hs.HISA_ERR_INVALID_ARG  # weights without indexer heads
    assert call(nbytes=need - 1) == hs.HISA_ERR_WORKSPACE
    assert call(ws=None) == hs.HISA_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p(4104)) == hs.HISA_ERR_WORKSPACE


def test_binding_refuses_tensors_on_the_wrong_side():
    """The Python binding checks where each tensor lives before calling the library: the device
    calls refuse CPU tensors (a host address must not reach a kernel) and hisa_forward_host
    refuses CUDA tensors for its host arguments."""
    torch = pytest.importorskip("torch")
    p = _p()
    cpu = torch.zeros(16, dtype=torch.bfloat16)
    calls = (lambda: hs.hisa_block_pool(p, cpu, torch.zeros(16, dtype=torch.float32)),
             lambda: hs.sparse_attn_fwd(p, cpu, cpu, cpu, torch.zeros(4, dtype=torch.int32), cpu),
             lambda: hs._hptr(type("FakeCuda", (), {"is_cuda": True})()))
    for call in calls:
        with pytest.raises(hs.HisaError) as err:
            call()
        assert err.value.status == hs.HISA_ERR_INVALID_ARG
        assert isinstance(err.value, RuntimeError)
    assert hs._hptr(cpu).value == cpu.data_ptr()


def test_sparse_attn_kernel_choice_follows_shape_and_workspace():
    """hisa_sparse_attn_kernel (host logic only): the query-tile kernel needs d = 128, many queries per
    sequence and the full workspace; otherwise the gather kernels run."""
    p = hs.params(1, 65536, 65536, 128, 128, 64, 2048, 16, 16, 128)
    need = hs.hisa_sparse_attn_workspace_size(p)
    assert hs.hisa_sparse_attn_kernel(p, need) == hs.ATTN_QTILE
    assert hs.hisa_sparse_attn_kernel(p, need - 1) == hs.ATTN_GATHER
    assert hs.hisa_sparse_attn_kernel(p, 0) == hs.ATTN_GATHER
    decode = hs.params(32, 1, 131072, 128, 128, 64, 2048, 16, 16, 128)
    assert hs.hisa_sparse_attn_kernel(decode, 1 << 40) == hs.ATTN_GATHER
    d64 = hs.params(1, 1024, 1024, 64, 64, 4, 128, 1, 1, 64)
    assert hs.hisa_sparse_attn_kernel(d64, 1 << 40) == hs.ATTN_GATHER
    with pytest.raises(hs.HisaError):
        hs.hisa_sparse_attn_kernel(hs.params(1, 8, 8, 64, 64, 4, 8, 3, 2, 128), 0)  # 3 heads on 2 KV heads
