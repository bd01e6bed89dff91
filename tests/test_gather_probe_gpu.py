"""The measurement probe on the GPU: it runs for every supported row size and launch shape and
really copies rows (every warp adds its first copied word to the sink)."""
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("row_bytes", [32, 64, 128, 256])
@pytest.mark.parametrize("ctas", [1, 2, 3])
def test_gather_probe_copies_rows(row_bytes, ctas):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_sparse_attention_block_b200 as hs

    rows = torch.full((1 << 20,), 1, dtype=torch.uint8, device="cuda")  # every word 0x01010101
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    hs.hisa_gather_probe(rows, row_bytes, 1 << 16, sink, ctas_per_sm=ctas)
    torch.cuda.synchronize()
    # 4 warps per CTA, each with at least one tile (4096 tiles of 16 gathers), each adding 0x01010101
    warps = 4 * ctas * torch.cuda.get_device_properties(0).multi_processor_count
    assert int(sink.item()) & 0xFFFFFFFF == (warps * 0x01010101) & 0xFFFFFFFF
