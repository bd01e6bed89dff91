"""The seeded input generator: published SplitMix64 outputs, value maps and the recipe."""
import math

import numpy as np

import synth
from synth.workloads import WORKLOADS, k_idx_rows_int, needle_table, probe_signs


def test_splitmix64_published_outputs():
    # SplitMix64 from state 0: the first two outputs of the published generator.
    z = np.array([0x9E3779B97F4A7C15, (2 * 0x9E3779B97F4A7C15) % 2**64], dtype=np.uint64)
    out = synth._mix64(z)
    assert int(out[0]) == 0xE220A8397B1DCDAF
    assert int(out[1]) == 0x6E789E6AA1B965F4


def test_stream_is_index_addressable():
    a = synth.raw_u64(0, synth.T_K, 0, 1000)
    b = synth.raw_u64(0, synth.T_K, 123, 10)
    assert np.array_equal(a[123:133], b)
    assert not np.array_equal(synth.raw_u64(0, synth.T_V, 0, 10), a[:10])
    assert not np.array_equal(synth.raw_u64(1, synth.T_K, 0, 10), a[:10])


def test_irwin_hall_constant_and_moments():
    assert synth.IH_SCALE == np.float32(math.sqrt(3.0 / (65536.0**2 - 1)))
    x = synth.bf16_bits_to_f32(synth.normal_bf16(0, synth.T_Q, 0, 1 << 20)).astype(np.float64)
    assert abs(x.mean()) < 5e-3
    assert abs(x.var() - 1.0) < 1e-2
    assert np.abs(x).max() <= 3.47


def test_integer_values():
    v = synth.int_values(0, synth.T_QIDX, 0, 1 << 18)
    assert v.min() == -4 and v.max() == 4
    counts = np.bincount(v.astype(np.int64) + 4, minlength=9) / len(v)
    assert np.all(np.abs(counts - 1 / 9) < 5e-3)
    b = synth.int_bf16(0, synth.T_QIDX, 0, 1000)
    assert np.array_equal(synth.bf16_bits_to_f32(b), synth.int_values(0, synth.T_QIDX, 0, 1000).astype(np.float32))


def test_needles():
    w = WORKLOADS["prefill_8k"]
    nb = needle_table(w, 0)
    assert len(nb) == 8 and len(set(nb.tolist())) == 8
    assert nb.min() >= 1 and nb.max() <= w.n_blk - 2
    sg = probe_signs(w, 0)
    t0 = int(nb[0]) * w.block
    shifted = k_idx_rows_int(w, 0, t0, w.block).astype(np.int64)
    base = synth.int_values(w.seed, synth.T_KIDX, t0 * w.d_idx, w.block * w.d_idx).reshape(w.block, w.d_idx)
    assert np.array_equal(shifted, np.clip(base + 2 * sg, -4, 4))
