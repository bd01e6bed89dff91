"""Seeded, index-addressable synthetic inputs shared by the CUDA path and the oracle.

This module holds the input recipe only; it contains none of the attention
method's arithmetic.  Every value is a pure function of (seed, tensor id, flat
element index), so any row of any tensor can be regenerated on its own: the
oracle regenerates only the rows it needs, the device generator in
``synth/synth.cu`` fills whole tensors in HBM, and both produce the same bits.

Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014).  Its state advances by the
golden-ratio increment and each output is the state passed through the
variant-13 finaliser.  Here the i-th output of stream (seed, tensor) is
``mix64(base + (i + 1) * GAMMA)`` with ``base = mix64(seed * GAMMA + tensor)``.

Value maps
  * integer indexer values: ``((u >> 32) * 9 >> 32) - 4`` in {-4..4}, stored as
    exact bf16.  With these, every block sum and dot product of the indexer is
    an integer below 2**24, so fp32 results are exact.
  * head weights of a multi-head indexer: ``((u >> 32) * 5 >> 32)`` mapped to
    {-2, -1, 1, 2, 3} (fp32), so every weighted score stays an exact integer.
  * unit-variance stand-ins for N(0,1): Irwin-Hall with n = 4 over the four
    16-bit fields of ``u``: ``(sum - 131070) * C`` with ``C = sqrt(3/(2**32-1))``
    rounded once to fp32, one fp32 multiply (round to nearest even), then bf16
    round to nearest even.  Mean 0, variance 1, support +-3.46.
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Tensor ids of the streams.
T_QIDX, T_KIDX, T_Q, T_K, T_V, T_NEEDLE, T_WIDX = 1, 2, 3, 4, 5, 6, 7

# fp32 constant sqrt(3 / (65536**2 - 1)); the value the device generator uses
# is the same bit pattern (checked in tests).
IH_SCALE_BITS = 0x37DDB3D7
IH_SCALE = np.array([IH_SCALE_BITS], dtype=np.uint32).view(np.float32)[0]
IH_CENTRE = 131070


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def stream_base(seed: int, tensor: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) * GAMMA + np.uint64(tensor)
    return _mix64(np.array([s], dtype=np.uint64))[0]


def raw_u64(seed: int, tensor: int, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of stream (seed, tensor) as uint64."""
    base = stream_base(seed, tensor)
    idx = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        st = base + (idx + np.uint64(1)) * GAMMA
    return _mix64(st)


def _f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


_WEIGHTS = np.array([-2.0, -1.0, 1.0, 2.0, 3.0], dtype=np.float32)


def weight_values(seed: int, tensor: int, start: int, count: int) -> np.ndarray:
    """Indexer head weights in {-2, -1, 1, 2, 3} as fp32."""
    u = raw_u64(seed, tensor, start, count)
    return _WEIGHTS[((u >> np.uint64(32)) * np.uint64(5)) >> np.uint64(32)]


def int_values(seed: int, tensor: int, start: int, count: int) -> np.ndarray:
    """Integer indexer values in {-4..4} as int8."""
    u = raw_u64(seed, tensor, start, count)
    with np.errstate(over="ignore"):
        v = ((u >> np.uint64(32)) * np.uint64(9)) >> np.uint64(32)
    return (v.astype(np.int64) - 4).astype(np.int8)


def int_bf16(seed: int, tensor: int, start: int, count: int) -> np.ndarray:
    return _f32_to_bf16_bits(int_values(seed, tensor, start, count).astype(np.float32))


def normal_bf16(seed: int, tensor: int, start: int, count: int) -> np.ndarray:
    """Unit-variance Irwin-Hall (n=4) values as bf16 bit patterns."""
    u = raw_u64(seed, tensor, start, count)
    m16 = np.uint64(0xFFFF)
    s = (u & m16) + ((u >> np.uint64(16)) & m16) + ((u >> np.uint64(32)) & m16) + (u >> np.uint64(48))
    centred = (s.astype(np.int64) - IH_CENTRE).astype(np.float32)  # exact: |x| < 2**24
    return _f32_to_bf16_bits(centred * IH_SCALE)


def needle_blocks(seed: int, seq: int, n_blk: int, n_needle: int) -> np.ndarray:
    """Distinct needle blocks drawn from {1 .. n_blk-2} by a partial Fisher-Yates shuffle."""
    pool = np.arange(1, n_blk - 1, dtype=np.int64)
    n_needle = min(n_needle, len(pool))
    u = raw_u64(seed, T_NEEDLE, seq << 20, max(n_needle, 1))
    for i in range(n_needle):
        span = len(pool) - i
        with np.errstate(over="ignore"):
            j = i + int(((u[i] >> np.uint64(32)) * np.uint64(span)) >> np.uint64(32))
        pool[i], pool[j] = pool[j], pool[i]
    return np.sort(pool[:n_needle]).astype(np.int32)


def needle_signs(q_probe_bf16: np.ndarray) -> np.ndarray:
    """sign(q) per dimension of the probe query, as int8 in {-1, 0, 1}."""
    return np.sign(bf16_bits_to_f32(q_probe_bf16)).astype(np.int8)


def apply_needles(k_rows_int: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """Shift integer keys toward the probe direction: clamp(k + 2*sign, -4, 4)."""
    return np.clip(k_rows_int.astype(np.int16) + 2 * signs.astype(np.int16), -4, 4).astype(np.int8)
