"""The exactness argument of the stochastic-rounding kernels, checked on the CPU.

The CUDA quantizers decide "round up" (R < f * 2^16, the oracle's rule of
stochastic_oracle.e2m1_encode_sr) on the fp32 bits: from magnitude 1 up,
adding 2^22 - 1 - 64 R to the bits and clearing the low 22 mantissa bits
gives the lower or the upper E2M1 neighbour; below 1, the magnitude is first
shifted by 1 with an add rounded toward +inf, which keeps ceil(f * 2^16), the
only part of f that an integer R is compared with; values from 6 up land on 6
or above, which the conversion's satfinite turns into 6.  This file restates
that bit-level decision in numpy and holds it to the oracle's rule on edge
magnitudes for every R and on random values; the GPU parity tests then check
the kernels themselves against the oracle.
"""
import numpy as np

from oracle import stochastic_oracle as S

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)


def _add_round_up(a, c):
    """fp32 a + c rounded toward +inf (a, c >= 0 fp32): the exact sum as an
    fp64 two-sum, then the next fp32 up when rounding to nearest fell below."""
    a64, c64 = a.astype(np.float64), c.astype(np.float64)
    s = a64 + c64
    bp = s - a64
    err = (a64 - (s - bp)) + (c64 - bp)        # a + c = s + err exactly
    r = s.astype(np.float32)
    below = (r.astype(np.float64) < s) | ((r.astype(np.float64) == s) & (err > 0))
    return np.where(below, np.nextafter(r, np.float32(np.inf)), r).astype(np.float32)


def _bit_level_codes(u, r16):
    u = np.asarray(u, dtype=np.float32)
    a = np.abs(u)
    c = np.where(a < 1.0, np.float32(1.0), np.float32(0.0)).astype(np.float32)
    b = _add_round_up(a, c).view(np.uint32).astype(np.uint64)
    k = np.uint64(0x3FFFFF) - (r16.astype(np.uint64) << np.uint64(6))
    t = ((b + k) & np.uint64(0xFFC00000)).astype(np.uint32).view(np.float32)
    m = np.minimum(t - c, np.float32(6.0))      # the conversion's satfinite
    idx = np.searchsorted(GRID, m)
    assert np.array_equal(GRID[idx], m), "the bit-level result left the E2M1 grid"
    return idx.astype(np.uint8) | np.where(np.signbit(u), np.uint8(8), np.uint8(0))


def test_edge_magnitudes_for_every_r():
    edges = np.concatenate([
        GRID, np.nextafter(GRID, np.float32(9)), np.nextafter(GRID, np.float32(-1)),
        np.float32([1e-30, 2.0 ** -149, 2.0 ** -17, 2.0 ** -18, 3 * 2.0 ** -18, 0.25, 0.75, 1.25, 1.75,
                    2.5, 3.5, 5.0, 0.5 - 2.0 ** -25, 1 - 2.0 ** -24, 2 - 2.0 ** -23, 6 - 2.0 ** -21, 7.0,
                    8.0, 100.0]),
    ]).astype(np.float32)
    edges = np.concatenate([edges, -edges])
    u = np.repeat(edges, 65536)
    r16 = np.tile(np.arange(65536, dtype=np.uint16), edges.size)
    assert np.array_equal(_bit_level_codes(u, r16), S.e2m1_encode_sr(u, r16))


def test_random_values_and_draws():
    rng = np.random.default_rng(2026)
    n = 1 << 20
    u = np.concatenate([
        rng.uniform(-8, 8, n),
        rng.standard_normal(n) * 2.0 ** rng.integers(-40, 3, n),
        np.frombuffer(rng.integers(0, 0x40FFFFFF, n, dtype=np.uint32).tobytes(), np.float32),
    ]).astype(np.float32)
    u = u[np.isfinite(u)]
    for r16 in (rng.integers(0, 65536, u.size), np.zeros(u.size, int), np.full(u.size, 65535)):
        r16 = r16.astype(np.uint16)
        assert np.array_equal(_bit_level_codes(u, r16), S.e2m1_encode_sr(u, r16))


def test_a_wrong_constant_is_caught():
    """Planted on the CPU: the carry constant without its -1 rounds up when
    rem == 64 R, where the rule says down."""
    u = np.float32([1.0 + 64 * 5 * 2.0 ** -23])          # rem = 320 = 64 * 5
    r16 = np.uint16([5])
    a = np.abs(u)
    b = a.view(np.uint32).astype(np.uint64)
    wrong = ((b + np.uint64(0x400000) - (r16.astype(np.uint64) << np.uint64(6))) & np.uint64(0xFFC00000))
    assert wrong.astype(np.uint32).view(np.float32)[0] == np.float32(1.5)
    assert _bit_level_codes(u, r16)[0] == S.e2m1_encode_sr(u, r16)[0] == 2   # 1.0, code 2
