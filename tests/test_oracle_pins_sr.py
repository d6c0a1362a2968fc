"""Pins of the stochastic-rounding oracle (CPU only).

[P5] "FP4" encyclopedia entry, section 技術原理: NVFP4 quantization rounds
     stochastically instead of truncating.  The defining property of
     stochastic rounding is pinned exactly: over all 2^16 random integers the
     rounded value equals the input to within 2^-16 of a grid step (its
     expectation), and it is always one of the two neighbouring grid values.
The Philox4x32-10 generator is pinned by the known-answer vectors that ship
with the authors' Random123 library (Salmon et al., "Parallel random numbers:
as easy as 1, 2, 3", SC 2011).
"""
import numpy as np
import pytest

from oracle import nvfp4_oracle as O
from oracle import stochastic_oracle as S
from nvfp4_block_scaled_15_b200 import inputs

# Random123 known-answer tests for philox4x32 with 10 rounds: (counter, key, output)
PHILOX_KAT = [
    ([0x00000000, 0x00000000, 0x00000000, 0x00000000], [0x00000000, 0x00000000],
     [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
    ([0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF], [0xFFFFFFFF, 0xFFFFFFFF],
     [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
    ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
     [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
]

ALL_R = np.arange(1 << 16, dtype=np.uint16)


def check_philox_known_answers():
    for ctr, key, want in PHILOX_KAT:
        got = S.philox4x32_10(np.array(ctr, dtype=np.uint64), np.array(key, dtype=np.uint64))
        assert got.tolist() == want, [hex(v) for v in got]
    # vectorised form equals the one-at-a-time form
    ctr = np.array([c for c, _, _ in PHILOX_KAT], dtype=np.uint64)
    key = np.array([k for _, k, _ in PHILOX_KAT], dtype=np.uint64)
    assert S.philox4x32_10(ctr, key).tolist() == [w for _, _, w in PHILOX_KAT]


def check_random_layout():
    """Step 5's layout, restated from single Philox calls for a few elements,
    and roughly uniform bits over a larger draw."""
    seed, offset = 0x0123456789ABCDEF, 0x00000007FFFFFFFE
    r = S.random16(5, 64, seed, offset)
    key = np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint64)
    for row, col in [(0, 0), (0, 15), (3, 37), (4, 63), (2, 24)]:
        b, e = divmod(col, 16)
        h, rest = divmod(e, 8)
        i, m = divmod(rest, 2)
        w = S.philox4x32_10(np.array([2 * b + h, row, offset & 0xFFFFFFFF, offset >> 32], dtype=np.uint64), key)
        assert r[row, col] == (int(w[i]) >> (16 * m)) & 0xFFFF
    big = S.random16(64, 4096, 5, 0).astype(np.int64)
    assert abs(big.mean() - 32767.5) < 0.01 * 65536
    bits = (big[..., None] >> np.arange(16)) & 1
    assert np.all(np.abs(bits.mean(axis=(0, 1)) - 0.5) < 0.01)
    # a different seed, offset or row gives different bits
    assert not np.array_equal(S.random16(4, 64, 1, 0), S.random16(4, 64, 2, 0))
    assert not np.array_equal(S.random16(4, 64, 1, 0), S.random16(4, 64, 1, 1))
    rr = S.random16(2, 64, 1, 0)
    assert not np.array_equal(rr[0], rr[1])


def _probe_values():
    """fp32 magnitudes across the E2M1 range: grid points, midpoints, random."""
    rng = np.random.default_rng(11)
    v = np.concatenate([O.E2M1_MAGNITUDES, [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0],
                        rng.uniform(0, 6, 200), [1e-30, 2.0 ** -20, 5.999999, 6.0, 7.5, np.inf]])
    return v.astype(np.float32)


def check_probability_of_rounding_up_exactly():
    """For every probe u, the number of R in [0, 2^16) that round up is
    ceil(f * 2^16) (f the fractional position between the neighbours), and the
    result is always lo or hi; magnitudes >= 6 give 6 for every R."""
    mags = O.E2M1_MAGNITUDES
    for a in _probe_values():
        codes = S.e2m1_encode_sr(np.full(ALL_R.shape, a, dtype=np.float32), ALL_R)
        vals = O.e2m1_decode(codes)
        if a >= 6:
            assert np.all(vals == 6.0)
            continue
        lo = mags[mags <= a].max()
        hi = mags[mags > a].min()
        assert set(np.unique(vals)) <= {lo, hi}
        f = (np.float64(a) - lo) / (hi - lo)
        assert np.count_nonzero(vals == hi) == int(np.ceil(f * 65536)), a


def check_expectation_equals_input():
    """E over all 2^16 draws of the rounded value is u to within 2^-16 of the
    step (stochastic rounding is unbiased), where deterministic rounding is
    off by up to half a step."""
    mags = O.E2M1_MAGNITUDES
    for a in _probe_values():
        if not a < 6:
            continue
        codes = S.e2m1_encode_sr(np.full(ALL_R.shape, a, dtype=np.float32), ALL_R)
        mean = O.e2m1_decode(codes).mean()
        step = mags[mags > a].min() - mags[mags <= a].max()
        assert abs(mean - np.float64(a)) <= step * 2.0 ** -16 + 1e-15, a


def check_grid_points_sign_and_zero():
    """Grid values are kept for every R; the code keeps the sign bit, so a
    negative value that rounds to 0 gives -0 (code 8)."""
    for c in range(16):
        v = np.float32(O.e2m1_decode(np.uint8(c)))
        codes = S.e2m1_encode_sr(np.full(ALL_R.shape, v, dtype=np.float32), ALL_R)
        assert np.all(codes == c), c
    codes = S.e2m1_encode_sr(np.full(ALL_R.shape, -0.1, dtype=np.float32), ALL_R)
    assert set(np.unique(codes)) == {8, 9}
    assert S.e2m1_encode_sr(np.float32(-7.0), np.uint16(0)) == 15


def check_quantizer_scales_and_neighbours():
    """Block scales, g and amax equal the deterministic quantizer's; every
    code is one of the two grid neighbours of u = (x g) / sd; zero blocks and
    zero-scale blocks give zero codes; equal seeds give equal codes."""
    x = inputs.activations_with_outliers(16, 512, seed=21, fraction=0.01, factor=50.0).copy()
    x[3, 32:48] = 0
    packed, sf, g, a = S.quantize_sr(x, seed=9, offset=3)
    p2, sf2, g2, a2 = O.quantize(x)
    assert np.array_equal(sf, sf2) and g == g2 and a == a2
    u = (O.bf16_to_f32(x) * g).astype(np.float32).reshape(16, 32, 16)
    sd = O.e4m3_decode(sf)[:, :, None]
    u = np.where(sd == 0, np.float32(0), (u / np.where(sd == 0, 1, sd)).astype(np.float32))
    got = O.e2m1_decode(O.unpack_codes(packed)).reshape(16, 32, 16)
    mags = O.E2M1_MAGNITUDES
    au = np.minimum(np.abs(u).astype(np.float64), 6.0)
    lo = mags[np.clip(np.searchsorted(mags, au, side="right") - 1, 0, 7)]
    hi = mags[np.clip(np.searchsorted(mags, au, side="left"), 0, 7)]
    assert np.all((np.abs(got) == lo) | (np.abs(got) == hi))
    assert not O.unpack_codes(packed)[3, 32:48].any()
    assert np.array_equal(S.quantize_sr(x, seed=9, offset=3)[0], packed)
    assert not np.array_equal(S.quantize_sr(x, seed=10, offset=3)[0], packed)


def check_tensor_mean_converges():
    """Averaged over 64 offsets, the dequantized tensor approaches x (the
    deterministic quantizer's error does not average away)."""
    x = inputs.gaussian_bf16((8, 256), seed=31)
    xf = O.bf16_to_f32(x).astype(np.float64)
    acc = np.zeros_like(xf)
    for off in range(64):
        p, sf, g, _ = S.quantize_sr(x, seed=1, offset=off)
        acc += O.dequantize(p, sf, g)
    err_sr = np.abs(acc / 64 - xf).mean()
    p, sf, g, _ = O.quantize(x)
    err_rn = np.abs(O.dequantize(p, sf, g) - xf).mean()
    assert err_sr < 0.35 * err_rn, (err_sr, err_rn)


PINS = [check_philox_known_answers, check_random_layout, check_probability_of_rounding_up_exactly,
        check_expectation_equals_input, check_grid_points_sign_and_zero, check_quantizer_scales_and_neighbours,
        check_tensor_mean_converges]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_planted_mistakes():
    """Plausible mistakes in the oracle, planted on the CPU, each caught by a pin."""
    import contextlib

    @contextlib.contextmanager
    def planted(obj, name, value):
        old = getattr(obj, name)
        setattr(obj, name, value)
        try:
            yield
        finally:
            setattr(obj, name, old)

    orig_philox, orig_encode, orig_random = S.philox4x32_10, S.e2m1_encode_sr, S.random16

    def philox_no_key_bump(counter, key):
        with planted(S, "PHILOX_W0", 0), planted(S, "PHILOX_W1", 0):
            return orig_philox(counter, key)

    def encode_le(u, r16):                      # R <= f 2^16: rounds up too often
        u = np.asarray(u, dtype=np.float32)
        a = np.abs(u).astype(np.float64)
        mags = O.E2M1_MAGNITUDES
        lo = np.clip(np.searchsorted(mags, a, side="right") - 1, 0, 7)
        hi = np.minimum(lo + 1, 7)
        step = np.where(hi > lo, mags[hi] - mags[lo], 1.0)
        up = np.asarray(r16, dtype=np.float64) <= (a - mags[lo]) / step * 65536
        code = np.where(a >= 6, 7, np.where(up, hi, lo)).astype(np.uint8)
        return code | np.where(np.signbit(u), np.uint8(8), np.uint8(0))

    def encode_nearest(u, r16):                 # deterministic rounding in disguise
        return O.e2m1_encode(u)

    def random_swapped_halves(rows, k, seed, offset):
        r = orig_random(rows, k, seed, offset).reshape(rows, k // 2, 2)
        return r[..., ::-1].reshape(rows, k).copy()

    def random_reversed(rows, k, seed, offset):
        return orig_random(rows, k, seed, offset)[:, ::-1].copy()

    mistakes = [
        ("Philox without the key schedule", "philox4x32_10", philox_no_key_bump, check_philox_known_answers),
        ("R <= f instead of R < f", "e2m1_encode_sr", encode_le, check_probability_of_rounding_up_exactly),
        ("round to nearest", "e2m1_encode_sr", encode_nearest, check_expectation_equals_input),
        ("16-bit halves swapped", "random16", random_swapped_halves, check_random_layout),
        ("elements in reverse", "random16", random_reversed, check_random_layout),
    ]
    for what, name, fake, pin in mistakes:
        with planted(S, name, fake):
            with pytest.raises(AssertionError):
                pin()
        assert S.philox4x32_10 is orig_philox and S.e2m1_encode_sr is orig_encode, what
