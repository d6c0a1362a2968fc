"""Pins of the CPU oracle against what the pages and mathematics fix.

Each ``check_*`` function raises AssertionError when the oracle disagrees with
a page-printed value, a closed form, an error bound stated by the pages, or
brute force.  ``test_planted_mistakes`` plants plausible mistakes in the
oracle (on the CPU) and shows that some check catches each of them.
"""
from pathlib import Path

import numpy as np
import pytest

from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs

GOLDEN = Path(__file__).parent / "golden"


def _golden_values(name):
    vals = []
    for line in (GOLDEN / name).read_text(encoding="utf-8").splitlines():
        line = line.strip()
        if line and not line.startswith("#"):
            vals.append(line)
    return vals


def _facts():
    out = {}
    for line in _golden_values("page_facts.txt"):
        k, v = line.split()
        out[k] = float(v)
    return out


FACTS = _facts()


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def _bits_f32(b):
    return np.asarray(b, dtype=np.uint32).view(np.float32)


# --------------------------------------------------------------------------
# E2M1
# --------------------------------------------------------------------------
def check_e2m1_table():
    """The 16 printed values, in code order, with -0 distinct from +0."""
    printed = _golden_values("e2m1_values.txt")
    dec = O.e2m1_decode(np.arange(16))
    for code, text in enumerate(printed):
        want = float(text)
        assert dec[code] == want, (code, dec[code], want)
        assert np.signbit(dec[code]) == text.startswith("-"), code
    assert np.max(np.abs(dec)) == FACTS["e2m1_max"]


def check_e2m1_onnx_rule():
    """FP4 wiki (技術原理): E != 0: (-1)^S 2^(E-1) (1 + M/2); E == 0: (-1)^S M/2."""
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = (2.0 ** (e - 1)) * (1 + m * 0.5) if e != 0 else m * 0.5
        want = -mag if s else mag
        got = O.e2m1_decode([code])[0]
        assert got == want and np.signbit(got) == bool(s), (code, got, want)


def _e2m1_closed_form(u):
    """Round-to-nearest-even onto {0,.5,1,1.5,2,3,4,6} written as its decision
    thresholds: a tie goes to the neighbour with the even code."""
    a = np.abs(u.astype(np.float64))
    mag_code = np.select(
        [a <= 0.25, a < 0.75, a <= 1.25, a < 1.75, a <= 2.5, a < 3.5, a <= 5.0],
        [0, 1, 2, 3, 4, 5, 6], default=7)
    return (mag_code | np.where(np.signbit(u), 8, 0)).astype(np.uint8)


def _e2m1_sweep():
    top = int(np.array(8.0, dtype=np.float32).view(np.uint32))
    pos = _bits_f32(np.arange(0, top, 331, dtype=np.uint32))
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], dtype=np.float32)
    near = np.concatenate([ties, np.nextafter(ties, np.float32(0)), np.nextafter(ties, np.float32(10))])
    big = _f32([6.5, 7.0, 100.0, 1e30, np.finfo(np.float32).max])
    tiny = _f32([0.0, 1e-45, 1e-30, 0.2499999])
    allpos = np.concatenate([pos, near.astype(np.float32), big, tiny]).astype(np.float32)
    return np.concatenate([allpos, -allpos]).astype(np.float32)


def check_e2m1_encoder():
    u = _e2m1_sweep()
    got = O.e2m1_encode(u)
    want = _e2m1_closed_form(u)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (u[bad[:5]], got[bad[:5]], want[bad[:5]])


# --------------------------------------------------------------------------
# E4M3
# --------------------------------------------------------------------------
def check_e4m3_page_example():
    b = O.e4m3_encode_satfinite(_f32([FACTS["e4m3_example_in"]]))
    assert O.e4m3_decode(b)[0] == np.float32(FACTS["e4m3_example_out"])


def check_e4m3_grid():
    printed = np.array([float(v) for v in _golden_values("e4m3_grid_half_to_one.txt")])
    allv = O.e4m3_decode(np.arange(256)).astype(np.float64)
    in_range = np.unique(allv[(allv >= 0.5) & (allv <= 1.0)])
    assert np.array_equal(in_range, printed), in_range


def check_e4m3_max_and_saturation():
    allv = O.e4m3_decode(np.arange(256)).astype(np.float64)
    assert np.nanmax(allv) == FACTS["e4m3_max"]
    b = O.e4m3_encode_satfinite(_f32([448.0, 449.0, 464.0, 480.0, 1e6]))
    assert np.all(O.e4m3_decode(b) == np.float32(448.0)) and np.all(b == 0x7E)


def _e4m3_closed_form(s):
    """Nearest E4M3 value from the exponent/mantissa definition: 3 mantissa bits,
    bias 7, subnormal step 2^-9, largest finite 448; ties to even mantissa (np.rint)."""
    s = s.astype(np.float64)
    _, e = np.frexp(s)                  # s = m * 2^e, m in [0.5, 1)
    ex = np.maximum(e - 1, -6)          # unbiased exponent, subnormals share -6
    step = np.exp2(ex - 3.0)
    v = np.rint(s / step) * step
    return np.minimum(v, 448.0)


def check_e4m3_encoder():
    top = int(np.array(500.0, dtype=np.float32).view(np.uint32))
    s = _bits_f32(np.arange(0, top, 97, dtype=np.uint32))
    mids = (O.e4m3_decode(np.arange(126)).astype(np.float64) + O.e4m3_decode(np.arange(1, 127)).astype(np.float64)) / 2
    s = np.concatenate([s, mids.astype(np.float32)]).astype(np.float32)
    got = O.e4m3_decode(O.e4m3_encode_satfinite(s)).astype(np.float64)
    want = _e4m3_closed_form(s)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (s[bad[:5]], got[bad[:5]], want[bad[:5]])


def check_e4m3_relative_error():
    rng = np.random.default_rng(11)
    s = np.exp2(rng.uniform(-6, np.log2(448.0), 200000)).astype(np.float32)
    got = O.e4m3_decode(O.e4m3_encode_satfinite(s)).astype(np.float64)
    rel = np.abs(got - s) / s
    assert rel.max() <= FACTS["e4m3_rel_error"], rel.max()


# --------------------------------------------------------------------------
# Two-level quantization
# --------------------------------------------------------------------------
def _random_tensor(rows, k, seed, outliers=True):
    if outliers:
        return inputs.activations_with_outliers(rows, k, seed=seed, fraction=0.05, factor=40.0)
    return inputs.gaussian_bf16((rows, k), seed=seed)


def check_global_scale():
    """g is the fp32 reciprocal of the page's s_global = amax / (6 * 448)."""
    for a in [1.0, 3.5, 0.0078125, 123.456, 1e-3, 65504.0]:
        g = O.global_scale(np.float32(a))
        s_global = np.float64(np.float32(a)) / (FACTS["e2m1_max"] * FACTS["e4m3_max"])
        assert abs(np.float64(g) * s_global - 1.0) <= 2.0 ** -23, (a, g)
    assert FACTS["e2m1_max"] * FACTS["e4m3_max"] == FACTS["global_divisor"]
    assert O.global_scale(np.float32(0.0)) == np.float32(1.0)
    with pytest.raises(O.RangeError):
        O.global_scale(np.float32(1e-38))


def check_amax_block_saturates():
    """The block holding the tensor amax gets scale 448 and its amax element code +-6:
    the reason for the 6 * 448 factor ("low-precision-floats", NVFP4)."""
    for seed in (21, 22, 23):
        x = _random_tensor(64, 256, seed)
        packed, sf, g, a = O.quantize(x)
        codes = O.unpack_codes(packed)
        xf = O.bf16_to_f32(x)
        r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
        assert sf[r, c // 16] == 0x7E, (seed, hex(sf[r, c // 16]))
        assert codes[r, c] & 7 == 7, (seed, codes[r, c])
        assert bool(codes[r, c] & 8) == bool(xf[r, c] < 0)


def _blocks(x_bits, packed, sf, g):
    xf = O.bf16_to_f32(x_bits).astype(np.float64)
    xh = O.dequantize(packed, sf, g)
    rows, k = xf.shape
    A = np.max(np.abs(xf.reshape(rows, k // 16, 16)), axis=2)
    sd = O.e4m3_decode(sf).astype(np.float64)
    return xf, xh, A, sd


def check_error_bound():
    """|x - x_hat| <= 3A/16 per element, for blocks whose E4M3 scale is normal."""
    for seed in (31, 32):
        x = _random_tensor(128, 512, seed)
        packed, sf, g, _ = O.quantize(x)
        xf, xh, A, sd = _blocks(x, packed, sf, g)
        err = np.abs(xf - xh).reshape(A.shape + (16,))
        normal = sd >= 2.0 ** -6
        assert normal.sum() > 100
        lim = FACTS["nvfp4_abs_error_over_amax"] * A[:, :, None]
        assert np.all(err[normal] <= lim[normal]), np.max((err / np.maximum(lim, 1e-300))[normal])


def check_zero_threshold():
    """|x| < 0.25 s_nv quantizes to +-0, and 0.25 s_nv <= 4.69% of the block amax."""
    for seed in (41, 42):
        x = _random_tensor(128, 512, seed)
        packed, sf, g, _ = O.quantize(x)
        codes = O.unpack_codes(packed)
        xf, _, A, sd = _blocks(x, packed, sf, g)
        s_nv = (sd / np.float64(g))[:, :, None]
        ratio = (np.abs(xf).reshape(A.shape + (16,)) / np.where(s_nv > 0, s_nv, np.inf))
        cz = (codes.reshape(A.shape + (16,)) & 7) == 0
        assert np.all(cz[ratio < 0.25 * (1 - 2.0 ** -20)])
        assert not np.any(cz[ratio > 0.25 * (1 + 2.0 ** -20)])
        normal = sd >= 2.0 ** -6
        thr = 0.25 * s_nv[:, :, 0]
        assert np.all(thr[normal] <= FACTS["nvfp4_zero_threshold_over_amax"] * A[normal])


def check_bits_per_value():
    x = _random_tensor(32, 1024, 51, outliers=False)
    packed, sf, g, _ = O.quantize(x)
    bits = (packed.nbytes + sf.nbytes) * 8 / x.size
    assert bits == FACTS["bits_per_value"]
    assert sf.shape[1] * FACTS["block"] == x.shape[1]


def check_bruteforce_nearest_code():
    """Each code is the nearest of the 16 E2M1 values to x*g/sd (ties even,
    saturating); where x*g/sd sits within fp32 rounding of a tie, both are allowed."""
    x = _random_tensor(8, 64, 61)
    packed, sf, g, _ = O.quantize(x)
    codes = O.unpack_codes(packed)
    xf = O.bf16_to_f32(x).astype(np.float64)
    sd = np.repeat(O.e4m3_decode(sf).astype(np.float64), 16, axis=1)
    cand = O.e2m1_decode(np.arange(16))
    for i in range(xf.shape[0]):
        for j in range(xf.shape[1]):
            if sd[i, j] == 0:
                assert codes[i, j] == 0
                continue
            v = xf[i, j] * np.float64(g) / sd[i, j]
            d = np.abs(cand - v)
            best = d.min()
            ok = [c for c in range(16) if d[c] <= best * (1 + 2.0 ** -20) + 1e-300
                  and (np.signbit(cand[c]) == (v < 0) or cand[c] != 0)]
            assert codes[i, j] in ok, (i, j, v, codes[i, j], ok)


def check_packing_low_nibble_first():
    """FP4 wiki (技術原理): the first element goes in the low 4 bits."""
    row = np.zeros((1, 16), dtype=np.float64)
    row[0, 0], row[0, 1] = 1.0, -0.5            # amax 1: u0 = 6 -> code 7, u1 = -3 -> code 13
    x = inputs.f64_to_bf16_bits(row)
    packed, sf, g, _ = O.quantize(x)
    assert sf[0, 0] == 0x7E
    assert packed[0, 0] == 0xD7, hex(packed[0, 0])


# --------------------------------------------------------------------------
# Block-scaled GEMM
# --------------------------------------------------------------------------
def _random_codes(rng, rows, k):
    return O.pack_codes(rng.integers(0, 16, size=(rows, k), dtype=np.uint8))


def check_gemm_unit_scales_is_plain_matmul():
    """Unit block scales and g = 1 reduce to a matmul of E2M1 values, done here
    exactly in integers (2 * every E2M1 value is an integer)."""
    rng = np.random.default_rng(71)
    M, N, K = 24, 40, 96
    a, b = _random_codes(rng, M, K), _random_codes(rng, N, K)
    one = np.full((M, K // 16), 0x38, np.uint8)
    onen = np.full((N, K // 16), 0x38, np.uint8)
    d, s, alpha = O.gemm_ref(a, one, 1.0, b, onen, 1.0)
    twice = np.array([0, 1, 2, 3, 4, 6, 8, 12, 0, -1, -2, -3, -4, -6, -8, -12], np.int64)
    ia = twice[O.unpack_codes(a)]
    ib = twice[O.unpack_codes(b)]
    exact = ia @ ib.T
    assert alpha == 1.0
    assert np.array_equal(d * 4, exact.astype(np.float64))
    assert np.array_equal(s * 4, (np.abs(ia) @ np.abs(ib).T).astype(np.float64))


def check_gemm_bruteforce_loops():
    rng = np.random.default_rng(72)
    M, N, K = 3, 5, 48
    a, b = _random_codes(rng, M, K), _random_codes(rng, N, K)
    sa = rng.integers(0, 0x7F, size=(M, K // 16), dtype=np.uint8)
    sb = rng.integers(0, 0x7F, size=(N, K // 16), dtype=np.uint8)
    ga, gb = np.float32(37.5), np.float32(0.125)
    d, s, alpha = O.gemm_ref(a, sa, ga, b, sb, gb)
    ca, cb = O.unpack_codes(a), O.unpack_codes(b)
    table = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    def val(c):
        return -table[c & 7] if c & 8 else table[c & 7]
    def e4m3(byte):
        e, m = (byte >> 3) & 15, byte & 7
        return m / 512.0 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
    for i in range(M):
        for j in range(N):
            acc = 0.0
            for kk in range(K):
                acc += val(int(ca[i, kk])) * e4m3(int(sa[i, kk // 16])) * val(int(cb[j, kk])) * e4m3(int(sb[j, kk // 16]))
            ref = float(np.float32(1.0) / (ga * gb)) * acc
            assert abs(d[i, j] - ref) <= 1e-12 * max(1.0, abs(ref)), (i, j, d[i, j], ref)


def check_gemm_block_broadcast():
    """A non-unit scale on (row 0, block 1) scales exactly elements 16..31 of row 0."""
    rng = np.random.default_rng(73)
    M, N, K = 4, 6, 64
    a, b = _random_codes(rng, M, K), _random_codes(rng, N, K)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sb = np.full((N, K // 16), 0x38, np.uint8)
    d1, _, _ = O.gemm_ref(a, sa, 1.0, b, sb, 1.0)
    sa2 = sa.copy()
    sa2[0, 1] = 0x40                                # 2.0
    d2, _, _ = O.gemm_ref(a, sa2, 1.0, b, sb, 1.0)
    va = O.e2m1_decode(O.unpack_codes(a))
    vb = O.e2m1_decode(O.unpack_codes(b))
    extra = va[0, 16:32] @ vb[:, 16:32].T
    assert np.array_equal(d2[1:], d1[1:])
    assert np.allclose(d2[0] - d1[0], extra, rtol=0, atol=1e-12)


def check_gemm_matches_dequantized_product():
    """D = alpha (s_a A)(s_b W)^T equals x_hat_a @ x_hat_b^T with x_hat = s_global s_block q."""
    xa = _random_tensor(16, 128, 81)
    xb = _random_tensor(24, 128, 82, outliers=False)
    pa, sa, ga, _ = O.quantize(xa)
    pb, sb, gb, _ = O.quantize(xb)
    d, s, alpha = O.gemm_ref(pa, sa, ga, pb, sb, gb)
    ref = O.dequantize(pa, sa, ga) @ O.dequantize(pb, sb, gb).T
    assert np.all(np.abs(d - ref) <= 2.0 ** -22 * (np.abs(ref) + s * float(alpha))), np.max(np.abs(d - ref))


def check_swizzle_round_trip():
    rng = np.random.default_rng(91)
    for rows, k in [(128, 64), (200, 320), (1, 16), (257, 1024)]:
        sf = rng.integers(0, 0x7F, size=(rows, k // 16), dtype=np.uint8)
        flat = O.swizzle_sf_tcgen05(sf)
        assert flat.size == O.sf_tcgen05_bytes(rows, k)
        assert np.array_equal(O.unswizzle_sf_tcgen05(flat, rows, k), sf)
        assert int(flat.astype(np.int64).sum()) == int(sf.astype(np.int64).sum())


CHECKS = [
    check_e2m1_table, check_e2m1_onnx_rule, check_e2m1_encoder,
    check_e4m3_page_example, check_e4m3_grid, check_e4m3_max_and_saturation,
    check_e4m3_encoder, check_e4m3_relative_error,
    check_global_scale, check_amax_block_saturates, check_error_bound,
    check_zero_threshold, check_bits_per_value, check_bruteforce_nearest_code,
    check_packing_low_nibble_first,
    check_gemm_unit_scales_is_plain_matmul, check_gemm_bruteforce_loops,
    check_gemm_block_broadcast, check_gemm_matches_dequantized_product,
    check_swizzle_round_trip,
]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()


# --------------------------------------------------------------------------
# Planted mistakes: each plausible error in the oracle trips at least one pin
# --------------------------------------------------------------------------
def _mut_table(mp):
    mp.setattr(O, "E2M1_MAGNITUDES", np.array([0, 0.5, 1, 1.5, 2, 3, 4, 5], dtype=np.float64))


def _mut_ties_away(mp):
    real = O.e2m1_encode
    def enc(u):
        u = np.asarray(u, dtype=np.float32)
        with np.errstate(over="ignore"):
            bumped = np.where(np.isin(np.abs(u), _f32([0.25, 1.25, 2.5, 5.0])), u * np.float32(1.0000001), u)
        return real(bumped.astype(np.float32))
    mp.setattr(O, "e2m1_encode", enc)


def _mut_e4m3_truncate(mp):
    vals = O.e4m3_decode(np.arange(127)).astype(np.float64)
    def enc(s):
        a = np.asarray(s, dtype=np.float32).astype(np.float64)
        return np.clip(np.searchsorted(vals, a, side="right") - 1, 0, 126).astype(np.uint8)
    mp.setattr(O, "e4m3_encode_satfinite", enc)


def _mut_single_level(mp):
    mp.setattr(O, "global_scale", lambda a: np.float32(6.0) / np.float32(a) if a else np.float32(1.0))


def _mut_nibbles(mp):
    mp.setattr(O, "pack_codes", lambda c: (np.asarray(c)[..., 1::2] | (np.asarray(c)[..., 0::2] << 4)).astype(np.uint8))
    mp.setattr(O, "unpack_codes", lambda p: np.stack([np.asarray(p) >> 4, np.asarray(p) & 15], -1).reshape(np.asarray(p).shape[:-1] + (-1,)).astype(np.uint8))


def _mut_no_div6(mp):
    real = O.quantize_with_scale
    mp.setattr(O, "quantize_with_scale", lambda x, g: real(x, np.float32(g) * np.float32(6.0)))


def _mut_alpha(mp):
    mp.setattr(O, "gemm_alpha", lambda ga, gb: np.float32(np.float32(ga) * np.float32(gb)))


def _mut_block_index(mp):
    def deq(packed, sf):
        q = O.e2m1_decode(O.unpack_codes(packed))
        rows, k = q.shape
        sd = O.e4m3_decode(sf).astype(np.float64)
        return (q.reshape(rows, 16, k // 16) * sd[:, None, :]).reshape(rows, k)   # k % nblk, not k // 16
    mp.setattr(O, "dequantize_blocks", deq)


MUTATIONS = [_mut_table, _mut_ties_away, _mut_e4m3_truncate, _mut_single_level,
             _mut_nibbles, _mut_no_div6, _mut_alpha, _mut_block_index]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_planted_mistakes(mutate, monkeypatch):
    mutate(monkeypatch)
    caught = []
    for check in CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError, O.RangeError):
            caught.append(check.__name__)
            break
    assert caught, f"no pin catches {mutate.__name__}"
