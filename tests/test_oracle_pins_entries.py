"""Pins of the oracle functions the full-size parity tests lean on.

* ``f64_to_bf16_rne`` defines the "1 bf16 ulp of the oracle's rounded value"
  every bf16 output check uses.  It is pinned against two roundings written
  independently of it: round-half-even on the fp64 bit pattern in integer
  arithmetic, and torch's fp32 -> bf16 conversion on fp32-exact inputs; over
  every bf16 value, every midpoint between neighbours (ties go to the even
  pattern), each midpoint's fp64 neighbours (a rounding through fp32 first
  would turn them into ties), subnormals, overflow and a random sweep.
* ``gemm_ref_entries`` and ``mxfp4_oracle.gemm_ref_mx_entries`` compute the
  reference at listed coordinates for the full-size GEMM/GEMV tests.  They
  must equal the whole-matrix references (``gemm_ref`` / ``gemm_ref_mx``) at
  every coordinate of small cases, in any coordinate order, and a pure-Python
  triple loop written from the scaled-GEMM definition ("NVIDIA NVFP4 与
  Micro-Scaling" section 三; the MXFP4 form from "low-precision-floats",
  FP4 / MXFP4 / NVFP4).
``test_planted_mistakes`` plants a truncating or twice-rounding bf16
conversion and swapped or shifted indexes, and shows a pin catches each.
"""
import numpy as np
import pytest
import torch

from oracle import mxfp4_oracle as MX
from oracle import nvfp4_oracle as O

# --------------------------------------------------------------------------
# bf16 rounding, restated independently
# --------------------------------------------------------------------------
_BF16_MAX = float(np.uint32(0x7F7F0000).view(np.float32))


def _rne_int(v: float) -> int:
    """bf16 bits of one finite fp64 value by integer round-half-even.

    Normal range (|v| >= 2^-126): keep the fp64 sign, exponent and top 7
    fraction bits, round on the 45 dropped bits; a carry runs into the
    exponent by plain integer addition.  Below 2^-126 the bf16 grid is
    m * 2^-133: v * 2^133 is exact in fp64 and Python's round() rounds a
    float half to even.  Results at or beyond 2^128 are infinities."""
    if v == 0.0:
        return 0x8000 if np.signbit(v) else 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    if a < 2.0 ** -126:
        q = round(a * 2.0 ** 133)                       # 0 .. 128 (128 is the smallest normal)
        return sign | q
    bits = int(np.float64(a).view(np.uint64))
    q, rem = bits >> 45, bits & ((1 << 45) - 1)
    half = 1 << 44
    if rem > half or (rem == half and (q & 1)):
        q += 1
    val = float(np.uint64(q << 45).view(np.float64))   # 8 significant bits: exact in fp32
    if val >= 2.0 ** 128:
        return sign | 0x7F80
    return sign | int(np.float32(val).view(np.uint32) >> 16)


def _finite_bf16_patterns():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (b >> 7) & 0xFF
    return b[exp != 0xFF]


def _bf16_values(bits):
    return O.bf16_to_f32(bits).astype(np.float64)


def check_bf16_every_value_kept():
    b = _finite_bf16_patterns()
    got = O.f64_to_bf16_rne(_bf16_values(b))
    assert np.array_equal(got, b)


def _midpoints():
    """Midpoints between consecutive positive finite bf16 values, with the
    even pattern of each pair, and the midpoint above the largest value."""
    lo = np.arange(0, 0x7F7F, dtype=np.uint16)
    hi = lo + 1
    mid = (_bf16_values(lo) + _bf16_values(hi)) / 2            # exact in fp64
    even = np.where(lo % 2 == 0, lo, hi).astype(np.uint16)
    return mid, even


def check_bf16_ties_to_even():
    mid, even = _midpoints()
    assert np.array_equal(O.f64_to_bf16_rne(mid), even)
    assert np.array_equal(O.f64_to_bf16_rne(-mid), even | np.uint16(0x8000))


def check_bf16_near_ties():
    """One fp64 ulp either side of each tie decides it (a rounding through
    fp32 first would see an exact tie and go to the even pattern)."""
    mid, _ = _midpoints()
    lo = np.arange(0, 0x7F7F, dtype=np.uint16)
    above = np.nextafter(mid, np.inf)
    below = np.nextafter(mid, -np.inf)
    assert np.array_equal(O.f64_to_bf16_rne(above), (lo + 1).astype(np.uint16))
    assert np.array_equal(O.f64_to_bf16_rne(below), lo)


def check_bf16_against_integer_rounding():
    rng = np.random.default_rng(2024)
    e = rng.uniform(-140, 128, 200_000)
    v = rng.choice([-1.0, 1.0], e.size) * np.exp2(e) * rng.uniform(1, 2, e.size)
    v = v[np.abs(v) < 2.0 ** 128]
    v = np.concatenate([v, [0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 2.0 ** -126,
                            np.nextafter(2.0 ** -126, 0), _BF16_MAX, -_BF16_MAX]])
    got = O.f64_to_bf16_rne(v)
    want = np.array([_rne_int(float(t)) for t in v], dtype=np.uint16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:4]], got[bad[:4]], want[bad[:4]])


def check_bf16_against_torch():
    """fp32-exact inputs (fp64 -> fp32 is then exact): torch's fp32 -> bf16 cast."""
    rng = np.random.default_rng(77)
    f = rng.integers(0, 0x7F7FFFFF, 400_000, dtype=np.uint32)
    f = np.concatenate([f, f | np.uint32(0x80000000)]).view(np.float32)
    f = f[np.isfinite(f)]
    mid, _ = _midpoints()
    f = np.concatenate([f, mid.astype(np.float32)])            # ties are fp32-exact
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f64_to_bf16_rne(f.astype(np.float64))
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (f[bad[:4]], got[bad[:4]], want[bad[:4]])


def check_bf16_overflow():
    top_mid = _BF16_MAX + 2.0 ** (127 - 8)                      # halfway to 2^128
    assert O.f64_to_bf16_rne(np.array([top_mid]))[0] == 0x7F80  # tie: even is the "2^128" pattern, inf
    assert O.f64_to_bf16_rne(np.array([np.nextafter(top_mid, 0)]))[0] == 0x7F7F
    assert O.f64_to_bf16_rne(np.array([-1e39]))[0] == 0xFF80


# --------------------------------------------------------------------------
# Entry-wise GEMM references
# --------------------------------------------------------------------------
_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e2m1(c):
    return -_TABLE[c & 7] if c & 8 else _TABLE[c & 7]


def _e4m3(byte):
    e, m = (byte >> 3) & 15, byte & 7
    return m / 512.0 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)


def _nv_case(seed, m=5, n=7, k=64):
    rng = np.random.default_rng(seed)
    a = rng.integers(0, 256, (m, k // 2), dtype=np.uint8)
    b = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    sa = rng.integers(0, 0x7F, (m, k // 16), dtype=np.uint8)
    sb = rng.integers(0, 0x7F, (n, k // 16), dtype=np.uint8)
    return a, sa, np.float32(3.75), b, sb, np.float32(0.3125)


def check_entries_equal_whole_matrix():
    a, sa, ga, b, sb, gb = _nv_case(5)
    d, s, alpha = O.gemm_ref(a, sa, ga, b, sb, gb)
    m, n = d.shape
    rows = np.repeat(np.arange(m), n)
    cols = np.tile(np.arange(n), m)
    perm = np.random.default_rng(6).permutation(rows.size)
    rows, cols = np.concatenate([rows[perm], [2, 2]]), np.concatenate([cols[perm], [3, 3]])
    de, se, alpha_e = O.gemm_ref_entries(a, sa, ga, b, sb, gb, rows, cols)
    assert alpha_e == alpha
    tol = 1e-13 * s[rows, cols] * float(alpha)
    assert np.all(np.abs(de - d[rows, cols]) <= tol)
    assert np.all(np.abs(se - s[rows, cols]) <= 1e-13 * s[rows, cols])


def check_entries_triple_loop():
    a, sa, ga, b, sb, gb = _nv_case(9, m=3, n=4, k=48)
    ca, cb = O.unpack_codes(a), O.unpack_codes(b)
    rows, cols = np.array([0, 2, 1, 2, 0]), np.array([3, 0, 1, 2, 0])
    de, se, alpha = O.gemm_ref_entries(a, sa, ga, b, sb, gb, rows, cols)
    al = float(np.float32(1.0) / (ga * gb))
    for i, (r, c) in enumerate(zip(rows, cols)):
        acc = sum(_e2m1(int(ca[r, kk])) * _e4m3(int(sa[r, kk // 16])) * _e2m1(int(cb[c, kk])) * _e4m3(int(sb[c, kk // 16]))
                  for kk in range(ca.shape[1]))
        mag = sum(abs(_e2m1(int(ca[r, kk])) * _e4m3(int(sa[r, kk // 16])) * _e2m1(int(cb[c, kk])) * _e4m3(int(sb[c, kk // 16])))
                  for kk in range(ca.shape[1]))
        assert abs(de[i] - al * acc) <= 1e-12 * max(1.0, abs(al) * mag), (r, c)
        assert abs(se[i] - mag) <= 1e-12 * max(1.0, mag), (r, c)


def _mx_case(seed, m=4, n=6, k=96):
    rng = np.random.default_rng(seed)
    a = rng.integers(0, 256, (m, k // 2), dtype=np.uint8)
    b = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    sa = rng.integers(110, 140, (m, k // 32), dtype=np.uint8)
    sb = rng.integers(110, 140, (n, k // 32), dtype=np.uint8)
    return a, sa, b, sb


def check_mx_entries_equal_whole_matrix():
    a, sa, b, sb = _mx_case(11)
    d, s = MX.gemm_ref_mx(a, sa, b, sb)
    m, n = d.shape
    rows = np.repeat(np.arange(m), n)
    cols = np.tile(np.arange(n), m)
    perm = np.random.default_rng(12).permutation(rows.size)
    rows, cols = rows[perm], cols[perm]
    de, se = MX.gemm_ref_mx_entries(a, sa, b, sb, rows, cols)
    assert np.all(np.abs(de - d[rows, cols]) <= 1e-13 * s[rows, cols])
    assert np.all(np.abs(se - s[rows, cols]) <= 1e-13 * s[rows, cols])


def check_mx_entries_triple_loop():
    a, sa, b, sb = _mx_case(13, m=3, n=3, k=64)
    ca, cb = O.unpack_codes(a), O.unpack_codes(b)
    rows, cols = np.array([2, 0, 1]), np.array([1, 2, 0])
    de, se = MX.gemm_ref_mx_entries(a, sa, b, sb, rows, cols)
    for i, (r, c) in enumerate(zip(rows, cols)):
        terms = [_e2m1(int(ca[r, kk])) * 2.0 ** (int(sa[r, kk // 32]) - 127)
                 * _e2m1(int(cb[c, kk])) * 2.0 ** (int(sb[c, kk // 32]) - 127) for kk in range(ca.shape[1])]
        assert de[i] == sum(terms), (r, c)          # powers of two times small integers: exact
        assert se[i] == sum(abs(t) for t in terms), (r, c)


CHECKS = [
    check_bf16_every_value_kept, check_bf16_ties_to_even, check_bf16_near_ties,
    check_bf16_against_integer_rounding, check_bf16_against_torch, check_bf16_overflow,
    check_entries_equal_whole_matrix, check_entries_triple_loop,
    check_mx_entries_equal_whole_matrix, check_mx_entries_triple_loop,
]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()


# --------------------------------------------------------------------------
# Planted mistakes (on the CPU, in the oracle)
# --------------------------------------------------------------------------
def _mut_bf16_truncate(mp):
    def trunc(v):
        y = np.asarray(v, dtype=np.float64).astype(np.float32)
        return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    mp.setattr(O, "f64_to_bf16_rne", trunc)


def _mut_bf16_via_fp32(mp):
    real = O.f64_to_bf16_rne
    mp.setattr(O, "f64_to_bf16_rne", lambda v: real(np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)))


def _mut_bf16_ties_away(mp):
    def away(v):
        v = np.asarray(v, dtype=np.float64)
        _, exp = np.frexp(v)
        exp = np.maximum(exp, -125)
        t = np.ldexp(v, 8 - exp)
        q = np.sign(t) * np.floor(np.abs(t) + 0.5)
        with np.errstate(over="ignore"):
            y = np.ldexp(q, exp - 8).astype(np.float32)
        return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    mp.setattr(O, "f64_to_bf16_rne", away)


def _mut_entries_swapped(mp):
    real = O.gemm_ref_entries
    mp.setattr(O, "gemm_ref_entries", lambda a, sa, ga, b, sb, gb, rows, cols: real(a, sa, ga, b, sb, gb, cols, rows))


def _mut_entries_scale_row(mp):
    def entries(a, sa, ga, b, sb, gb, rows, cols):
        alpha = O.gemm_alpha(ga, gb)
        d, s = np.empty(len(rows)), np.empty(len(rows))
        for i, (r, c) in enumerate(zip(rows, cols)):
            ar = O.dequantize_blocks(a[r:r + 1], sa[c % sa.shape[0]:c % sa.shape[0] + 1])[0]   # B's row index on A's scales
            bc = O.dequantize_blocks(b[c:c + 1], sb[c:c + 1])[0]
            d[i] = np.float64(alpha) * np.dot(ar, bc)
            s[i] = np.dot(np.abs(ar), np.abs(bc))
        return d, s, alpha
    mp.setattr(O, "gemm_ref_entries", entries)


def _mut_mx_entries_swapped(mp):
    def entries(a, sa, b, sb, rows, cols):
        d, s = np.empty(len(rows)), np.empty(len(rows))
        for i, (r, c) in enumerate(zip(rows, cols)):
            ar = MX.dequantize_mx(a[r:r + 1], sa[r:r + 1])[0]
            bc = MX.dequantize_mx(b[c:c + 1], sb[r % sb.shape[0]:r % sb.shape[0] + 1])[0]   # A's row picks B's scales
            d[i] = np.dot(ar, bc)
            s[i] = np.dot(np.abs(ar), np.abs(bc))
        return d, s
    mp.setattr(MX, "gemm_ref_mx_entries", entries)


def _mut_mx_entries_no_scale(mp):
    def entries(a, sa, b, sb, rows, cols):
        d, s = np.empty(len(rows)), np.empty(len(rows))
        for i, (r, c) in enumerate(zip(rows, cols)):
            ar = O.e2m1_decode(O.unpack_codes(a[r]))
            bc = MX.dequantize_mx(b[c:c + 1], sb[c:c + 1])[0]
            d[i] = np.dot(ar, bc)
            s[i] = np.dot(np.abs(ar), np.abs(bc))
        return d, s
    mp.setattr(MX, "gemm_ref_mx_entries", entries)


MUTATIONS = [_mut_bf16_truncate, _mut_bf16_via_fp32, _mut_bf16_ties_away, _mut_entries_swapped,
             _mut_entries_scale_row, _mut_mx_entries_swapped, _mut_mx_entries_no_scale]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_planted_mistakes(mutate, monkeypatch):
    mutate(monkeypatch)
    caught = []
    for check in CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
            break
    assert caught, f"no pin catches {mutate.__name__}"
