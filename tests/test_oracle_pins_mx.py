"""Pins of the MXFP4 oracle against what the pages fix (CPU only).

[P2] mxFP4/nvFP4 最小化知识, (一) mxFP4的技术局限: 32 elements share one E8M0
     scale; an optimal scale of 0.9 can only become 0.5 or 1.0 and becomes 1.0,
     an 11.1 % scale error.
[P4] low-precision-floats, FP4 / MXFP4 / NVFP4: s_mx = 2^ceil(log2(A/6))
     ("TensorRT usually rounds up"), 1 <= rho_mx < 2, A/6 = 1.99 -> 2 and
     2.01 -> 4, |e| <= s_mx < A/3, zero threshold 0.25 s_mx in [A/24, A/12].
"""
import numpy as np
import pytest

from oracle import mxfp4_oracle as MX
from oracle import nvfp4_oracle as NV
from nvfp4_block_scaled_15_b200 import inputs


def _bf16(v):
    return inputs.f64_to_bf16_bits(np.asarray(v, dtype=np.float64))


def _scale(a):
    return MX.e8m0_decode(MX.mx_scale_exponent(np.float32(a)) + MX.E8M0_BIAS)


def test_p2_optimal_scale_0_9_becomes_1_0():
    # A = 5.40625 (a bf16 value) gives A/6 = 0.901..., between 0.5 and 1.0
    a = NV.bf16_to_f32(_bf16([5.40625]))[0]
    assert 0.89 < a / 6 < 0.91
    assert _scale(a) == 1.0
    assert abs((1.0 - 0.9) / 0.9 - 0.111) < 1e-3          # the page's 11.1 %


def test_p4_rounding_up_examples():
    # A/6 = 1.99 rounds up to 2 (rho ~ 1), 2.01 to 4 (rho ~ 2)
    lo = NV.bf16_to_f32(_bf16([11.9375]))[0]               # A/6 = 1.9896
    hi = NV.bf16_to_f32(_bf16([12.0625]))[0]               # A/6 = 2.0104
    assert _scale(lo) == 2.0 and _scale(hi) == 4.0
    assert 1.0 <= _scale(lo) / (lo / 6) < 1.01
    assert 1.98 < _scale(hi) / (hi / 6) < 2.0


def test_rho_in_one_two_and_powers_of_two_exact():
    rng = np.random.default_rng(5)
    a = NV.bf16_to_f32(_bf16(np.exp(rng.uniform(-60, 60, 20000))))
    s = _scale(a)
    rho = s / (a.astype(np.float64) / 6)
    assert np.all(rho >= 1.0) and np.all(rho < 2.0)
    # A = 6 * 2^j: the scale is exactly 2^j
    j = np.arange(-100, 100)
    assert np.array_equal(_scale(np.ldexp(np.float32(6.0), j)), np.ldexp(1.0, j))


def test_error_bound_zero_threshold_and_no_saturation():
    x = inputs.activations_with_outliers(64, 1024, seed=21, fraction=0.02, factor=40.0)
    packed, sf = MX.quantize_mx(x)
    xf = NV.bf16_to_f32(x).astype(np.float64).reshape(64, 32, 32)
    xh = MX.dequantize_mx(packed, sf).reshape(64, 32, 32)
    s = MX.e8m0_decode(sf)[:, :, None]
    a = np.max(np.abs(xf), axis=2, keepdims=True)
    err = np.abs(xf - xh)
    assert np.all(err <= s) and np.all(err < a / 3)                 # |e| <= s_mx < A/3
    assert np.all((0.25 * s >= a / 24) & (0.25 * s <= a / 12))      # threshold in [A/24, A/12]
    codes = NV.unpack_codes(packed).reshape(64, 32, 32)
    small = np.abs(xf) < 0.25 * s
    assert np.all((codes[small] & 7) == 0)                          # below the threshold -> +-0
    assert np.all(np.abs(xf) / s <= 6.0)                            # rounding up: no saturation


def test_codes_are_nearest_e2m1_of_scaled_values():
    x = inputs.gaussian_bf16((8, 256), seed=33)
    packed, sf = MX.quantize_mx(x)
    u = NV.bf16_to_f32(x).astype(np.float64).reshape(8, 8, 32) / MX.e8m0_decode(sf)[:, :, None]
    codes = NV.unpack_codes(packed).reshape(8, 8, 32)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for c, v in zip(codes.reshape(-1), u.reshape(-1)):
        d = np.abs(mags - abs(v))
        best = np.flatnonzero(d == d.min())
        want = best[0] if best.size == 1 else best[best % 2 == 0][0]   # ties to the even code
        assert (c & 7) == want and ((c & 8) != 0) == np.signbit(v)


def test_one_scale_per_32_elements():
    # a large value in elements 16..31 must set the scale of elements 0..15 too
    x = np.full((1, 64), 0.5)
    x[0, 20] = 48.0
    packed, sf = MX.quantize_mx(_bf16(x))
    assert sf.shape == (1, 2)
    assert MX.e8m0_decode(sf[0, 0]) == 8.0 and MX.e8m0_decode(sf[0, 1]) == 0.125


def test_e8m0_bytes_are_torch_float8_e8m0fnu():
    """P2 names torch.float8_e8m0fnu as the scale type: the stored bytes decode
    to the same powers of two under it, and A = 6 stores scale 1.0 as 127."""
    import torch
    b = np.arange(0, 255, dtype=np.uint8)
    ref = torch.from_numpy(b).view(torch.float8_e8m0fnu).double().numpy()
    assert np.array_equal(MX.e8m0_decode(b), ref)
    _, sf = MX.quantize_mx(_bf16(np.full((1, 32), 6.0)))
    assert sf[0, 0] == 127


def test_all_zero_block_and_nonfinite():
    packed, sf = MX.quantize_mx(_bf16(np.zeros((1, 32))))
    assert sf[0, 0] == 0 and not packed.any()
    bad = _bf16(np.zeros((1, 32)))
    bad[0, 3] = 0x7F80
    with pytest.raises(NV.RangeError):
        MX.quantize_mx(bad)


def test_unit_scale_gemm_is_integer_matmul_and_triple_loop():
    rng = np.random.default_rng(9)
    ca = rng.integers(0, 16, (3, 64), dtype=np.uint8)
    cb = rng.integers(0, 16, (5, 64), dtype=np.uint8)
    one = np.full((3, 2), 127, np.uint8)
    d, s = MX.gemm_ref_mx(NV.pack_codes(ca), one, NV.pack_codes(cb), np.full((5, 2), 127, np.uint8))
    ia = (NV.e2m1_decode(ca) * 2).astype(np.int64)       # E2M1 values are multiples of 0.5
    ib = (NV.e2m1_decode(cb) * 2).astype(np.int64)
    assert np.array_equal(d * 4, (ia @ ib.T).astype(np.float64))
    # scaled: a plain triple loop
    sa = rng.integers(120, 135, (3, 2)).astype(np.uint8)
    sb = rng.integers(120, 135, (5, 2)).astype(np.uint8)
    d, _ = MX.gemm_ref_mx(NV.pack_codes(ca), sa, NV.pack_codes(cb), sb)
    for i in range(3):
        for j in range(5):
            acc = 0.0
            for kk in range(64):
                acc += (NV.e2m1_decode(ca[i, kk]) * 2.0 ** (int(sa[i, kk // 32]) - 127)
                        * NV.e2m1_decode(cb[j, kk]) * 2.0 ** (int(sb[j, kk // 32]) - 127))
            assert d[i, j] == acc


def _pins_fail_with(monkeypatch, name, fn):
    monkeypatch.setattr(MX, name, fn)
    failures = 0
    for t in (test_p2_optimal_scale_0_9_becomes_1_0, test_p4_rounding_up_examples,
              test_rho_in_one_two_and_powers_of_two_exact, test_error_bound_zero_threshold_and_no_saturation,
              test_one_scale_per_32_elements, test_e8m0_bytes_are_torch_float8_e8m0fnu):
        try:
            t()
        except (AssertionError, ValueError):     # a broken shape counts as caught too
            failures += 1
    return failures


def test_planted_mistakes_are_caught(monkeypatch):
    real_exp = MX.mx_scale_exponent

    def rounded(a):                       # round(log2(A/6)) instead of rounding up
        v = np.asarray(a, dtype=np.float32) / np.float32(6)
        return np.clip(np.rint(np.log2(np.maximum(v, 1e-45))).astype(np.int64), -127, 127)

    def floored(a):
        return real_exp(a) - (np.asarray(a) > 0) * 1

    def no_sixth(a):                      # forget the /6
        return real_exp(np.asarray(a, dtype=np.float32) * np.float32(6))

    for name, fn in [("mx_scale_exponent", rounded), ("mx_scale_exponent", floored),
                     ("mx_scale_exponent", no_sixth)]:
        with monkeypatch.context() as m:
            assert _pins_fail_with(m, name, fn) > 0, name
    with monkeypatch.context() as m:      # one scale per 16 elements
        m.setattr(MX, "MX_BLOCK", 16)
        assert _pins_fail_with(m, "MX_BLOCK", 16) > 0
    with monkeypatch.context() as m:      # wrong E8M0 bias
        m.setattr(MX, "E8M0_BIAS", 128)
        assert _pins_fail_with(m, "E8M0_BIAS", 128) > 0
