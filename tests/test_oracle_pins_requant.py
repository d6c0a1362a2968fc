"""Pins of the oracle's output-scale functions (FP8 and NVFP4 outputs of the
GEMM under the output scale g_d) against what the pages and independent
routines fix (CPU only).

[P1] "NVIDIA NVFP4 与 Micro-Scaling", section 三: D = g_d * (...); the output
     scale g_d is applied to the GEMM result, which often lands as FP8; the
     _scaled_mm example passes scale_result=g_d = 4.0 with an
     float8_e4m3fn output.
[P4] "low-precision-floats": E4M3 relative error <= 2^-4 in its normal range;
     NVFP4 error |x - x_hat| <= 3A/16 per block when g = 6 * 448 / amax.
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as O

E4M3_POS = O.e4m3_decode(np.arange(127)).astype(np.float64)


def _torch_e4m3(v):
    """Bytes of torch's own float32 -> float8_e4m3fn cast (round to nearest even)."""
    return torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _sweep_f32():
    """Signed fp32 values over the E4M3 range: every E4M3 value, every midpoint
    between neighbours, one fp32 ulp either side of each, plus a log sweep."""
    mids = (E4M3_POS[1:] + E4M3_POS[:-1]) / 2
    pts = np.concatenate([E4M3_POS, mids]).astype(np.float32)
    up = np.nextafter(pts, np.float32(np.inf))
    dn = np.nextafter(pts, np.float32(0))
    rng = np.random.default_rng(3)
    logs = np.exp2(rng.uniform(-12, np.log2(463.9), 20000)).astype(np.float32)
    mag = np.concatenate([pts, up, dn, logs, np.float32([0.0, 463.0, 463.99997])])
    mag = mag[mag < 464]
    return np.concatenate([mag, -mag]).astype(np.float32)


def check_signed_e4m3_matches_torch():
    """In the finite E4M3 range the signed encoder equals torch's RNE cast."""
    v = _sweep_f32()
    got = O.e4m3_encode_signed_satfinite(v)
    want = _torch_e4m3(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])


def check_signed_e4m3_saturates_and_keeps_sign():
    """satfinite: |v| beyond the range gives +-448 (0x7E / 0xFE); -0 is 0x80."""
    v = np.float32([464.0, 1e9, 3.4e38, -464.0, -1e9, -0.0, 0.0])
    got = O.e4m3_encode_signed_satfinite(v)
    assert got.tolist() == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x80, 0x00]


def check_fp8_output_multiplies_by_g_d():
    """P1's example g_d = 4.0: the FP8 output decodes to 4 v within E4M3's
    relative error 2^-4 (P4), for 4 v in E4M3's normal range."""
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(4096) * 20).astype(np.float32)
    v = v[(np.abs(v) * 4 >= 2.0 ** -6) & (np.abs(v) * 4 <= 448)]
    d = O.e4m3_decode(O.fp8_output(v, np.float32(4.0))).astype(np.float64)
    rel = np.abs(d - 4.0 * v) / (4.0 * np.abs(v))
    assert np.all(rel <= 2.0 ** -4)
    assert np.all(np.sign(d) == np.sign(v))


def _block_scale_independent(ab, g):
    """E4M3 of fp32(fp32(ab * g) / 6) through torch's cast, saturated at 448."""
    s = (np.float32(ab) * np.float32(g)).astype(np.float32) / np.float32(6.0)
    s = np.minimum(s.astype(np.float32), np.float32(448.0))
    return _torch_e4m3(s)


def check_fp32_values_quantizer_bruteforce():
    """fp32 inputs with full 24-bit significands: each block scale is the
    torch E4M3 cast of (ab*g)/6, each code the nearest E2M1 value to x*g/sd
    (ties even; both allowed within fp32 rounding of a tie)."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((6, 64)) * np.exp2(rng.uniform(-3, 3, (6, 1)))).astype(np.float32)
    x[2, 5] = np.float32(1.0000001) * 37
    g = np.float32(2688.0) / np.float32(np.max(np.abs(x)))
    codes, sf = O.quantize_values_with_scale(x, g)
    ab = np.max(np.abs(x.reshape(6, 4, 16)), axis=2)
    assert np.array_equal(sf, _block_scale_independent(ab, g))
    sd = np.repeat(O.e4m3_decode(sf).astype(np.float64), 16, axis=1)
    cand = O.e2m1_decode(np.arange(16))
    for i in range(6):
        for j in range(64):
            u = np.float64(x[i, j]) * np.float64(g) / sd[i, j]
            dist = np.abs(cand - u)
            ok = [c for c in range(16) if dist[c] <= dist.min() * (1 + 2.0 ** -20) + 1e-300
                  and (np.signbit(cand[c]) == (u < 0) or cand[c] != 0)]
            assert codes[i, j] in ok, (i, j, u, codes[i, j], ok)


def check_nvfp4_output_bound_and_amax():
    """With g_d = 2688 / amax(v): the amax block's scale is 448 and its largest
    element codes to +-6 (P4's reason for 6 * 448); |v - v_hat| <= 3A/16 per
    block (P4); the returned amax is max |v|."""
    rng = np.random.default_rng(17)
    v = (rng.standard_normal((32, 256)) * 3).astype(np.float32)
    v[7, 100] = np.float32(-41.25)
    amax = np.float32(np.max(np.abs(v)))
    g = np.float32(2688.0) / amax
    packed, sf, a = O.nvfp4_output(v, g)
    assert a == amax
    assert sf[7, 100 // 16] == 0x7E
    assert O.unpack_codes(packed)[7, 100] == 0xF                    # -6
    vh = O.dequantize(packed, sf, g).reshape(32, 16, 16)
    vb = v.astype(np.float64).reshape(32, 16, 16)
    A = np.max(np.abs(vb), axis=2, keepdims=True)
    normal = (O.e4m3_decode(sf) >= 2.0 ** -6)[:, :, None]
    assert np.all((np.abs(vb - vh) <= 3 * A / 16 + 1e-12) | ~normal)


CHECKS = [check_signed_e4m3_matches_torch, check_signed_e4m3_saturates_and_keeps_sign,
          check_fp8_output_multiplies_by_g_d, check_fp32_values_quantizer_bruteforce,
          check_nvfp4_output_bound_and_amax]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_requant_pin(check):
    check()


# --------------------------------------------------------------------------
# Planted mistakes
# --------------------------------------------------------------------------
def _mut_divide_by_g_d(mp):
    real = O.e4m3_encode_signed_satfinite
    mp.setattr(O, "fp8_output", lambda v, g: real((np.asarray(v, np.float32) / np.float32(g)).astype(np.float32)))


def _mut_drop_sign(mp):
    mp.setattr(O, "e4m3_encode_signed_satfinite",
               lambda v: O.e4m3_encode_satfinite(np.abs(np.asarray(v, dtype=np.float32))))


def _mut_truncate(mp):
    def enc(v):
        v = np.asarray(v, dtype=np.float32)
        mag = np.clip(np.searchsorted(E4M3_POS, np.abs(v).astype(np.float64), side="right") - 1, 0, 126)
        return (mag.astype(np.uint8) | (np.signbit(v).astype(np.uint8) << 7)).astype(np.uint8)
    mp.setattr(O, "e4m3_encode_signed_satfinite", enc)


def _mut_ignore_g_d(mp):
    real = O.quantize_values_with_scale
    mp.setattr(O, "quantize_values_with_scale", lambda x, g: real(x, np.float32(1.0)))


def _mut_amax_scaled(mp):
    real = O.nvfp4_output
    def out(v, g):
        p, s, a = real(v, g)
        return p, s, np.float32(a * np.float32(g))
    mp.setattr(O, "nvfp4_output", out)


MUTATIONS = [_mut_divide_by_g_d, _mut_drop_sign, _mut_truncate, _mut_ignore_g_d, _mut_amax_scaled]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_planted_mistakes(mutate, monkeypatch):
    mutate(monkeypatch)
    caught = False
    for check in CHECKS:
        try:
            check()
        except AssertionError:
            caught = True
            break
    assert caught, f"no pin catches {mutate.__name__}"
