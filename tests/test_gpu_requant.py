"""GEMM outputs under the output scale g_d: FP8 (E4M3) bytes and NVFP4
(codes + block scales) written by the GEMM epilogue, against the oracle.

"NVIDIA NVFP4 与 Micro-Scaling", section 三: D = g_d * (...), the output
landing as FP8 (its _scaled_mm example: scale_result=g_d, float8_e4m3fn).

Two kinds of checks:
  * exact accumulation: codes in 0..15 and block scales in {0.5, 1, 2} with
    g_a = g_b = 1 make every partial sum a multiple of 1/16 below 2^20, so
    the fp32 accumulator holds D exactly whatever the summation order, and
    the quantized outputs must equal the oracle's bit for bit;
  * realistic data: the fp32 value v is known only within 2^-20 alpha S, so
    each output byte must lie between the oracle's outputs at the two ends of
    that interval (all quantizers here are monotone); almost all are unique.
"""
import numpy as np
import pytest
import torch

import oracle_pool
from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import BOUND, dev_bf16, host_u8

pytestmark = pytest.mark.gpu


def _exact_operands(rng, rows, k):
    codes = rng.integers(0, 16, (rows, k), dtype=np.uint8)
    sf = rng.choice(np.uint8([0x30, 0x38, 0x40]), (rows, k // 16))
    return O.pack_codes(codes), sf


def _dev_operand(packed, sf):
    return torch.from_numpy(packed).cuda(), torch.from_numpy(O.swizzle_sf_tcgen05(sf)).cuda()


def _f32_dev(x):
    return torch.tensor([float(np.float32(x))], dtype=torch.float32, device="cuda")


def _exact_case(m, n, k, seed):
    rng = np.random.default_rng(seed)
    pa, sa = _exact_operands(rng, m, k)
    pb, sb = _exact_operands(rng, n, k)
    d, _, alpha = O.gemm_ref(pa, sa, np.float32(1), pb, sb, np.float32(1))
    v = d.astype(np.float32)
    assert alpha == 1 and np.array_equal(v.astype(np.float64), d)      # exactly representable
    return pa, sa, pb, sb, v


def _e4m3_ordinal(b):
    b = np.asarray(b, dtype=np.int64)
    return np.where(b & 0x80, -(b & 0x7F), b & 0x7F)


def _e2m1_ordinal(c):
    c = np.asarray(c, dtype=np.int64)
    return np.where(c & 8, -(c & 7), c & 7)


EXACT_SHAPES = [
    (256, 256, 512),     # CTA-pair kernel
    (128, 384, 256),     # one-CTA kernel, 256-wide N tiles
    (300, 128, 512),     # one-CTA kernel, N <= 128
    (130, 320, 256),     # CTA-pair kernel, M tail, N tail in a 256 tile
    (77, 64, 1024),      # one small tile
]


@pytest.mark.parametrize("m,n,k", EXACT_SHAPES, ids=lambda v: str(v))
@pytest.mark.parametrize("layout", [0, 1], ids=["sf_rowmajor", "sf_tcgen05"])
def test_requant_exact(lib, m, n, k, layout):
    pa, sa, pb, sb, v = _exact_case(m, n, k, seed=m * 7 + n + k)
    g_d = np.float32(2688.0) / np.float32(np.max(np.abs(v)))
    a_codes, a_sf = _dev_operand(pa, sa)
    b_codes, b_sf = _dev_operand(pb, sb)
    one = _f32_dev(1.0)
    pitch = n // 2 + 48                                    # wider rows: nothing past N/2 may change
    codes = torch.full((m, pitch), 0xA5, dtype=torch.uint8, device="cuda")
    sf = torch.full((lib.nvfp4_sf_bytes(m, n, layout),), 0xA5, dtype=torch.uint8, device="cuda")
    amax = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    lib.nvfp4_gemm_requant(a_codes, a_sf, one, b_codes, b_sf, one, m, n, k, _f32_dev(g_d), codes, pitch, sf,
                           layout, amax)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    want_codes, want_sf, want_amax = O.nvfp4_output(v, g_d)
    got = host_u8(codes)
    assert np.array_equal(got[:, : n // 2], want_codes), np.argwhere(got[:, : n // 2] != want_codes)[:4].tolist()
    assert np.all(got[:, n // 2:] == 0xA5)
    got_sf = host_u8(sf)
    got_sf = got_sf.reshape(m, n // 16) if layout == 0 else O.unswizzle_sf_tcgen05(got_sf, m, n)
    assert np.array_equal(got_sf, want_sf), np.argwhere(got_sf != want_sf)[:4].tolist()
    assert np.float32(amax.item()) == want_amax


@pytest.mark.parametrize("m,n,k", EXACT_SHAPES + [(140, 200, 256), (3, 13, 512)], ids=lambda v: str(v))
@pytest.mark.parametrize("g_d", [4.0, 0.37], ids=["g4", "g0.37"])
def test_fp8_out_exact(lib, m, n, k, g_d):
    """FP8 output bytes for the page's example g_d = 4.0 and an arbitrary one;
    N = 200 and 13 leave partial 16-column blocks."""
    pa, sa, pb, sb, v = _exact_case(m, n, k, seed=m + 3 * n + k)
    a_codes, a_sf = _dev_operand(pa, sa)
    b_codes, b_sf = _dev_operand(pb, sb)
    one = _f32_dev(1.0)
    pitch = (n + 15) // 16 * 16 + 32
    d = torch.full((m + 3, pitch), 0x5A, dtype=torch.uint8, device="cuda")
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    lib.nvfp4_gemm_fp8_out(a_codes, a_sf, one, b_codes, b_sf, one, m, n, k, _f32_dev(g_d), d, pitch, amax)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    got = host_u8(d)
    want = O.fp8_output(v, np.float32(g_d))
    assert np.array_equal(got[:m, :n], want), np.argwhere(got[:m, :n] != want)[:4].tolist()
    assert np.all(got[:m, n:] == 0x5A) and np.all(got[m:] == 0x5A)
    assert np.float32(amax.item()) == np.float32(np.max(np.abs(v)))


def test_requant_chain_feeds_next_gemm(lib):
    """Layer 1 writes NVFP4 (tensor-core scales) that layer 2 consumes as its A
    operand directly; layer 2's output against the oracle chain."""
    m, n1, k = 256, 512, 512
    pa, sa, pb, sb, v = _exact_case(m, n1, k, seed=5)
    g_d = np.float32(2688.0) / np.float32(np.max(np.abs(v)))
    a_codes, a_sf = _dev_operand(pa, sa)
    b_codes, b_sf = _dev_operand(pb, sb)
    one = _f32_dev(1.0)
    h = lib.empty_quantized(m, n1, lib.SF_TCGEN05, "cuda")
    h.g.copy_(_f32_dev(g_d))
    lib.nvfp4_gemm_requant(a_codes, a_sf, one, b_codes, b_sf, one, m, n1, k, h.g, h.codes, n1 // 2, h.sf,
                           lib.SF_TCGEN05, h.amax)
    w2 = inputs.gaussian_bf16((384, n1), seed=77, std=0.02)
    q2 = lib.quantize(dev_bf16(w2), lib.SF_TCGEN05)
    d2 = lib.gemm(h, q2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    hp, hs, _ = O.nvfp4_output(v, g_d)
    p2, s2, g2, _ = O.quantize(w2)
    d_ref, s_ref, alpha = O.gemm_ref(hp, hs, g_d, p2, s2, g2)
    err = np.abs(d2.cpu().numpy().astype(np.float64) - d_ref)
    assert np.all(err <= BOUND * np.float64(alpha) * s_ref)


def _admissible_nvfp4(d_ref, s_ref, alpha, g_d, got_codes, got_sf):
    """Each block scale lies between the scales of the block amax's interval
    ends; each code, for the scale the GPU chose, between the codes of the
    element's interval ends.  Returns the fraction of elements whose code is
    unique over the interval."""
    e = BOUND * np.float64(alpha) * s_ref          # d_ref already holds alpha; s_ref does not
    c = d_ref
    lo = np.nextafter((c - e).astype(np.float32), np.float32(-np.inf))
    hi = np.nextafter((c + e).astype(np.float32), np.float32(np.inf))
    rows, n = c.shape
    mag_lo = np.where((lo <= 0) & (hi >= 0), np.float32(0), np.minimum(np.abs(lo), np.abs(hi)))
    mag_hi = np.maximum(np.abs(lo), np.abs(hi))
    ab_lo = mag_lo.reshape(rows, n // 16, 16).max(axis=2)
    ab_hi = mag_hi.reshape(rows, n // 16, 16).max(axis=2)
    g = np.float32(g_d)

    def scale(ab):
        return O.e4m3_encode_satfinite(((ab * g).astype(np.float32) / np.float32(6.0)).astype(np.float32))

    s_lo, s_hi = scale(ab_lo), scale(ab_hi)
    assert np.all((got_sf >= s_lo) & (got_sf <= s_hi)), "block scale outside its admissible range"
    sd = np.repeat(O.e4m3_decode(got_sf).astype(np.float32), 16, axis=1)

    def codes(x):
        t = (x * g).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            u = np.where(sd == 0, np.float32(0), t / np.where(sd == 0, np.float32(1), sd)).astype(np.float32)
        return np.where(sd == 0, 0, _e2m1_ordinal(O.e2m1_encode(u)))

    o_lo, o_hi = codes(lo), codes(hi)
    got = _e2m1_ordinal(O.unpack_codes(got_codes))
    assert np.all((got >= o_lo) & (got <= o_hi)), "code outside its admissible range"
    return float(np.mean(o_lo == o_hi))


@pytest.mark.parametrize("m,n,k", [(1000, 1024, 2048), (200, 256, 8192), (96, 128, 1024)], ids=lambda v: str(v))
def test_requant_realistic_admissible(lib, m, n, k):
    a = inputs.activations_with_outliers(m, k, seed=m + k, fraction=0.01, factor=30.0)
    b = inputs.gaussian_bf16((n, k), seed=n + k, std=0.02)
    qa = lib.quantize(dev_bf16(a), lib.SF_TCGEN05)
    qb = lib.quantize(dev_bf16(b), lib.SF_TCGEN05)
    pa, sa, ga, _ = O.quantize(a)
    pb, sb, gb, _ = O.quantize(b)
    d_ref, s_ref, alpha = O.gemm_ref(pa, sa, ga, pb, sb, gb)
    g_d = np.float32(2688.0) / np.float32(np.max(np.abs(d_ref)))
    out = lib.gemm_requant(qa, qb, _f32_dev(g_d), layout=lib.SF_ROWMAJOR)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    uniq = _admissible_nvfp4(d_ref, s_ref, alpha, g_d, host_u8(out.codes), host_u8(out.sf).reshape(m, n // 16))
    assert uniq > 0.99, uniq
    amax = np.float64(out.amax.item())
    e = BOUND * np.float64(alpha) * s_ref
    c = np.abs(d_ref)
    assert np.max(c - e) * (1 - 2.0 ** -23) <= amax <= np.max(c + e) * (1 + 2.0 ** -23)
    d8 = lib.gemm_fp8_out(qa, qb, _f32_dev(4.0))
    torch.cuda.synchronize()
    got8 = _e4m3_ordinal(host_u8(d8.view(torch.uint8)))
    lo = np.nextafter((d_ref - e).astype(np.float32), np.float32(-np.inf))
    hi = np.nextafter((d_ref + e).astype(np.float32), np.float32(np.inf))
    o_lo = _e4m3_ordinal(O.fp8_output(lo, np.float32(4.0)))
    o_hi = _e4m3_ordinal(O.fp8_output(hi, np.float32(4.0)))
    assert np.all((got8 >= o_lo) & (got8 <= o_hi))
    assert np.mean(o_lo == o_hi) > 0.99


def test_requant_full_size(lib):
    """Prefill workload 8192^3 with an NVFP4 output: every one of the 4,194,304
    16-column blocks (scale and 16 codes) inside its admissible range, most
    codes unique over it, and amax_d between the interval ends' maxima."""
    a, w = inputs.prefill_gemm()
    qa = lib.quantize(dev_bf16(a), lib.SF_TCGEN05)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    g_d = np.float32(2688.0 / 40.0)
    out = lib.gemm_requant(qa, qw, _f32_dev(g_d), layout=lib.SF_ROWMAJOR)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    amax = out.amax.item()
    codes = host_u8(out.codes)
    sf = host_u8(out.sf).reshape(8192, 512)
    pa, sa, ga, _ = oracle_pool.quantize(a)
    pw, sw, gw, _ = oracle_pool.quantize(w)
    d_ref, s_ref, alpha = oracle_pool.gemm_ref(pa, sa, ga, pw, sw, gw)
    e = BOUND * np.float64(alpha) * s_ref
    c = np.abs(d_ref)
    assert np.max(c - e) * (1 - 2.0 ** -23) <= amax <= np.max(c + e) * (1 + 2.0 ** -23)
    del c, e
    unique = []
    for r0 in range(0, 8192, 1024):
        r1 = r0 + 1024
        unique.append(_admissible_nvfp4(d_ref[r0:r1], s_ref[r0:r1], alpha, g_d, codes[r0:r1], sf[r0:r1]))
    assert np.mean(unique) > 0.99


def test_requant_rejects_bad_arguments(lib):
    q = lib.quantize(dev_bf16(inputs.gaussian_bf16((128, 256), seed=2)), lib.SF_TCGEN05)
    g = _f32_dev(1.0)
    codes = torch.empty((128, 128), dtype=torch.uint8, device="cuda")
    sf = torch.empty(lib.nvfp4_sf_bytes(128, 256, lib.SF_TCGEN05), dtype=torch.uint8, device="cuda")
    base = (q.codes, q.sf, q.g, q.codes, q.sf, q.g)
    for n, ldd, layout, want in [(120, 64, 0, lib.ERR_UNSUPPORTED_SHAPE),    # N % 16 != 0
                                 (96, 48, 1, lib.ERR_UNSUPPORTED_SHAPE),     # tensor-core layout needs N % 64
                                 (128, 32, 0, lib.ERR_INVALID_ARG),          # pitch below N/2
                                 (128, 72, 0, lib.ERR_MISALIGNED)]:          # pitch not a multiple of 16
        with pytest.raises(lib.NVFP4Error) as e:
            lib.nvfp4_gemm_requant(*base, 128, n, 256, g, codes, ldd, sf, layout)
        assert e.value.status == want
    with pytest.raises(lib.NVFP4Error) as e:
        lib.nvfp4_gemm_fp8_out(*base, 128, 128, 256, None, codes, 128)
    assert e.value.status == lib.ERR_INVALID_ARG
