"""MXFP4 parity: the CUDA quantizer (and GEMM) against the CPU oracle.

MXFP4 is the format the pages set against NVFP4 ("mxFP4/nvFP4 最小化知识" (一);
"low-precision-floats", FP4 / MXFP4 / NVFP4): one E8M0 scale per 32 elements,
rounded up to a power of two, no global scale.
"""
import numpy as np
import pytest
import torch

import oracle_pool
from oracle import mxfp4_oracle as MX
from oracle import nvfp4_oracle as NV
from nvfp4_block_scaled_15_b200 import inputs
from parity import check_bf16, check_f32, dev_bf16, host_bf16_bits, host_u8

pytestmark = pytest.mark.gpu


def _quantize_both(lib, x_bits, layout):
    q = lib.mxfp4_quantize(dev_bf16(x_bits), layout)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    packed, sf = MX.quantize_mx(x_bits)
    want_sf = sf.reshape(-1) if layout == lib.SF_ROWMAJOR else NV.swizzle_sf_tcgen05(sf)
    codes = host_u8(q.codes)
    bad = np.argwhere(codes != packed)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:3].tolist()}"
    got_sf = host_u8(q.sf)
    assert got_sf.size == want_sf.size
    bad = np.nonzero(got_sf != want_sf)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:5].tolist()}"


SHAPES = [(128, 256), (200, 384), (1, 128), (3, 8192), (129, 1024), (130, 28672)]


@pytest.mark.parametrize("rows,k", SHAPES, ids=lambda v: str(v))
@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_mx_quantize_matches_oracle(lib, rows, k, layout):
    x = inputs.activations_with_outliers(rows, k, seed=700 + rows, fraction=0.01, factor=50.0)
    _quantize_both(lib, x, layout)


@pytest.mark.parametrize("rows,k", [(5, 32), (7, 96), (2, 8224)], ids=lambda v: str(v))
def test_mx_quantize_rowmajor_k_multiple_of_32(lib, rows, k):
    _quantize_both(lib, inputs.gaussian_bf16((rows, k), seed=31 + k), lib.SF_ROWMAJOR)


def test_mx_quantize_extreme_blocks(lib):
    """All-zero blocks (scale byte 0), -0, bf16 subnormals, values near the
    bf16 maximum, blocks whose A/6 is a power of two exactly."""
    rng = np.random.default_rng(3)
    x = rng.normal(size=(16, 256))
    x[0, :32] = 0.0
    x[1, :32] = -0.0
    x[2, :32] *= 1e-39                     # bf16 subnormals
    x[3, :32] = rng.normal(size=32) * 1e37
    x[4, :32] = 1.5
    x[4, 7] = 6.0 * 2 ** -20               # A / 6 = 2^-20
    x[5, :32] = 1e-30
    bits = inputs.f64_to_bf16_bits(x)
    bits[1, :32] = 0x8000                  # exact -0
    _quantize_both(lib, bits, lib.SF_TCGEN05)
    _quantize_both(lib, bits, lib.SF_ROWMAJOR)


def test_mx_quantize_nonfinite_block_reports_range(lib):
    x = inputs.gaussian_bf16((4, 128), seed=8).copy()
    x[2, 40] = 0x7F80                      # +inf in block 1 of row 2
    q = lib.mxfp4_quantize(dev_bf16(x), lib.SF_ROWMAJOR)
    assert lib.nvfp4_check_device_status() == lib.ERR_RANGE
    sf = host_u8(q.sf).reshape(4, 4)
    assert sf[2, 1] == 0xFF
    assert not host_u8(q.codes)[2, 16:32].any()             # elements 32..63 = bytes 16..31
    clean = x.copy()
    clean[2, 32:64] = 0
    _, want = MX.quantize_mx(clean)
    mask = np.ones_like(sf, dtype=bool)
    mask[2, 1] = False
    assert np.array_equal(sf[mask], want[mask])


# --------------------------------------------------------------------------
# MXFP4 block-scaled GEMM (tcgen05.mma kind::mxf4, E8M0 scales, no alpha)
# --------------------------------------------------------------------------

def _mx_gemm_case(lib, a_bits, b_bits, out_dtype):
    qa = lib.mxfp4_quantize(dev_bf16(a_bits), lib.SF_TCGEN05)
    qb = lib.mxfp4_quantize(dev_bf16(b_bits), lib.SF_TCGEN05)
    d = lib.mxfp4_gemm(qa, qb, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    pa, sa = MX.quantize_mx(a_bits)
    pb, sb = MX.quantize_mx(b_bits)
    assert np.array_equal(host_u8(qa.codes), pa) and np.array_equal(host_u8(qb.codes), pb)
    d_ref, s_ref = MX.gemm_ref_mx(pa, sa, pb, sb)
    return d, d_ref, s_ref


MX_SHAPES = [
    (1, 1, 128),          # one element, one scale atom
    (200, 136, 384),      # M and N tails, a last K stage with one 128-wide atom
    (129, 257, 512),      # tails past one tile in both directions
    (300, 100, 1152),     # N <= 128 kernel, odd atom count
    (128, 384, 2048),     # M <= 128 kernel (256-wide N tiles + a tail)
    (64, 512, 8192),      # long K
    (300, 520, 384),      # CTA-pair kernel: odd 128-row groups, half stage at the end
    (1000, 700, 1024),    # CTA-pair kernel: tails, several tiles
    (2048, 2560, 256),    # more tiles than SMs
]


@pytest.mark.parametrize("m,n,k", MX_SHAPES, ids=lambda v: str(v))
def test_mx_gemm_matches_oracle(lib, m, n, k):
    a = inputs.activations_with_outliers(m, k, seed=m + 3 * k, fraction=0.01, factor=30.0)
    b = inputs.gaussian_bf16((n, k), seed=n + 5 * k, std=0.02)
    d32, d_ref, s_ref = _mx_gemm_case(lib, a, b, torch.float32)
    check_f32(d32.cpu().numpy(), d_ref, s_ref, 1.0)
    d16, _, _ = _mx_gemm_case(lib, a, b, torch.bfloat16)
    check_bf16(host_bf16_bits(d16), d_ref, s_ref, 1.0)


def test_mx_gemm_output_pitch(lib):
    m, n, k = 130, 136, 256
    a = inputs.gaussian_bf16((m, k), seed=191)
    b = inputs.gaussian_bf16((n, k), seed=192)
    qa = lib.mxfp4_quantize(dev_bf16(a), lib.SF_TCGEN05)
    qb = lib.mxfp4_quantize(dev_bf16(b), lib.SF_TCGEN05)
    big = torch.full((m + 40, 288), -7.0, dtype=torch.bfloat16, device="cuda")
    lib.nvfp4_mxfp4_gemm(qa.codes, qa.sf, qb.codes, qb.sf, m, n, k, big, 288, lib.OUT_BF16)
    torch.cuda.synchronize()
    pa, sa = MX.quantize_mx(a)
    pb, sb = MX.quantize_mx(b)
    d_ref, s_ref = MX.gemm_ref_mx(pa, sa, pb, sb)
    check_bf16(host_bf16_bits(big[:m, :n]), d_ref, s_ref, 1.0)
    assert torch.all(big[:m, n:] == -7.0) and torch.all(big[m:, :] == -7.0)


def _mx_probe(lib, m, n, k, sa, sb):
    """All-ones codes (E2M1 1.0 = code 2) with the given row-major E8M0 scales."""
    codes_a = torch.full((m, k // 2), 0x22, dtype=torch.uint8, device="cuda")
    codes_b = torch.full((n, k // 2), 0x22, dtype=torch.uint8, device="cuda")
    sfa = torch.from_numpy(NV.swizzle_sf_tcgen05(sa)).cuda()
    sfb = torch.from_numpy(NV.swizzle_sf_tcgen05(sb)).cuda()
    assert sfa.numel() == MX.sf_tcgen05_bytes_mx(m, k) == lib.nvfp4_mxfp4_sf_bytes(m, k, lib.SF_TCGEN05)
    d = torch.empty((m, n), dtype=torch.float32, device="cuda")
    lib.nvfp4_mxfp4_gemm(codes_a, sfa, codes_b, sfb, m, n, k, d, n, lib.OUT_F32)
    torch.cuda.synchronize()
    return d.cpu().numpy()


@pytest.mark.parametrize("m,n", [(256, 256), (128, 256), (256, 128)], ids=["cta_pair", "m128", "n128"])
@pytest.mark.parametrize("side", ["a", "b"])
def test_mx_scale_layout_probes(lib, side, m, n):
    """Exactly one (row, block) E8M0 scale is 2.0 (byte 128), all others 1.0
    (byte 127): only that row (A side) or column (B side) of D grows, by exactly
    32 (one block of 32 products 1 x 1).  Pins the 32-element scale blocks and
    their placement in the tensor-core layout, for each of the three kernels."""
    k = 640                        # 20 scales per row: 5 atoms, the last stage half full
    kb = k // 32
    limit = m if side == "a" else n
    for row, blk in [(0, 0), (37, 5), (77, 18), (100, 19), (161, 9), (255, 13), (127, 1)]:
        if row >= limit:
            continue
        sa = np.full((m, kb), 127, np.uint8)
        sb = np.full((n, kb), 127, np.uint8)
        (sa if side == "a" else sb)[row, blk] = 128
        d = _mx_probe(lib, m, n, k, sa, sb)
        want = np.full((m, n), float(k))
        if side == "a":
            want[row, :] += 32.0
        else:
            want[:, row] += 32.0
        assert np.array_equal(d, want), (side, row, blk, np.argwhere(d != want)[:4].tolist())


def test_mx_gemm_full_size(lib):
    """8192^3 with the prefill inputs in MXFP4: every code byte and scale of
    both operands bit-exact in both layouts, and every one of the 67,108,864
    bf16 outputs against the oracle (1 ulp, or the carried bound)."""
    a, w = inputs.prefill_gemm()
    qa = lib.mxfp4_quantize(dev_bf16(a), lib.SF_ROWMAJOR)
    qw = lib.mxfp4_quantize(dev_bf16(w), lib.SF_ROWMAJOR)
    ta = lib.mxfp4_quantize(dev_bf16(a), lib.SF_TCGEN05)
    tw = lib.mxfp4_quantize(dev_bf16(w), lib.SF_TCGEN05)
    d = lib.mxfp4_gemm(ta, tw, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    pa, sa = oracle_pool.quantize_mx(a)
    pw, sw = oracle_pool.quantize_mx(w)
    for q, t, p_ref, s_ref in ((qa, ta, pa, sa), (qw, tw, pw, sw)):
        assert np.array_equal(host_u8(q.codes), p_ref) and np.array_equal(host_u8(t.codes), p_ref)
        assert np.array_equal(host_u8(q.sf).reshape(8192, -1), s_ref)
        assert np.array_equal(host_u8(t.sf).reshape(-1), NV.swizzle_sf_tcgen05(s_ref))
    d_ref, s_ref = oracle_pool.gemm_ref_mx(pa, sa, pw, sw)
    check_bf16(host_bf16_bits(d), d_ref, s_ref, 1.0)


def test_mx_gemm_rejects_bad_arguments(lib):
    q = lib.mxfp4_quantize(dev_bf16(inputs.gaussian_bf16((128, 256), seed=1)), lib.SF_TCGEN05)
    d = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    c, sf = q.codes, q.sf
    for args, want in [((c, sf, c, sf, 128, 128, 192, d, 128), lib.ERR_UNSUPPORTED_SHAPE),   # K % 128 != 0
                       ((c, sf, c, sf, 128, 128, 256, d, 64), lib.ERR_INVALID_ARG),          # ldd < N
                       ((c[:, 8:], sf, c, sf, 128, 128, 256, d, 128), lib.ERR_MISALIGNED)]:  # codes + 8 B
        with pytest.raises(lib.NVFP4Error) as e:
            lib.nvfp4_mxfp4_gemm(*args, lib.OUT_BF16)
        assert e.value.status == want
