"""Hadamard-rotated quantize parity: the CUDA path against the CPU oracle.

"NVIDIA NVFP4 与 Micro-Scaling", section 4.1: x is rotated by an orthogonal
Walsh-Hadamard matrix before quantization.  Codes, scales, g and the amax of
the rotated tensor are compared bit for bit (the oracle fixes the fp32
order of the transform); a GEMM of two rotated operands is checked against
the oracle's GEMM of its own rotated operands within 2^-20 * alpha * S.
"""
import numpy as np
import pytest
import torch

import oracle_pool
from oracle import hadamard_oracle as H
from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import check_bf16, check_f32, dev_bf16, f32_scalar, host_bf16_bits, host_u8

pytestmark = pytest.mark.gpu

ORDERS = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512]


def _both(nv, x_bits, order, layout, amax=None):
    xd = dev_bf16(x_bits)
    amax_t = None if amax is None else torch.tensor([amax], dtype=torch.float32, device="cuda")
    q = nv.quantize_hadamard(xd, order, layout, amax=amax_t)
    torch.cuda.synchronize()
    assert nv.nvfp4_check_device_status() == nv.OK
    return q, H.quantize_hadamard(x_bits, order, amax_value=amax)


def _assert_same(nv, q, ref, layout):
    codes_ref, sf_ref, g_ref, amax_ref = ref
    assert f32_scalar(q.amax).tobytes() == np.float32(amax_ref).tobytes(), (f32_scalar(q.amax), amax_ref)
    assert f32_scalar(q.g).tobytes() == np.float32(g_ref).tobytes()
    codes = host_u8(q.codes)
    bad = np.argwhere(codes != codes_ref)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:3].tolist()}"
    sf = host_u8(q.sf)
    want = sf_ref.reshape(-1) if layout == nv.SF_ROWMAJOR else O.swizzle_sf_tcgen05(sf_ref)
    bad = np.nonzero(sf != want)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:5].tolist()}"


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("rows,k", [(200, 1536), (3, 12288)])
@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_hadamard_quantize_matches_oracle(lib, order, rows, k, layout):
    """Several tiles, a ragged row tail (200 = 128 + 72) and a ragged second
    segment of 512 blocks (12288 / 16 = 768)."""
    x = inputs.activations_with_outliers(rows, k, seed=300 + order, fraction=0.01, factor=50.0)
    q, ref = _both(lib, x, order, layout)
    _assert_same(lib, q, ref, layout)


@pytest.mark.parametrize("order", [16, 32, 128])
def test_hadamard_quantize_odd_pitch_and_small_k(lib, order):
    """Rows whose pitch is off the 32-B grid take the 128-bit load path."""
    rows, k, ld = 37, 512, 520
    x = inputs.gaussian_bf16((rows, k), seed=71)
    pitched = np.zeros((rows, ld), dtype=np.uint16)
    pitched[:, :k] = x
    q = lib.quantize_hadamard(dev_bf16(pitched)[:, :k], order, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    _assert_same(lib, q, H.quantize_hadamard(x, order), lib.SF_TCGEN05)


def test_order_one_equals_plain_quantizer(lib):
    x = inputs.activations_with_outliers(130, 2048, seed=81, fraction=0.01, factor=50.0)
    xd = dev_bf16(x)
    a = lib.quantize_hadamard(xd, 1, lib.SF_TCGEN05)
    b = lib.quantize(xd, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and torch.equal(a.sf, b.sf)
    assert torch.equal(a.g, b.g) and torch.equal(a.amax, b.amax)


def test_given_amax(lib):
    x = inputs.gaussian_bf16((64, 1024), seed=91)
    amax = float(H.quantize_hadamard(x, 64)[3]) / 3
    q, ref = _both(lib, x, 64, lib.SF_ROWMAJOR, amax=amax)
    _assert_same(lib, q, ref, lib.SF_ROWMAJOR)
    assert np.any(ref[1] == 0x7E)


def test_all_zero_and_nonfinite(lib):
    z = np.zeros((8, 256), dtype=np.uint16)
    q, ref = _both(lib, z, 32, lib.SF_TCGEN05)
    _assert_same(lib, q, ref, lib.SF_TCGEN05)
    assert f32_scalar(q.g) == np.float32(1.0)
    x = inputs.gaussian_bf16((16, 256), seed=93).copy()
    x[5, 40] = 0x7F80                                   # +inf spreads over its 128-element segment
    q = lib.quantize_hadamard(dev_bf16(x), 128, lib.SF_TCGEN05)
    assert lib.nvfp4_check_device_status() == lib.ERR_RANGE
    assert f32_scalar(q.g) == 0.0 and not host_u8(q.codes).any()


@pytest.mark.parametrize("order", [16, 128])
def test_rotated_gemm_matches_oracle(lib, order):
    """Both operands rotated with the same order: the GEMM of the rotated
    codes against the oracle's GEMM of its rotated codes (fp32 bound and
    bf16 rule), and the product stays close to x W^T."""
    m, n, k = 200, 272, 1024
    a = inputs.activations_with_outliers(m, k, seed=400, fraction=0.01, factor=30.0)
    w = inputs.gaussian_bf16((n, k), seed=401, std=0.02)
    qa = lib.quantize_hadamard(dev_bf16(a), order, lib.SF_TCGEN05)
    qw = lib.quantize_hadamard(dev_bf16(w), order, lib.SF_TCGEN05)
    d32 = lib.gemm(qa, qw, out_dtype=torch.float32)
    d16 = lib.gemm(qa, qw)
    torch.cuda.synchronize()
    pa, sa, ga, _ = H.quantize_hadamard(a, order)
    pw, sw, gw, _ = H.quantize_hadamard(w, order)
    d_ref, s_ref, alpha = O.gemm_ref(pa, sa, ga, pw, sw, gw)
    check_f32(d32.cpu().numpy(), d_ref, s_ref, alpha)
    check_bf16(host_bf16_bits(d16), d_ref, s_ref, alpha)
    exact = O.bf16_to_f32(a).astype(np.float64) @ O.bf16_to_f32(w).astype(np.float64).T
    rel = np.linalg.norm(d32.cpu().numpy() - exact) / np.linalg.norm(exact)
    assert rel < 0.15, rel


@pytest.mark.parametrize("order", [16, 128])
def test_full_size_every_byte(lib, order):
    """Quantize-bandwidth workload [16384, 8192] with 1% outlier channels:
    the amax of y and g exact, every code byte and scale equal to the
    oracle's (run over the host cores by rows)."""
    x = inputs.quantize_bandwidth()
    q = lib.quantize_hadamard(dev_bf16(x), order, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    codes_ref, sf_ref, g, amax = oracle_pool.quantize_hadamard(x, order)
    assert f32_scalar(q.amax) == amax and f32_scalar(q.g) == g
    assert np.array_equal(host_u8(q.codes), codes_ref)
    assert np.array_equal(O.unswizzle_sf_tcgen05(host_u8(q.sf), *x.shape), sf_ref)


@pytest.mark.parametrize("order", [1, 16, 32, 128, 512])
@pytest.mark.parametrize("rows,k", [(200, 1536), (3, 12288)])
@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_rotated_stochastic_matches_oracle(lib, order, rows, k, layout):
    """Rotation then stochastic rounding, bit-exact: the Philox bits of each
    position in y are drawn identically on both sides."""
    x = inputs.activations_with_outliers(rows, k, seed=700 + order, fraction=0.01, factor=50.0)
    seed, offset = 0xABCDEF0123456789, 77 + order
    q = lib.quantize_hadamard_stochastic(dev_bf16(x), order, seed, offset, layout)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    _assert_same(lib, q, H.quantize_hadamard_sr(x, order, seed, offset), layout)


@pytest.mark.parametrize("order", [16, 128])
def test_rotated_stochastic_full_size_every_byte(lib, order):
    """The same workload rotated then rounded stochastically (order 128 takes
    the two-adjacent-blocks kernels): every byte equal to the oracle's."""
    x = inputs.quantize_bandwidth()
    q = lib.quantize_hadamard_stochastic(dev_bf16(x), order, 42, 1, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    codes_ref, sf_ref, g, amax = oracle_pool.quantize_hadamard_sr(x, order, 42, 1)
    assert f32_scalar(q.amax) == amax and f32_scalar(q.g) == g
    assert np.array_equal(host_u8(q.codes), codes_ref)
    assert np.array_equal(O.unswizzle_sf_tcgen05(host_u8(q.sf), *x.shape), sf_ref)
