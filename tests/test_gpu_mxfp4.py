"""MXFP4 parity: the CUDA quantizer (and GEMM) against the CPU oracle.

MXFP4 is the format the pages set against NVFP4 ("mxFP4/nvFP4 最小化知识" (一);
"low-precision-floats", FP4 / MXFP4 / NVFP4): one E8M0 scale per 32 elements,
rounded up to a power of two, no global scale.
"""
import numpy as np
import pytest
import torch

from oracle import mxfp4_oracle as MX
from oracle import nvfp4_oracle as NV
from nvfp4_block_scaled_15_b200 import inputs
from parity import dev_bf16, host_u8

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
