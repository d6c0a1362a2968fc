"""Degenerate and extreme inputs on the GPU, against the oracle.

Empty tensors (the amax of nothing is 0, so g = 1), a one-column weight
matrix for the GEMV, and bf16 values at both ends of the format in one tensor.
"""
import numpy as np
import pytest
import torch

from oracle import hadamard_oracle as H
from oracle import nvfp4_oracle as O
from oracle import stochastic_oracle as S
from nvfp4_block_scaled_15_b200 import inputs
from parity import check_bf16, dev_bf16, f32_scalar, host_bf16_bits, host_u8

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,k", [(0, 256), (5, 0), (0, 0)], ids=lambda v: str(v))
@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_empty_tensors(lib, rows, k, layout):
    x = torch.empty((rows, k), dtype=torch.bfloat16, device="cuda")
    _, _, g_ref, a_ref = O.quantize(np.zeros((rows, k), dtype=np.uint16))
    assert g_ref == np.float32(1.0) and a_ref == 0
    for q in (lib.quantize(x, layout), lib.quantize_hadamard(x, 16, layout),
              lib.quantize_stochastic(x, 1, 2, layout), lib.quantize_hadamard_stochastic(x, 16, 1, 2, layout)):
        torch.cuda.synchronize()
        assert lib.nvfp4_check_device_status() == lib.OK
        assert f32_scalar(q.g) == 1.0 and f32_scalar(q.amax) == 0.0
        assert q.codes.numel() == 0
    if k % 32 == 0:
        lib.mxfp4_quantize(x, layout)
        assert lib.nvfp4_check_device_status() == lib.OK
    out = torch.full((1,), 7.0, dtype=torch.float32, device="cuda")
    lib.nvfp4_amax(x, rows, k, max(k, 8), out)
    assert f32_scalar(out) == 0.0


@pytest.mark.parametrize("m,k", [(1, 64), (32, 8192)], ids=lambda v: str(v))
def test_gemv_single_output_column(lib, m, k):
    x = inputs.gaussian_bf16((m, k), seed=600 + m)
    w = inputs.gaussian_bf16((1, k), seed=601, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    y = lib.gemv_batched(dev_bf16(x), qw)
    assert lib.nvfp4_check_device_status() == lib.OK
    px, sx, gx, _ = O.quantize(x)
    pw, sw, gw, _ = O.quantize(w)
    d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, pw, sw, gw)
    check_bf16(host_bf16_bits(y), d_ref, s_ref, alpha)


def _extremes():
    """The largest finite bf16 (0x7F7F, about 3.39e38, so g = 2688/amax is about
    7.9e-36), the smallest subnormal (0x0001), negative zero, and normal values
    in between; blocks far below the amax get zero scales and zero codes."""
    x = inputs.gaussian_bf16((4, 256), seed=77).copy()
    x[0, 3] = 0x7F7F
    x[0, 20] = 0xFF7F
    x[1, 0:16] = 0x0001
    x[1, 16:32] = 0x8000
    x[2, 100] = 0x7F00
    return x


@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_bf16_extremes(lib, layout):
    x = _extremes()
    xd = dev_bf16(x)
    q = lib.quantize(xd, layout)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    codes_ref, sf_ref, g_ref, a_ref = O.quantize(x)
    assert f32_scalar(q.g) == g_ref and f32_scalar(q.amax) == a_ref
    assert np.array_equal(host_u8(q.codes), codes_ref)
    want = sf_ref.reshape(-1) if layout == lib.SF_ROWMAJOR else O.swizzle_sf_tcgen05(sf_ref)
    assert np.array_equal(host_u8(q.sf), want)
    qs = lib.quantize_stochastic(xd, 3, 4, layout)
    torch.cuda.synchronize()
    codes_s, sf_s, _, _ = S.quantize_sr(x, 3, 4)
    assert np.array_equal(host_u8(qs.codes), codes_s)
    qh = lib.quantize_hadamard(xd, 16, layout)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK       # |y| <= 2 * 3.39e38 / 4: still finite
    codes_h, sf_h, g_h, a_h = H.quantize_hadamard(x, 16)
    assert f32_scalar(qh.amax) == a_h and np.array_equal(host_u8(qh.codes), codes_h)
