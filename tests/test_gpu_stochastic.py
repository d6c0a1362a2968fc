"""Stochastic-rounding quantize parity: the CUDA path against the CPU oracle.

"FP4" encyclopedia entry, 技術原理: NVFP4 quantization rounds stochastically.
Both sides draw the same Philox4x32-10 bits (each from the published
definition), so codes, scales, g and amax are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle_pool
from oracle import nvfp4_oracle as O
from oracle import stochastic_oracle as S
from nvfp4_block_scaled_15_b200 import inputs
from parity import dev_bf16, f32_scalar, host_u8

pytestmark = pytest.mark.gpu

SEEDS = [(0, 0), (1234567, 42), (0xFEDCBA9876543210, 0xFFFFFFFF00000001)]


def _assert_same(nv, q, ref, layout):
    codes_ref, sf_ref, g_ref, amax_ref = ref
    assert f32_scalar(q.amax).tobytes() == np.float32(amax_ref).tobytes()
    assert f32_scalar(q.g).tobytes() == np.float32(g_ref).tobytes()
    codes = host_u8(q.codes)
    bad = np.argwhere(codes != codes_ref)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:3].tolist()}"
    sf = host_u8(q.sf)
    want = sf_ref.reshape(-1) if layout == nv.SF_ROWMAJOR else O.swizzle_sf_tcgen05(sf_ref)
    assert np.array_equal(sf, want)


@pytest.mark.parametrize("seed,offset", SEEDS)
@pytest.mark.parametrize("rows,k", [(200, 1536), (3, 12288), (130, 4096)])
@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_stochastic_quantize_matches_oracle(lib, seed, offset, rows, k, layout):
    """Several tiles, a ragged row tail, a ragged second segment of 512
    blocks, and seeds/offsets whose high words are set."""
    x = inputs.activations_with_outliers(rows, k, seed=500 + rows, fraction=0.01, factor=50.0)
    q = lib.quantize_stochastic(dev_bf16(x), seed, offset, layout)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    _assert_same(lib, q, S.quantize_sr(x, seed, offset), layout)


def test_scales_equal_deterministic_and_codes_differ(lib):
    x = inputs.gaussian_bf16((256, 2048), seed=61)
    xd = dev_bf16(x)
    a = lib.quantize_stochastic(xd, 7, 0, lib.SF_TCGEN05)
    b = lib.quantize(xd, lib.SF_TCGEN05)
    c = lib.quantize_stochastic(xd, 7, 1, lib.SF_TCGEN05)
    d = lib.quantize_stochastic(xd, 7, 0, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    assert torch.equal(a.sf, b.sf) and torch.equal(a.g, b.g)
    assert not torch.equal(a.codes, b.codes) and not torch.equal(a.codes, c.codes)
    assert torch.equal(a.codes, d.codes)


def test_pitched_rows_and_given_amax(lib):
    rows, k, ld = 37, 512, 520
    x = inputs.gaussian_bf16((rows, k), seed=71)
    pitched = np.zeros((rows, ld), dtype=np.uint16)
    pitched[:, :k] = x
    amax = float(O.amax(x)) / 2
    q = lib.quantize_stochastic(dev_bf16(pitched)[:, :k], 3, 9, lib.SF_ROWMAJOR,
                                amax=torch.tensor([amax], dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    _assert_same(lib, q, S.quantize_sr(x, 3, 9, amax_value=amax), lib.SF_ROWMAJOR)


def test_edge_tensor_and_nonfinite(lib):
    """Ties, -0, subnormal and zero block scales, a zero block; +inf reports RANGE."""
    x = np.zeros((4, 128))
    x[0, 0] = 2688.0
    x[1, 0:16] = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -0.1]
    x[2, 0:16] = 0.01 * np.linspace(-1, 1, 16)
    x[2, 16:32] = 0.0005 * np.linspace(-1, 1, 16)
    x[3, :] = inputs.normal(5, 0, 128) * 10.0
    x[3, 64:80] = 0.0
    xb = inputs.f64_to_bf16_bits(x)
    xb[3, 90] = 0x8000                                   # -0
    q = lib.quantize_stochastic(dev_bf16(xb), 99, 5, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    _assert_same(lib, q, S.quantize_sr(xb, 99, 5), lib.SF_TCGEN05)
    xb = inputs.gaussian_bf16((16, 128), seed=51).copy()
    xb[3, 17] = 0x7F80
    q = lib.quantize_stochastic(dev_bf16(xb), 1, 1, lib.SF_TCGEN05)
    assert lib.nvfp4_check_device_status() == lib.ERR_RANGE
    assert f32_scalar(q.g) == 0.0 and not host_u8(q.codes).any()


def test_full_size_every_byte(lib):
    """Quantize-bandwidth workload [16384, 8192]: g and amax exact, every code
    byte and every scale equal to the oracle's (run over the host cores by
    rows, each row drawing the random integers of its own index)."""
    x = inputs.quantize_bandwidth()
    seed, offset = 0x5EED, 11
    q = lib.quantize_stochastic(dev_bf16(x), seed, offset, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    codes_ref, sf_ref, g, amax = oracle_pool.quantize_sr(x, seed, offset)
    assert f32_scalar(q.amax) == amax and f32_scalar(q.g) == g
    assert np.array_equal(host_u8(q.codes), codes_ref)
    assert np.array_equal(O.unswizzle_sf_tcgen05(host_u8(q.sf), *x.shape), sf_ref)


def test_mean_over_offsets_is_unbiased(lib):
    """Averaged over 256 offsets on the GPU, the dequantized values approach
    x far more closely than one deterministic quantization does."""
    x = inputs.gaussian_bf16((64, 256), seed=81)
    xd = dev_bf16(x)
    xf = O.bf16_to_f32(x).astype(np.float64)
    acc = np.zeros_like(xf)
    for off in range(256):
        q = lib.quantize_stochastic(xd, 2024, off, lib.SF_ROWMAJOR)
        acc += O.dequantize(host_u8(q.codes), host_u8(q.sf).reshape(64, 16), f32_scalar(q.g))
    p, sf, g, _ = O.quantize(x)
    err_rn = np.abs(O.dequantize(p, sf, g) - xf).mean()
    assert np.abs(acc / 256 - xf).mean() < 0.2 * err_rn
