"""Quantize parity: the CUDA quantizer against the CPU oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle_pool
from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import dev_bf16, f32_scalar, host_u8

pytestmark = pytest.mark.gpu


def _quantize_both(nv, x_bits, layout, amax=None, ld=None):
    rows, k = x_bits.shape
    if ld is not None and ld != k:
        pitched = np.zeros((rows, ld), dtype=np.uint16)
        pitched[:, :k] = x_bits
        xd = dev_bf16(pitched)[:, :k]
    else:
        xd = dev_bf16(x_bits)
    amax_t = None if amax is None else torch.tensor([amax], dtype=torch.float32, device="cuda")
    q = nv.quantize(xd, layout, amax=amax_t)
    torch.cuda.synchronize()
    assert nv.nvfp4_check_device_status() == nv.OK
    ref = O.quantize(x_bits, amax_value=amax)
    return q, ref


def _assert_same(nv, q, ref, layout, rows, k):
    codes_ref, sf_ref, g_ref, amax_ref = ref
    assert f32_scalar(q.g).tobytes() == np.float32(g_ref).tobytes(), (f32_scalar(q.g), g_ref)
    assert f32_scalar(q.amax).tobytes() == np.float32(amax_ref).tobytes()
    codes = host_u8(q.codes)
    bad = np.argwhere(codes != codes_ref)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:3].tolist()}"
    sf = host_u8(q.sf)
    want = sf_ref.reshape(-1) if layout == nv.SF_ROWMAJOR else O.swizzle_sf_tcgen05(sf_ref)
    assert sf.size == want.size
    bad = np.nonzero(sf != want)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:5].tolist()}"


SHAPES = [(128, 256), (256, 256), (200, 320), (1, 64), (3, 8192), (129, 1024), (130, 28672)]


@pytest.mark.parametrize("rows,k", SHAPES)
@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_quantize_matches_oracle(lib, rows, k, layout):
    x = inputs.activations_with_outliers(rows, k, seed=100 + rows, fraction=0.01, factor=50.0)
    q, ref = _quantize_both(lib, x, layout)
    _assert_same(lib, q, ref, layout, rows, k)


@pytest.mark.parametrize("rows,k", [(5, 48), (7, 16), (2, 208)])
def test_quantize_rowmajor_k_multiple_of_16(lib, rows, k):
    x = inputs.gaussian_bf16((rows, k), seed=7 + k)
    q, ref = _quantize_both(lib, x, lib.SF_ROWMAJOR)
    _assert_same(lib, q, ref, lib.SF_ROWMAJOR, rows, k)


def test_quantize_pitched_rows(lib):
    x = inputs.gaussian_bf16((37, 512), seed=31)
    q, ref = _quantize_both(lib, x, lib.SF_TCGEN05, ld=520)
    _assert_same(lib, q, ref, lib.SF_TCGEN05, 37, 512)


def _edge_tensor():
    """g = 1 exactly (amax 2688), then blocks that hit every E2M1 tie point,
    -0, subnormal and zero block scales, a constant block and a zero block."""
    rows, k = 4, 128
    x = np.zeros((rows, k))
    x[0, 0] = 2688.0                                        # tensor amax -> g = 1
    ties = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -0.1]
    x[1, 0:16] = ties                                       # block max 6 -> scale 1 -> u = x
    x[1, 16:32] = [6.0] + [0.24, 0.26, 0.74, 0.76, 1.24, 1.26, 1.74, 1.76, 2.49, 2.51, 3.49, 3.51, 4.99, 5.01, -6.0]
    x[2, 0:16] = 0.01 * np.linspace(-1, 1, 16)              # scale 0.01/6: E4M3 subnormal
    x[2, 16:32] = 0.0005 * np.linspace(-1, 1, 16)           # scale rounds to 0 -> codes 0
    x[2, 32:48] = 3.0                                       # constant block
    x[3, :] = inputs.normal(5, 0, k) * 10.0
    x[3, 64:80] = 0.0                                       # zero block
    return inputs.f64_to_bf16_bits(x)


@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
def test_quantize_edge_cases(lib, layout):
    x = _edge_tensor()
    q, ref = _quantize_both(lib, x, layout)
    _assert_same(lib, q, ref, layout, *x.shape)
    assert f32_scalar(q.g) == np.float32(1.0)


def test_quantize_all_zero_tensor(lib):
    x = np.zeros((8, 256), dtype=np.uint16)
    q, ref = _quantize_both(lib, x, lib.SF_TCGEN05)
    _assert_same(lib, q, ref, lib.SF_TCGEN05, 8, 256)
    assert f32_scalar(q.g) == np.float32(1.0)


def test_quantize_given_amax_saturates(lib):
    """A caller amax below the true amax: scales clamp at 448, codes at +-6."""
    x = inputs.gaussian_bf16((64, 256), seed=41)
    amax = float(O.amax(x)) / 4
    q, ref = _quantize_both(lib, x, lib.SF_TCGEN05, amax=amax)
    _assert_same(lib, q, ref, lib.SF_TCGEN05, 64, 256)
    assert np.any(ref[1] == 0x7E)


def test_quantize_nonfinite_reports_range(lib):
    x = inputs.gaussian_bf16((16, 128), seed=51).copy()
    x[3, 17] = 0x7F80                                       # +inf
    xd = dev_bf16(x)
    q = lib.quantize(xd, lib.SF_TCGEN05)
    assert lib.nvfp4_check_device_status() == lib.ERR_RANGE
    assert lib.nvfp4_check_device_status() == lib.OK        # cleared
    assert f32_scalar(q.g) == 0.0
    assert not host_u8(q.codes).any() and not host_u8(q.sf).any()


def test_quantize_tiny_amax_reports_range(lib):
    x = np.zeros((2, 64))
    x[0, 5] = 1e-38
    xb = inputs.f64_to_bf16_bits(x)
    with pytest.raises(O.RangeError):
        O.quantize(xb)
    lib.quantize(dev_bf16(xb), lib.SF_ROWMAJOR)
    assert lib.nvfp4_check_device_status() == lib.ERR_RANGE


def test_amax_entry_point(lib):
    x = inputs.activations_with_outliers(300, 1024, seed=61, fraction=0.01, factor=50.0)
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.nvfp4_amax(dev_bf16(x), 300, 1024, 1024, out)
    assert f32_scalar(out) == O.amax(x)


def test_swizzle_matches_oracle(lib):
    rng = np.random.default_rng(3)
    for rows, k in [(1, 64), (200, 320), (257, 1024)]:
        sf = rng.integers(0, 0x7F, size=(rows, k // 16), dtype=np.uint8)
        src = torch.from_numpy(sf).cuda()
        dst = torch.full((lib.nvfp4_sf_bytes(rows, k, lib.SF_TCGEN05),), 0xAB, dtype=torch.uint8, device="cuda")
        lib.nvfp4_swizzle_sf(src, rows, k, dst)
        assert np.array_equal(host_u8(dst), O.swizzle_sf_tcgen05(sf))


def test_quantize_full_size_every_byte(lib):
    """Quantize-bandwidth workload [16384, 8192] with 1% outlier channels:
    amax, g, all 67,108,864 code bytes and all 8,388,608 block scales
    bit-exact against the oracle (run over the host cores by row slices)."""
    x = inputs.quantize_bandwidth()
    q = lib.quantize(dev_bf16(x), lib.SF_TCGEN05)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    codes_ref, sf_ref, g, amax = oracle_pool.quantize(x)
    assert f32_scalar(q.amax) == amax and f32_scalar(q.g) == g
    assert np.array_equal(host_u8(q.codes), codes_ref)
    assert np.array_equal(host_u8(q.sf), O.swizzle_sf_tcgen05(sf_ref))
