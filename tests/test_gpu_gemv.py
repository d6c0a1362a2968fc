"""Decode batched GEMV parity (activations quantized inside the call).

Two paths serve the call: for M <= 8 and K <= 8192 one kernel whose CTAs
each quantize the activations (held in registers) into shared memory, and
otherwise a quantizing prologue followed by the GEMV; the shapes below reach
both, with ragged N, K not a multiple of 256 and tiles split between CTAs."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import check_bf16, dev_bf16, host_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m", [1, 3, 5, 8, 13, 16, 17, 32])
@pytest.mark.parametrize("n,k", [(1000, 1024), (128, 64), (384, 4096), (640, 2880)], ids=lambda v: str(v))
def test_gemv_matches_oracle(lib, m, n, k):
    x = inputs.gaussian_bf16((m, k), seed=300 + m)
    w = inputs.gaussian_bf16((n, k), seed=400 + n, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    y = lib.gemv_batched(dev_bf16(x), qw)
    assert lib.nvfp4_check_device_status() == lib.OK
    px, sx, gx, _ = O.quantize(x)
    pw, sw, gw, _ = O.quantize(w)
    d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, pw, sw, gw)
    check_bf16(host_bf16_bits(y), d_ref, s_ref, alpha)


@pytest.mark.parametrize("m", [1, 7, 12, 16])
def test_gemv_tiles_split_between_ctas(lib, m):
    """160 weight tiles on at most 148 CTAs: stream-K ranges split tiles
    between neighbouring CTAs, whose partial sums meet in the workspace.
    Every output is checked against the oracle."""
    n, k = 160 * 128, 1024
    x = inputs.gaussian_bf16((m, k), seed=900 + m)
    w = inputs.gaussian_bf16((n, k), seed=901, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    y = lib.gemv_batched(dev_bf16(x), qw)
    assert lib.nvfp4_check_device_status() == lib.OK
    px, sx, gx, _ = O.quantize(x)
    pw, sw, gw, _ = O.quantize(w)
    d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, pw, sw, gw)
    check_bf16(host_bf16_bits(y), d_ref, s_ref, alpha)


def test_gemv_repeated_calls_reuse_workspace(lib):
    """The workspace is re-initialised by every call: two calls, same answer
    (one shape with whole tiles per CTA, one with split tiles)."""
    for m, n, k in [(8, 640, 512), (8, 2048, 512)]:
        _repeated_calls(lib, m, n, k)


def _repeated_calls(lib, m, n, k):
    x = inputs.gaussian_bf16((m, k), seed=501)
    w = inputs.gaussian_bf16((n, k), seed=502, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMV_BATCHED, m, n, k), dtype=torch.uint8, device="cuda")
    xd = dev_bf16(x)
    y1 = lib.gemv_batched(xd, qw, workspace=ws).clone()
    y2 = lib.gemv_batched(xd, qw, workspace=ws)
    px, sx, gx, _ = O.quantize(x)
    pw, sw, gw, _ = O.quantize(w)
    d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, pw, sw, gw)
    check_bf16(host_bf16_bits(y1), d_ref, s_ref, alpha)
    check_bf16(host_bf16_bits(y2), d_ref, s_ref, alpha)


@pytest.mark.parametrize("m,n,k", [(5, 1100, 960), (16, 1024, 8192), (1, 8192 + 40, 4160), (12, 4096, 64),
                                   (3, 256, 12288), (4, 384, 8192), (20, 512, 10240)],
                         ids=lambda v: str(v))
def test_gemv_more_shapes(lib, m, n, k):
    """A partial last K stage (K % 256 != 0), ragged N, K = 64 (one MMA-K
    step per tile), N = 1024 with K = 8192 (every CTA one whole tile)."""
    x = inputs.activations_with_outliers(m, k, seed=950 + m, fraction=0.01, factor=30.0)
    w = inputs.gaussian_bf16((n, k), seed=951 + n, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    y = lib.gemv_batched(dev_bf16(x), qw)
    assert lib.nvfp4_check_device_status() == lib.OK
    px, sx, gx, _ = O.quantize(x)
    pw, sw, gw, _ = O.quantize(w)
    d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, pw, sw, gw)
    check_bf16(host_bf16_bits(y), d_ref, s_ref, alpha)


@pytest.mark.parametrize("m", [1, 8, 16])
def test_gemv_decode_full_size_sampled(lib, m):
    """Decode workload: W [28672, 8192] N(0,0.02) pre-quantized, x [M, 8192]
    N(0,1); 512 sampled output columns per row against the oracle."""
    x, w = inputs.decode_gemv(m)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    y = lib.gemv_batched(dev_bf16(x), qw)
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    assert torch.isfinite(y).all()
    gw = O.global_scale(O.amax(w))
    px, sx, gx, _ = O.quantize(x)
    cols = np.sort(np.random.default_rng(37).choice(w.shape[0], 512, replace=False))
    cw, sw = O.quantize_with_scale(w[cols], gw)
    d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, O.pack_codes(cw), sw, gw)
    check_bf16(host_bf16_bits(y)[:, cols], d_ref, s_ref, alpha)


@pytest.mark.parametrize("m", [1, 4, 8, 9, 16])
def test_gemv_weights_in_l2_repeated(lib, m):
    """All 148 CTAs running (160 weight tiles) with 94 MB of weights resident in
    L2, so the weight stages reach the tensor core while the CTAs are still
    quantizing the activations (the longest at K = 8192): an MMA issued before
    its activation operand is complete would show as a gross error.  Ten calls
    in a row must be identical and within 2 bf16 ulp of the block-scaled GEMM
    on the same quantized operands (parity of both against the oracle is
    tested elsewhere)."""
    n, k = 20480, 8192
    x = inputs.activations_with_outliers(m, k, seed=970 + m, fraction=0.01, factor=30.0)
    w = inputs.gaussian_bf16((n, k), seed=971, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    xd = dev_bf16(x)
    ref = lib.gemm(lib.quantize(xd, lib.SF_TCGEN05), qw)
    ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMV_BATCHED, m, n, k), dtype=torch.uint8, device="cuda")
    outs = [lib.gemv_batched(xd, qw, workspace=ws) for _ in range(10)]
    torch.cuda.synchronize()
    assert lib.nvfp4_check_device_status() == lib.OK
    first = host_bf16_bits(outs[0])
    for y in outs[1:]:
        assert np.array_equal(host_bf16_bits(y), first)
    ulps = np.abs(O.bf16_ordinal(first) - O.bf16_ordinal(host_bf16_bits(ref)))
    assert int(ulps.max()) <= 2, int(ulps.max())
