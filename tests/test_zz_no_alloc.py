"""The zero-allocation decode GEMV (nvfp4_gemv_batched_noalloc).

It serves callers that cannot allocate device memory (plug-ins whose host
framework owns the device memory and hands them only their inputs and
outputs, real-time paths that may not call the allocator once started).  It
must give what nvfp4_gemv_batched gives with a caller-allocated workspace, on
consecutive calls that reuse the library's fixed scratch, and it must refuse
shapes that do not fit that scratch.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import check_bf16, dev_bf16, host_bf16_bits

pytestmark = pytest.mark.gpu


def _noalloc(lib, xd, qw):
    m, k = xd.shape
    n = qw.rows
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    lib.nvfp4_gemv_batched_noalloc(xd, m, xd.stride(0), qw.codes, qw.sf, qw.g, n, k, y, y.stride(0))
    return y


@pytest.mark.parametrize("m,n,k", [(8, 1000, 1024), (16, 4096, 4096)], ids=lambda v: str(v))
def test_noalloc_matches_workspace_entry_point_on_two_calls(lib, m, n, k):
    w = inputs.gaussian_bf16((n, k), seed=700 + n, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    pw, sw, gw, _ = O.quantize(w)
    for call, seed in enumerate((801, 802)):          # two calls in a row, different activations
        x = inputs.gaussian_bf16((m, k), seed=seed + m)
        xd = dev_bf16(x)
        y_new = _noalloc(lib, xd, qw)
        y_old = lib.gemv_batched(xd, qw)
        torch.cuda.synchronize()
        assert lib.nvfp4_check_device_status() == lib.OK
        px, sx, gx, _ = O.quantize(x)
        d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, pw, sw, gw)
        new_bits = host_bf16_bits(y_new)
        old_bits = host_bf16_bits(y_old)
        # against the existing entry point, with the tolerance of the parity tests
        check_bf16(new_bits, O.bf16_to_f32(old_bits).astype(np.float64), s_ref, alpha)
        # and both against the oracle
        check_bf16(new_bits, d_ref, s_ref, alpha)
        check_bf16(old_bits, d_ref, s_ref, alpha)


@pytest.mark.parametrize("m", [1, 4])
def test_noalloc_decode_size_split_tiles_on_two_calls(lib, m):
    """The decode workload (W [28672, 8192]: tiles split between CTAs) at
    M <= 8, the kernel whose fix-up counters live in the shared scratch from
    one call to the next: two calls in a row, each equal bit for bit to the
    workspace entry point's output, and 512 sampled columns against the
    oracle."""
    x_first, w = inputs.decode_gemv(m)
    n, k = w.shape
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    gw = O.global_scale(O.amax(w))
    cols = np.sort(np.random.default_rng(53).choice(n, 512, replace=False))
    cw, sw = O.quantize_with_scale(w[cols], gw)
    for x in (x_first, inputs.gaussian_bf16((m, k), seed=811 + m)):
        xd = dev_bf16(x)
        y_new = _noalloc(lib, xd, qw)
        y_old = lib.gemv_batched(xd, qw)
        torch.cuda.synchronize()
        assert lib.nvfp4_check_device_status() == lib.OK
        new_bits = host_bf16_bits(y_new)
        assert np.array_equal(new_bits, host_bf16_bits(y_old))
        px, sx, gx, _ = O.quantize(x)
        d_ref, s_ref, alpha = O.gemm_ref(px, sx, gx, O.pack_codes(cw), sw, gw)
        check_bf16(new_bits[:, cols], d_ref, s_ref, alpha)


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    fake = 1 << 20
    st = lib.raw_status("nvfp4_gemv_batched_noalloc", fake, 32, 32768, fake, fake, fake, 32768, 32768, fake,
                        32768, None)
    assert st == lib.ERR_WORKSPACE
