"""Quantize-and-multiply (nvfp4_gemm_quant_a and its _prepare / _run and
_amax forms): a bf16 A quantized inside the call, then the block-scaled GEMM.
Where one kernel does both (M, N > 128), its codes, scales, g_a and D must
equal, bit for bit, those of the quantize pass followed by the GEMM, and both
must agree with the oracle.  Both of its schedules are covered: tiles row
block by row block (B's codes within 64 MiB) and m-fastest tiles with A
quantized chunk by chunk along K (larger B, the long-K workload)."""
import numpy as np
import pytest
import torch

import oracle_pool
from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import check_bf16, check_f32, dev_bf16, f32_scalar, host_bf16_bits, host_u8

pytestmark = pytest.mark.gpu

# (M, N, K, extra row pitch of A in elements)
SHAPES = [
    (200, 136, 640, 0),      # one row block, 56 padding rows of the scale layout, K not a multiple of 512 blocks
    (1000, 520, 1088, 0),    # four row blocks, tails in M and N, odd number of K stages
    (777, 300, 4096, 8),     # A rows 16-B but not 32-B aligned: 128-bit loads
    (2048, 4096, 8192, 0),   # a full 8192-wide row per quantizer pass, 256 tiles (more than one wave)
    (4352, 384, 12288, 0),   # 17 row blocks, K beyond one pass per row
    (600, 8488, 16384, 8),   # B's codes > 64 MiB (one group of 3 row blocks); ragged M and N
    (2100, 8488, 16384, 0),  # B's codes > 64 MiB: 9 row blocks in 3 groups of 3, the last row block 52 rows
]


def _a_input(m, k, pad, seed):
    a = inputs.activations_with_outliers(m, k, seed=seed, fraction=0.01, factor=30.0)
    if pad == 0:
        return a, dev_bf16(a)
    big = torch.zeros((m, k + pad), dtype=torch.bfloat16, device="cuda")
    big[:, :k] = dev_bf16(a)
    return a, big[:, :k]


def _two_kernel(lib, a_dev, qw, out_dtype):
    qa = lib.quantize(a_dev, lib.SF_TCGEN05)
    d = lib.gemm(qa, qw, out_dtype=out_dtype)
    return qa, d


def _check_same_as_two_kernel(lib, a_dev, qw, m, k, out_dtype):
    ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMM_QUANT_A, m, qw.rows, k), dtype=torch.uint8, device="cuda")
    d = lib.gemm_quant_a(a_dev, qw, out_dtype=out_dtype, workspace=ws)
    assert lib.nvfp4_check_device_status() == lib.OK
    qa, d2 = _two_kernel(lib, a_dev, qw, out_dtype)
    assert lib.nvfp4_check_device_status() == lib.OK
    codes, sf, g = lib.quant_a_workspace_views(ws, m, k)
    assert torch.equal(codes, qa.codes)
    assert torch.equal(sf, qa.sf)
    assert torch.equal(g, qa.g)
    assert torch.equal(d.view(torch.int16) if d.dtype == torch.bfloat16 else d.view(torch.int32),
                       d2.view(torch.int16) if d2.dtype == torch.bfloat16 else d2.view(torch.int32))
    return d, qa


@pytest.mark.parametrize("m,n,k,pad", SHAPES, ids=lambda v: str(v))
def test_quant_a_against_oracle_and_two_kernel_path(lib, m, n, k, pad):
    a, a_dev = _a_input(m, k, pad, seed=m + 3 * k)
    w = inputs.gaussian_bf16((n, k), seed=n + k, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    d, qa = _check_same_as_two_kernel(lib, a_dev, qw, m, k, torch.float32)
    ga = O.global_scale(O.amax(a))
    gw = O.global_scale(O.amax(w))
    assert f32_scalar(qa.g) == ga
    rng = np.random.default_rng(m * 7 + n)
    rows = rng.choice(m, min(m, 96), replace=False)
    cols = rng.choice(n, min(n, 96), replace=False)
    ur, uc = np.sort(rows), np.sort(cols)
    ca, sa = O.quantize_with_scale(a[ur], ga)
    cw, sw = O.quantize_with_scale(w[uc], gw)
    assert np.array_equal(host_u8(qa.codes)[ur], O.pack_codes(ca))
    d_ref, s_ref, alpha = O.gemm_ref_entries(O.pack_codes(ca), sa, ga, O.pack_codes(cw), sw, gw,
                                             np.repeat(np.arange(len(ur)), len(uc)),
                                             np.tile(np.arange(len(uc)), len(ur)))
    got = d.cpu().numpy()[np.repeat(ur, len(uc)), np.tile(uc, len(ur))]
    check_f32(got, d_ref, s_ref, alpha)


def test_quant_a_bf16_out_prefill_full_size(lib):
    """Prefill workload 8192^3 through the quantize-and-multiply call: the
    whole bf16 D, A's codes and scales equal the two-kernel path's bit for bit
    (whose D tests/test_gpu_gemm.py::test_gemm_prefill_full_size checks
    against the oracle on every output); every code byte and scale of A, and
    256 sampled outputs, against the oracle."""
    a, w = inputs.prefill_gemm()
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    a_dev = dev_bf16(a)
    d, qa = _check_same_as_two_kernel(lib, a_dev, qw, a.shape[0], a.shape[1], torch.bfloat16)
    assert torch.isfinite(d).all()
    # every code byte and block scale of A (the quantize-and-GEMM kernel's, equal to qa's) against the oracle
    ca_all, sa_all, ga, _ = oracle_pool.quantize(a)
    assert f32_scalar(qa.g) == ga
    assert np.array_equal(host_u8(qa.codes), ca_all)
    assert np.array_equal(host_u8(qa.sf), O.swizzle_sf_tcgen05(sa_all))
    gw = O.global_scale(O.amax(w))
    rng = np.random.default_rng(41)
    rows = rng.choice(a.shape[0], 256)
    cols = rng.choice(w.shape[0], 256)
    ur, uc = np.unique(rows), np.unique(cols)
    ca, sa = O.quantize_with_scale(a[ur], ga)
    cw, sw = O.quantize_with_scale(w[uc], gw)
    ri = np.searchsorted(ur, rows)
    ci = np.searchsorted(uc, cols)
    d_ref, s_ref, alpha = O.gemm_ref_entries(O.pack_codes(ca), sa, ga, O.pack_codes(cw), sw, gw, ri, ci)
    check_bf16(host_bf16_bits(d)[rows, cols], d_ref, s_ref, alpha)


@pytest.mark.parametrize("n", [260, 264], ids=lambda v: f"n{v}")
def test_quant_a_bf16_into_wider_output(lib, n):
    """bf16 D written into a wider, taller buffer (row pitch n + 40): N = 260
    ends inside a 16-B chunk (direct stores from the 64-column drain), N = 264
    on a chunk boundary (TMA stores); equal to the two-kernel path, nothing
    outside the M x N window changes."""
    m, k = 300, 512
    _, a_dev = _a_input(m, k, 0, seed=n)
    w = inputs.gaussian_bf16((n, k), seed=n + 1, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    big = torch.full((m + 8, n + 40), -7.0, dtype=torch.bfloat16, device="cuda")
    lib.gemm_quant_a(a_dev, qw, out=big[:m, :n])
    _, d2 = _two_kernel(lib, a_dev, qw, torch.bfloat16)
    assert lib.nvfp4_check_device_status() == lib.OK
    assert torch.equal(big[:m, :n].contiguous().view(torch.int16), d2.view(torch.int16))
    assert torch.all(big[:m, n:] == -7.0)
    assert torch.all(big[m:, :] == -7.0)


def test_quant_a_amax_given_equals_own_amax(lib):
    """nvfp4_gemm_quant_a_amax with the amax from nvfp4_amax gives what
    nvfp4_gemm_quant_a gives with its own amax pass."""
    m, n, k = 1000, 520, 1088
    a, a_dev = _a_input(m, k, 0, seed=5)
    w = inputs.gaussian_bf16((n, k), seed=6, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    d1 = lib.gemm_quant_a(a_dev, qw, out_dtype=torch.float32)
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.nvfp4_amax(a_dev, m, k, a_dev.stride(0), amax)
    d2 = lib.gemm_quant_a(a_dev, qw, out_dtype=torch.float32, amax=amax)
    assert lib.nvfp4_check_device_status() == lib.OK
    assert float(amax.item()) == float(O.amax(a))
    assert torch.equal(d1.view(torch.int32), d2.view(torch.int32))


def test_quant_a_prepare_then_run_equals_one_call(lib):
    """_prepare then _run (with unrelated work enqueued between them) gives
    what one nvfp4_gemm_quant_a call gives, bit for bit, on the fused path and
    on the two-kernel path (N <= 128)."""
    for m, n, k in ((1000, 520, 1088), (300, 96, 512)):
        a, a_dev = _a_input(m, k, 0, seed=m)
        w = inputs.gaussian_bf16((n, k), seed=n, std=0.02)
        qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
        d1 = lib.gemm_quant_a(a_dev, qw, out_dtype=torch.float32)
        ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMM_QUANT_A, m, n, k), dtype=torch.uint8, device="cuda")
        d2 = torch.empty((m, n), dtype=torch.float32, device="cuda")
        lib.nvfp4_gemm_quant_a_prepare(a_dev, k, m, n, k, ws, ws.numel())
        other = torch.randn(1 << 20, device="cuda").sum()          # unrelated work between the calls
        lib.nvfp4_gemm_quant_a_run(a_dev, k, qw.codes, qw.sf, qw.g, m, n, k, d2, n, lib.OUT_F32, ws, ws.numel())
        assert lib.nvfp4_check_device_status() == lib.OK
        assert torch.isfinite(other)
        assert torch.equal(d1.view(torch.int32), d2.view(torch.int32))


def test_quant_a_workspace_reused_across_inputs(lib):
    """Five calls on one workspace with a different A each time: each call
    zeroes the row-block counters first, so no call starts its GEMM on rows
    left by the previous call; each result equals the two-kernel path's."""
    m, n, k = 1536, 512, 2048
    w = inputs.gaussian_bf16((n, k), seed=8, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMM_QUANT_A, m, n, k), dtype=torch.uint8, device="cuda")
    outs = []
    for i in range(5):
        _, a_dev = _a_input(m, k, 0, seed=100 + i)
        outs.append((a_dev, lib.gemm_quant_a(a_dev, qw, out_dtype=torch.float32, workspace=ws)))
    assert lib.nvfp4_check_device_status() == lib.OK
    for a_dev, d in outs:
        _, d2 = _two_kernel(lib, a_dev, qw, torch.float32)
        assert torch.equal(d.view(torch.int32), d2.view(torch.int32))


def test_quant_a_non_finite_input(lib):
    """An inf in A: the global scale is not finite, so g_a = 0, all codes and
    scales are zero, the status word reports a range error and D is NaN, as on
    the two-kernel path."""
    m, n, k = 300, 260, 512
    a = inputs.gaussian_bf16((m, k), seed=12)
    a[17, 100] = 0x7F80
    w = inputs.gaussian_bf16((n, k), seed=13, std=0.02)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMM_QUANT_A, m, n, k), dtype=torch.uint8, device="cuda")
    d = lib.gemm_quant_a(dev_bf16(a), qw, out_dtype=torch.float32, workspace=ws)
    assert lib.nvfp4_check_device_status() == lib.ERR_RANGE
    codes, sf, g = lib.quant_a_workspace_views(ws, m, k)
    assert float(g.item()) == 0.0
    assert not codes.any() and not sf.any()
    assert torch.isnan(d).all()


def test_quant_a_long_k_full_size(lib):
    """Long-K workload: A [4096, 28672] = a*silu(b) quantized inside the call
    (the m-fastest schedule: W's codes are 117 MB), W [8192, 28672] N(0, 0.02)
    pre-quantized.  The whole bf16 D, A's codes and scales equal the
    two-kernel path's bit for bit; every code byte and scale of A and W, and
    every one of the 33,554,432 outputs, against the oracle."""
    a, w = inputs.long_k()
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    d, qa = _check_same_as_two_kernel(lib, dev_bf16(a), qw, a.shape[0], a.shape[1], torch.bfloat16)
    assert torch.isfinite(d).all()
    ca_all, sa_all, ga, _ = oracle_pool.quantize(a)
    assert f32_scalar(qa.g) == ga
    assert np.array_equal(host_u8(qa.codes), ca_all)
    assert np.array_equal(host_u8(qa.sf), O.swizzle_sf_tcgen05(sa_all))
    pw, sw, gw, _ = oracle_pool.quantize(w)
    assert f32_scalar(qw.g) == gw and np.array_equal(host_u8(qw.codes), pw)
    d_ref, s_ref, alpha = oracle_pool.gemm_ref(ca_all, sa_all, ga, pw, sw, gw)
    check_bf16(host_bf16_bits(d), d_ref, s_ref, alpha)


def test_quant_a_two_streams_at_once(lib):
    """Two quantize-and-GEMM calls on two streams, three times over: their
    CTAs compete for the SMs, so each call has CTAs that start only after
    others of the same launch finished.  Warps take units of A from a ticket
    counter, so the resident CTAs quantize what their tiles wait for: both
    calls finish without a wait running out, with the single-call results."""
    m, n, k = 2048, 4096, 8192
    outs, refs, args = [], [], []
    for seed in (501, 502):
        a, _ = _a_input(m, k, 0, seed=seed)
        w = inputs.gaussian_bf16((n, k), seed=seed + 1, std=0.02)
        qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
        a_dev = dev_bf16(a)
        refs.append(lib.gemm_quant_a(a_dev, qw))
        ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMM_QUANT_A, m, n, k), dtype=torch.uint8, device="cuda")
        args.append((a_dev, qw, ws))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(3):
        outs = []
        for st, (a_dev, qw, ws) in zip(streams, args):
            with torch.cuda.stream(st):
                outs.append(lib.gemm_quant_a(a_dev, qw, workspace=ws, stream=st))
        torch.cuda.synchronize()
        assert lib.nvfp4_check_device_status() == lib.OK
        for d, ref in zip(outs, refs):
            assert torch.equal(d.view(torch.int16), ref.view(torch.int16))
