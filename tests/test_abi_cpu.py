"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/nvfp4.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent


@pytest.fixture(scope="module")
def built():
    from nvfp4_block_scaled_15_b200 import build
    return build.build()


@pytest.fixture(scope="module")
def nv(built):
    from nvfp4_block_scaled_15_b200 import nvfp4
    return nvfp4


def _declared_functions():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        text = h.read_text()
        names |= set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(built):
    lib = ctypes.CDLL(built)
    declared = _declared_functions()
    assert len(declared) >= 13
    missing = [n for n in declared if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_symbol(nv):
    for name in _declared_functions():
        assert hasattr(nv, name), name


def test_version_and_status_strings(nv):
    assert nv.nvfp4_abi_version() == 1
    assert nv.status_string(nv.OK) == "NVFP4_OK"
    assert nv.status_string(nv.ERR_TIMEOUT) == "NVFP4_ERR_TIMEOUT"
    assert nv.status_string(99) == "NVFP4_ERR_UNKNOWN"


def test_sf_bytes_matches_layout_definition(nv):
    from oracle import nvfp4_oracle as O
    for rows, k in [(1, 64), (128, 256), (200, 320), (16384, 8192), (28672, 8192)]:
        assert nv.nvfp4_sf_bytes(rows, k, nv.SF_ROWMAJOR) == rows * k // 16
        assert nv.nvfp4_sf_bytes(rows, k, nv.SF_TCGEN05) == O.sf_tcgen05_bytes(rows, k)
    assert nv.nvfp4_sf_bytes(10, 24, nv.SF_ROWMAJOR) == 0        # k not a multiple of 16
    assert nv.nvfp4_sf_bytes(-1, 64, nv.SF_ROWMAJOR) == 0


def test_workspace_bytes(nv):
    assert nv.nvfp4_workspace_bytes(nv.OP_GEMV_BATCHED, 16, 28672, 8192) >= 16 * 28672 * 4 + 32 * 4096
    assert nv.nvfp4_workspace_bytes(nv.OP_GEMV_BATCHED, 33, 128, 128) == 0     # M > 32
    assert nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, 4096, 8192, 28672) >= 4096 * 14336
    assert nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, 16, 16, 100) == 0      # K % 64
    # A codes, A's tensor-core scales, then g_a, amax_a, the unit ticket and one int
    # counter per (256-row block, K chunk of 4096)
    for m, n, k in ((8192, 8192, 8192), (300, 260, 512), (1, 1, 64), (20000, 4096, 1024), (4096, 8192, 28672)):
        rup = lambda v: (v + 255) // 256 * 256
        chunks = -(-k // 4096)
        want = (rup(m * k // 2) + rup(nv.nvfp4_sf_bytes(m, k, nv.SF_TCGEN05))
                + rup(128 + 4 * ((m + 255) // 256) * chunks))
        assert nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, m, n, k) == want


def test_argument_errors_return_before_any_device_work(nv):
    fake = 1 << 20                      # 16-B aligned, never dereferenced
    raw = nv.raw_status
    assert raw("nvfp4_quantize", None, 4, 64, 64, fake, fake, 1, fake, fake, 0, None) == nv.ERR_INVALID_ARG
    assert raw("nvfp4_quantize", fake, 4, 48, 48, fake, fake, 1, fake, fake, 0, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert raw("nvfp4_quantize", fake + 8, 4, 64, 64, fake, fake, 1, fake, fake, 0, None) == nv.ERR_MISALIGNED
    assert raw("nvfp4_quantize", fake, 4, 64, 60, fake, fake, 1, fake, fake, 0, None) == nv.ERR_INVALID_ARG
    assert raw("nvfp4_quantize", fake, 4, 64, 64, fake, fake, 7, fake, fake, 0, None) == nv.ERR_INVALID_ARG
    assert raw("nvfp4_gemm", fake, fake, fake, fake, fake, fake, 8, 8, 96, fake, 8, 0, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert raw("nvfp4_gemm", fake, fake, fake, fake, fake, fake, 0, 8, 64, fake, 8, 0, None) == nv.ERR_INVALID_ARG
    assert raw("nvfp4_gemm", fake, fake, fake, fake, fake, fake, 8, 8, 64, fake, 4, 0, None) == nv.ERR_INVALID_ARG
    assert raw("nvfp4_gemm", fake, fake, fake, fake, fake, fake, 8, 8, 64, fake + 1, 12, 0, None) == nv.ERR_MISALIGNED
    assert raw("nvfp4_gemm", fake, fake, fake, fake + 4, fake, fake, 8, 8, 64, fake, 8, 0, None) == nv.ERR_MISALIGNED
    assert raw("nvfp4_gemv_batched", fake, 33, 64, fake, fake, fake, 128, 64, fake, 128, fake, 1 << 30, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert raw("nvfp4_gemv_batched", fake, 4, 64, fake, fake, fake, 128, 64, fake, 128, fake, 16, None) == nv.ERR_WORKSPACE
    assert raw("nvfp4_gemm_quant_a", fake, 64, fake, fake, fake, 8, 8, 64, fake, 8, 0, fake, 16, None) == nv.ERR_WORKSPACE
    assert raw("nvfp4_gemm_quant_a_prepare", fake, 64, 8, 8, 64, fake, 16, None) == nv.ERR_WORKSPACE
    assert raw("nvfp4_gemm_quant_a_prepare", fake, 96, 8, 8, 96, fake, 1 << 20, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert raw("nvfp4_gemm_quant_a_run", fake, 64, fake, fake, fake, 8, 8, 64, fake, 8, 0, fake, 16, None) == nv.ERR_WORKSPACE
    assert raw("nvfp4_gemm_quant_a_run", fake, 64, fake, fake, fake, 8, 8, 64, fake, 4, 0, fake, 1 << 20, None) == nv.ERR_INVALID_ARG
    qa_amax = "nvfp4_gemm_quant_a_amax"
    assert raw(qa_amax, fake, 64, None, fake, fake, fake, 8, 8, 64, fake, 8, 0, fake, 1 << 20, None) == nv.ERR_INVALID_ARG
    assert raw(qa_amax, fake, 64, fake, fake, fake, fake, 8, 8, 64, fake, 8, 0, fake, 16, None) == nv.ERR_WORKSPACE
    assert raw("nvfp4_swizzle_sf", fake, 4, 48, fake, None) == nv.ERR_UNSUPPORTED_SHAPE
    qs = "nvfp4_quantize_stochastic"
    assert raw(qs, fake, 4, 48, 48, fake, fake, 1, fake, fake, 0, 1, 2, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert raw(qs, fake, 4, 64, 64, fake, fake, 1, fake, fake, 2, 1, 2, None) == nv.ERR_INVALID_ARG
    assert raw(qs, fake, 4, 64, 64, None, fake, 1, fake, fake, 0, 1, 2, None) == nv.ERR_INVALID_ARG
    # Hadamard order: a power of two in [1, 512] that divides k
    qh = "nvfp4_quantize_hadamard"
    for order in (0, 3, 1024, -16):
        assert raw(qh, fake, 4, 256, 256, order, fake, fake, 1, fake, fake, 0, None) == nv.ERR_INVALID_ARG
    assert raw(qh, fake, 4, 192, 192, 128, fake, fake, 1, fake, fake, 0, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert raw(qh, fake, 4, 48, 48, 16, fake, fake, 1, fake, fake, 0, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert raw(qh, fake, 4, 64, 64, 16, fake + 2, fake, 1, fake, fake, 0, None) == nv.ERR_MISALIGNED
    qhs = "nvfp4_quantize_hadamard_stochastic"
    assert raw(qhs, fake, 4, 256, 256, 3, fake, fake, 1, fake, fake, 0, 1, 2, None) == nv.ERR_INVALID_ARG
    assert raw(qhs, fake, 4, 192, 192, 128, fake, fake, 1, fake, fake, 0, 1, 2, None) == nv.ERR_UNSUPPORTED_SHAPE


def test_no_device_means_cuda_or_arch_error(nv):
    """Valid arguments on a machine without a B200 stop at the device check."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    fake = 1 << 20
    st = nv.raw_status("nvfp4_quantize", fake, 4, 64, 64, fake, fake, 1, fake, fake, 0, None)
    assert st in (nv.ERR_CUDA, nv.ERR_ARCH)
    # an empty tensor may come with null pointers: the arguments pass, the device check stops it
    for rows, k in [(0, 64), (4, 0)]:
        st = nv.raw_status("nvfp4_quantize", None, rows, k, 64, None, None, 1, fake, fake, 0, None)
        assert st in (nv.ERR_CUDA, nv.ERR_ARCH)
    assert nv.raw_status("nvfp4_quantize", None, 4, 64, 64, None, None, 1, fake, fake, 0, None) == nv.ERR_INVALID_ARG
