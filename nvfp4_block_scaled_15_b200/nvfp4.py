"""Thin Python binding of libnvfp4 (include/nvfp4.h).

Argument marshalling only: every function passes raw pointers, sizes and the
current CUDA stream to the C ABI and raises NVFP4Error on a non-zero status.
PyTorch provides device memory and streams; no computation happens here.
The library must be built (``python -m nvfp4_block_scaled_15_b200.build``);
importing this module fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m nvfp4_block_scaled_15_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

# status codes (nvfp4_status)
OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_MISALIGNED = 3
ERR_ARCH = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_RANGE = 7
ERR_WORKSPACE = 8
# nvfp4_sf_layout
SF_ROWMAJOR = 0
SF_TCGEN05 = 1
# nvfp4_out_dtype
OUT_BF16 = 0
OUT_F32 = 1
# nvfp4_op
OP_GEMV_BATCHED = 1
OP_GEMM_QUANT_A = 2

_vp, _i64, _sz, _i32, _u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64
_SIGS = {
    "nvfp4_abi_version": ([], _i32),
    "nvfp4_status_string": ([_i32], ctypes.c_char_p),
    "nvfp4_sf_bytes": ([_i64, _i64, _i32], _sz),
    "nvfp4_amax": ([_vp, _i64, _i64, _i64, _vp, _vp], _i32),
    "nvfp4_quantize": ([_vp, _i64, _i64, _i64, _vp, _vp, _i32, _vp, _vp, _i32, _vp], _i32),
    "nvfp4_quantize_stochastic": ([_vp, _i64, _i64, _i64, _vp, _vp, _i32, _vp, _vp, _i32, _u64, _u64, _vp],
                                  _i32),
    "nvfp4_quantize_hadamard_stochastic": ([_vp, _i64, _i64, _i64, _i32, _vp, _vp, _i32, _vp, _vp, _i32, _u64, _u64,
                                            _vp], _i32),
    "nvfp4_quantize_hadamard": ([_vp, _i64, _i64, _i64, _i32, _vp, _vp, _i32, _vp, _vp, _i32, _vp], _i32),
    "nvfp4_swizzle_sf": ([_vp, _i64, _i64, _vp, _vp], _i32),
    "nvfp4_gemm": ([_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _i32, _vp], _i32),
    "nvfp4_gemm_fp8_out": ([_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _vp], _i32),
    "nvfp4_gemm_requant": ([_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _i32, _vp, _vp],
                           _i32),
    "nvfp4_workspace_bytes": ([_i32, _i64, _i64, _i64], _sz),
    "nvfp4_gemv_batched": ([_vp, _i64, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _i64, _vp, _sz, _vp], _i32),
    "nvfp4_gemm_quant_a": ([_vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _i32, _vp, _sz, _vp], _i32),
    "nvfp4_gemm_quant_a_prepare": ([_vp, _i64, _i64, _i64, _i64, _vp, _sz, _vp], _i32),
    "nvfp4_gemm_quant_a_run": ([_vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _i32, _vp, _sz, _vp], _i32),
    "nvfp4_gemm_quant_a_amax": ([_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _i32, _vp, _sz, _vp],
                                _i32),
    "nvfp4_gemv_batched_noalloc": ([_vp, _i64, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _i64, _vp], _i32),
    "nvfp4_mxfp4_sf_bytes": ([_i64, _i64, _i32], _sz),
    "nvfp4_mxfp4_quantize": ([_vp, _i64, _i64, _i64, _vp, _vp, _i32, _vp], _i32),
    "nvfp4_mxfp4_gemm": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _i32, _vp], _i32),
    "nvfp4_check_device_status": ([_vp], _i32),
    "nvfp4_set_wait_limit_ns": ([_u64], None),
    "nvfp4_selftest_wait_timeout": ([_u64, _vp], _i32),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def nvfp4_status_string(status: int) -> str:
    return _lib.nvfp4_status_string(int(status)).decode()


status_string = nvfp4_status_string


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != OK:
        raise NVFP4Error(status, where)


# ---------------------------------------------------------------------------
# one wrapper per C entry point
# ---------------------------------------------------------------------------
def nvfp4_abi_version() -> int:
    return _lib.nvfp4_abi_version()


def nvfp4_sf_bytes(rows: int, k: int, layout: int) -> int:
    return _lib.nvfp4_sf_bytes(rows, k, layout)


def nvfp4_workspace_bytes(op: int, m: int, n: int, k: int) -> int:
    return _lib.nvfp4_workspace_bytes(op, m, n, k)


def nvfp4_amax(x, rows, k, ldx, amax_dev, stream=None) -> None:
    _check(_lib.nvfp4_amax(_p(x), rows, k, ldx, _p(amax_dev), _s(stream)), "nvfp4_amax")


def nvfp4_quantize(x, rows, k, ldx, codes, sf, layout, g_dev, amax_dev, amax_given=0, stream=None) -> None:
    _check(_lib.nvfp4_quantize(_p(x), rows, k, ldx, _p(codes), _p(sf), layout, _p(g_dev), _p(amax_dev),
                               int(amax_given), _s(stream)), "nvfp4_quantize")


def nvfp4_quantize_stochastic(x, rows, k, ldx, codes, sf, layout, g_dev, amax_dev, amax_given, seed, offset,
                              stream=None) -> None:
    _check(_lib.nvfp4_quantize_stochastic(_p(x), rows, k, ldx, _p(codes), _p(sf), layout, _p(g_dev), _p(amax_dev),
                                          int(amax_given), int(seed), int(offset), _s(stream)),
           "nvfp4_quantize_stochastic")


def nvfp4_quantize_hadamard(x, rows, k, ldx, order, codes, sf, layout, g_dev, amax_dev, amax_given=0,
                            stream=None) -> None:
    _check(_lib.nvfp4_quantize_hadamard(_p(x), rows, k, ldx, int(order), _p(codes), _p(sf), layout, _p(g_dev),
                                        _p(amax_dev), int(amax_given), _s(stream)), "nvfp4_quantize_hadamard")


def nvfp4_quantize_hadamard_stochastic(x, rows, k, ldx, order, codes, sf, layout, g_dev, amax_dev, amax_given,
                                       seed, offset, stream=None) -> None:
    _check(_lib.nvfp4_quantize_hadamard_stochastic(_p(x), rows, k, ldx, int(order), _p(codes), _p(sf), layout,
                                                   _p(g_dev), _p(amax_dev), int(amax_given), int(seed), int(offset),
                                                   _s(stream)), "nvfp4_quantize_hadamard_stochastic")


def nvfp4_swizzle_sf(sf_rowmajor, rows, k, sf_tc, stream=None) -> None:
    _check(_lib.nvfp4_swizzle_sf(_p(sf_rowmajor), rows, k, _p(sf_tc), _s(stream)), "nvfp4_swizzle_sf")


def nvfp4_gemm(a_codes, a_sf, g_a, b_codes, b_sf, g_b, m, n, k, d, ldd, out_dtype=OUT_BF16, stream=None) -> None:
    _check(_lib.nvfp4_gemm(_p(a_codes), _p(a_sf), _p(g_a), _p(b_codes), _p(b_sf), _p(g_b), m, n, k, _p(d), ldd,
                           out_dtype, _s(stream)), "nvfp4_gemm")


def nvfp4_gemm_fp8_out(a_codes, a_sf, g_a, b_codes, b_sf, g_b, m, n, k, g_d, d, ldd, amax_d=None,
                       stream=None) -> None:
    _check(_lib.nvfp4_gemm_fp8_out(_p(a_codes), _p(a_sf), _p(g_a), _p(b_codes), _p(b_sf), _p(g_b), m, n, k,
                                   _p(g_d), _p(d), ldd, _p(amax_d), _s(stream)), "nvfp4_gemm_fp8_out")


def nvfp4_gemm_requant(a_codes, a_sf, g_a, b_codes, b_sf, g_b, m, n, k, g_d, d_codes, ldd_bytes, d_sf, layout,
                       amax_d=None, stream=None) -> None:
    _check(_lib.nvfp4_gemm_requant(_p(a_codes), _p(a_sf), _p(g_a), _p(b_codes), _p(b_sf), _p(g_b), m, n, k,
                                   _p(g_d), _p(d_codes), ldd_bytes, _p(d_sf), layout, _p(amax_d), _s(stream)),
           "nvfp4_gemm_requant")


def nvfp4_gemv_batched(x, m, ldx, w_codes, w_sf, g_w, n, k, y, ldy, workspace, ws_bytes, stream=None) -> None:
    _check(_lib.nvfp4_gemv_batched(_p(x), m, ldx, _p(w_codes), _p(w_sf), _p(g_w), n, k, _p(y), ldy,
                                   _p(workspace), ws_bytes, _s(stream)), "nvfp4_gemv_batched")


def nvfp4_gemv_batched_noalloc(x, m, ldx, w_codes, w_sf, g_w, n, k, y, ldy, stream=None) -> None:
    """nvfp4_gemv_batched on the library's fixed scratch (no workspace argument)."""
    _check(_lib.nvfp4_gemv_batched_noalloc(_p(x), m, ldx, _p(w_codes), _p(w_sf), _p(g_w), n, k, _p(y), ldy,
                                           _s(stream)), "nvfp4_gemv_batched_noalloc")


def nvfp4_gemm_quant_a(a, lda, b_codes, b_sf, g_b, m, n, k, d, ldd, out_dtype, workspace, ws_bytes,
                       stream=None) -> None:
    _check(_lib.nvfp4_gemm_quant_a(_p(a), lda, _p(b_codes), _p(b_sf), _p(g_b), m, n, k, _p(d), ldd, out_dtype,
                                   _p(workspace), ws_bytes, _s(stream)), "nvfp4_gemm_quant_a")


def nvfp4_gemm_quant_a_prepare(a, lda, m, n, k, workspace, ws_bytes, stream=None) -> None:
    _check(_lib.nvfp4_gemm_quant_a_prepare(_p(a), lda, m, n, k, _p(workspace), ws_bytes, _s(stream)),
           "nvfp4_gemm_quant_a_prepare")


def nvfp4_gemm_quant_a_run(a, lda, b_codes, b_sf, g_b, m, n, k, d, ldd, out_dtype, workspace, ws_bytes,
                           stream=None) -> None:
    _check(_lib.nvfp4_gemm_quant_a_run(_p(a), lda, _p(b_codes), _p(b_sf), _p(g_b), m, n, k, _p(d), ldd, out_dtype,
                                       _p(workspace), ws_bytes, _s(stream)), "nvfp4_gemm_quant_a_run")


def nvfp4_gemm_quant_a_amax(a, lda, amax, b_codes, b_sf, g_b, m, n, k, d, ldd, out_dtype, workspace, ws_bytes,
                            stream=None) -> None:
    _check(_lib.nvfp4_gemm_quant_a_amax(_p(a), lda, _p(amax), _p(b_codes), _p(b_sf), _p(g_b), m, n, k, _p(d), ldd,
                                        out_dtype, _p(workspace), ws_bytes, _s(stream)), "nvfp4_gemm_quant_a_amax")


def nvfp4_mxfp4_sf_bytes(rows: int, k: int, layout: int) -> int:
    return _lib.nvfp4_mxfp4_sf_bytes(rows, k, layout)


def nvfp4_mxfp4_quantize(x, rows, k, ldx, codes, sf, layout, stream=None) -> None:
    _check(_lib.nvfp4_mxfp4_quantize(_p(x), rows, k, ldx, _p(codes), _p(sf), layout, _s(stream)),
           "nvfp4_mxfp4_quantize")


def nvfp4_mxfp4_gemm(a_codes, a_sf, b_codes, b_sf, m, n, k, d, ldd, out_dtype=OUT_BF16, stream=None) -> None:
    _check(_lib.nvfp4_mxfp4_gemm(_p(a_codes), _p(a_sf), _p(b_codes), _p(b_sf), m, n, k, _p(d), ldd, out_dtype,
                                 _s(stream)), "nvfp4_mxfp4_gemm")


def nvfp4_check_device_status(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status code."""
    return _lib.nvfp4_check_device_status(_s(stream))


def nvfp4_set_wait_limit_ns(limit_ns: int) -> None:
    _lib.nvfp4_set_wait_limit_ns(int(limit_ns))


def nvfp4_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(_lib.nvfp4_selftest_wait_timeout(int(limit_ns), _s(stream)), "nvfp4_selftest_wait_timeout")


def raw_status(name: str, *args) -> int:
    """Call a C entry point with raw arguments and return its status (for tests of argument checks)."""
    return getattr(_lib, name)(*args)


# ---------------------------------------------------------------------------
# allocation helpers (torch owns the memory; the work runs in the library)
# ---------------------------------------------------------------------------
class Quantized:
    """NVFP4 tensor: codes [rows, k/2] uint8, sf (layout bytes), g and amax (one fp32 each, on device)."""

    def __init__(self, codes, sf, g, amax, rows, k, layout):
        self.codes, self.sf, self.g, self.amax = codes, sf, g, amax
        self.rows, self.k, self.layout = rows, k, layout


def empty_quantized(rows: int, k: int, layout: int = SF_TCGEN05, device="cuda") -> Quantized:
    codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=device)
    sf = torch.empty(max(1, nvfp4_sf_bytes(rows, k, layout)), dtype=torch.uint8, device=device)
    scal = torch.empty(8, dtype=torch.float32, device=device)
    return Quantized(codes, sf, scal[0:1], scal[4:5], rows, k, layout)


def quantize(x: torch.Tensor, layout: int = SF_TCGEN05, out: Quantized | None = None, amax=None,
             stream=None) -> Quantized:
    """bf16 [rows, k] (row pitch x.stride(0)) -> NVFP4.  ``amax`` (device fp32) skips the amax pass."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    q = out if out is not None else empty_quantized(rows, k, layout, x.device)
    if amax is not None:
        q.amax.copy_(amax)
    nvfp4_quantize(x, rows, k, x.stride(0), q.codes, q.sf, layout, q.g, q.amax, 1 if amax is not None else 0,
                   stream)
    return q


def quantize_stochastic(x: torch.Tensor, seed: int, offset: int, layout: int = SF_TCGEN05,
                        out: Quantized | None = None, amax=None, stream=None) -> Quantized:
    """bf16 [rows, k] -> NVFP4 with stochastically rounded codes (Philox4x32-10 bits from seed, offset)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    q = out if out is not None else empty_quantized(rows, k, layout, x.device)
    if amax is not None:
        q.amax.copy_(amax)
    nvfp4_quantize_stochastic(x, rows, k, x.stride(0), q.codes, q.sf, layout, q.g, q.amax,
                              1 if amax is not None else 0, seed, offset, stream)
    return q


def quantize_hadamard(x: torch.Tensor, order: int, layout: int = SF_TCGEN05, out: Quantized | None = None,
                      amax=None, stream=None) -> Quantized:
    """bf16 [rows, k] -> NVFP4 of y = x H (block-diagonal Walsh-Hadamard of the given order over
    sqrt(order)).  ``amax`` (device fp32, max |y|) skips the amax pass."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    q = out if out is not None else empty_quantized(rows, k, layout, x.device)
    if amax is not None:
        q.amax.copy_(amax)
    nvfp4_quantize_hadamard(x, rows, k, x.stride(0), order, q.codes, q.sf, layout, q.g, q.amax,
                            1 if amax is not None else 0, stream)
    return q


def quantize_hadamard_stochastic(x: torch.Tensor, order: int, seed: int, offset: int, layout: int = SF_TCGEN05,
                                 out: Quantized | None = None, amax=None, stream=None) -> Quantized:
    """bf16 [rows, k] -> NVFP4 of y = x H with stochastically rounded codes."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    q = out if out is not None else empty_quantized(rows, k, layout, x.device)
    if amax is not None:
        q.amax.copy_(amax)
    nvfp4_quantize_hadamard_stochastic(x, rows, k, x.stride(0), order, q.codes, q.sf, layout, q.g, q.amax,
                                       1 if amax is not None else 0, seed, offset, stream)
    return q


def gemm(a: Quantized, b: Quantized, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
         stream=None) -> torch.Tensor:
    """D [M, N] = alpha (s_a A)(s_b B)^T for two TCGEN05-layout NVFP4 operands."""
    assert a.layout == SF_TCGEN05 and b.layout == SF_TCGEN05 and a.k == b.k
    od = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    d = out if out is not None else torch.empty((a.rows, b.rows), dtype=out_dtype, device=a.codes.device)
    nvfp4_gemm(a.codes, a.sf, a.g, b.codes, b.sf, b.g, a.rows, b.rows, a.k, d, d.stride(0), od, stream)
    return d


def gemm_requant(a: Quantized, b: Quantized, g_d: torch.Tensor, layout: int = SF_TCGEN05,
                 out: Quantized | None = None, stream=None) -> Quantized:
    """D = alpha (s_a A)(s_b B)^T quantized to NVFP4 under the given encode
    scale g_d (one fp32 on the device); out.amax receives max |D|."""
    assert a.layout == SF_TCGEN05 and b.layout == SF_TCGEN05 and a.k == b.k
    q = out if out is not None else empty_quantized(a.rows, b.rows, layout, a.codes.device)
    q.g.copy_(g_d.reshape(1))
    nvfp4_gemm_requant(a.codes, a.sf, a.g, b.codes, b.sf, b.g, a.rows, b.rows, a.k, q.g, q.codes,
                       q.codes.stride(0), q.sf, q.layout, q.amax, stream)
    return q


def gemm_fp8_out(a: Quantized, b: Quantized, g_d: torch.Tensor, out: torch.Tensor | None = None,
                 amax_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """FP8 (float8_e4m3fn) e4m3(v * g_d) for v = alpha (s_a A)(s_b B)^T; amax_out receives max |v|."""
    assert a.layout == SF_TCGEN05 and b.layout == SF_TCGEN05 and a.k == b.k
    d = out if out is not None else torch.empty((a.rows, b.rows), dtype=torch.float8_e4m3fn, device=a.codes.device)
    nvfp4_gemm_fp8_out(a.codes, a.sf, a.g, b.codes, b.sf, b.g, a.rows, b.rows, a.k, g_d, d, d.stride(0), amax_out,
                       stream)
    return d


def gemv_batched(x: torch.Tensor, w: Quantized, out: torch.Tensor | None = None, workspace=None,
                 stream=None) -> torch.Tensor:
    """y [M, N] for bf16 activations x [M, K] (M <= 32) and NVFP4 weights w [N, K]."""
    m, k = x.shape
    n = w.rows
    ws_bytes = nvfp4_workspace_bytes(OP_GEMV_BATCHED, m, n, k)
    ws = workspace if workspace is not None else torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    y = out if out is not None else torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    nvfp4_gemv_batched(x, m, x.stride(0), w.codes, w.sf, w.g, n, k, y, y.stride(0), ws, ws.numel(), stream)
    return y


def gemm_quant_a(a: torch.Tensor, b: Quantized, out_dtype=torch.bfloat16, out=None, workspace=None,
                 stream=None, amax: torch.Tensor | None = None) -> torch.Tensor:
    """D = A_q @ B_q^T with a bf16 A quantized inside the call; amax: A's tensor
    amax already on the device (1-element fp32), which skips the amax pass."""
    m, k = a.shape
    n = b.rows
    ws_bytes = nvfp4_workspace_bytes(OP_GEMM_QUANT_A, m, n, k)
    ws = workspace if workspace is not None else torch.empty(ws_bytes, dtype=torch.uint8, device=a.device)
    od = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    d = out if out is not None else torch.empty((m, n), dtype=out_dtype, device=a.device)
    if amax is None:
        nvfp4_gemm_quant_a(a, a.stride(0), b.codes, b.sf, b.g, m, n, k, d, d.stride(0), od, ws, ws.numel(), stream)
    else:
        nvfp4_gemm_quant_a_amax(a, a.stride(0), amax, b.codes, b.sf, b.g, m, n, k, d, d.stride(0), od, ws,
                                ws.numel(), stream)
    return d


def quant_a_workspace_views(ws: torch.Tensor, m: int, k: int):
    """A's codes [m, k/2], its tensor-core scales and g_a (1-element fp32) inside a
    gemm_quant_a workspace (the layout include/nvfp4.h states)."""
    codes_bytes = m * (k // 2)
    sf_off = (codes_bytes + 255) // 256 * 256
    sf_bytes = nvfp4_sf_bytes(m, k, SF_TCGEN05)
    g_off = sf_off + (sf_bytes + 255) // 256 * 256
    return (ws[:codes_bytes].view(m, k // 2), ws[sf_off:sf_off + sf_bytes],
            ws[g_off:g_off + 4].view(torch.float32))


class MXQuantized:
    """MXFP4 tensor: codes [rows, k/2] uint8 and E8M0 scales (layout bytes); no global scale."""

    def __init__(self, codes, sf, rows, k, layout):
        self.codes, self.sf = codes, sf
        self.rows, self.k, self.layout = rows, k, layout


def mxfp4_quantize(x: torch.Tensor, layout: int = SF_TCGEN05, out: MXQuantized | None = None,
                   stream=None) -> MXQuantized:
    """bf16 [rows, k] (row pitch x.stride(0)) -> MXFP4 (one pass)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, k = x.shape
    if out is None:
        codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=x.device)
        sf = torch.empty(max(1, nvfp4_mxfp4_sf_bytes(rows, k, layout)), dtype=torch.uint8, device=x.device)
        out = MXQuantized(codes, sf, rows, k, layout)
    nvfp4_mxfp4_quantize(x, rows, k, x.stride(0), out.codes, out.sf, layout, stream)
    return out


def mxfp4_gemm(a: MXQuantized, b: MXQuantized, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """D [M, N] = (s_a A)(s_b B)^T for two TCGEN05-layout MXFP4 operands."""
    assert a.layout == SF_TCGEN05 and b.layout == SF_TCGEN05 and a.k == b.k
    od = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    d = out if out is not None else torch.empty((a.rows, b.rows), dtype=out_dtype, device=a.codes.device)
    nvfp4_mxfp4_gemm(a.codes, a.sf, b.codes, b.sf, a.rows, b.rows, a.k, d, d.stride(0), od, stream)
    return d
