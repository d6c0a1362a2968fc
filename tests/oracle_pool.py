"""The oracle on whole full-size tensors, spread over the host cores.

Test infrastructure: used only by the full-size parity tests.  Nothing here
computes anything itself; it calls the oracle on pieces of a problem that the
oracle's definition makes independent:
  * quantization: once the global scale g is known (``O.amax`` and
    ``O.global_scale`` on the WHOLE tensor, in the calling process), every
    row's codes and block scales depend on that row alone, so workers run
    ``O.quantize_with_scale`` and ``O.pack_codes`` on slices of rows;
  * GEMM reference: each output column D[:, n] depends on weight row n only,
    so ``O.gemm_ref`` runs on slices of the weight rows and the slices of D
    and S are placed side by side;
  * stochastic rounding: given g, a row's codes depend on that row and on
    random integers that the oracle draws by the row's index (``row_ids``),
    so ``S.quantize_sr`` runs on slices of rows with their indices;
  * the rotated quantizer: the transform works inside a row, so the amax of
    y is the largest of the slices' maxima (``H.fwht_f32`` on each slice),
    and, given it, ``H.quantize_hadamard`` / ``H.quantize_hadamard_sr`` run
    on slices of rows;
  * MXFP4 (no global scale): rows quantize independently and each output
    column depends on one weight row, as for NVFP4.
Workers are started with ``spawn`` (safe after the process has used CUDA).
"""
from __future__ import annotations

import os

import numpy as np

from oracle import hadamard_oracle as H
from oracle import mxfp4_oracle as MX
from oracle import nvfp4_oracle as O
from oracle import stochastic_oracle as S

_ROWS_PER_TASK = 1024


def _workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _quantize_rows(kind, shm_in, shm_codes, shm_sf, rows, k, sf_block, params, r0, r1):
    """Codes and row-major scales of rows r0 .. r1 - 1 by the oracle function
    that ``kind`` names, the whole tensor's scale parameters given."""
    from multiprocessing import shared_memory
    si = shared_memory.SharedMemory(name=shm_in)
    sc = shared_memory.SharedMemory(name=shm_codes)
    ss = shared_memory.SharedMemory(name=shm_sf)
    try:
        x = np.ndarray((rows, k), dtype=np.uint16, buffer=si.buf)
        codes = np.ndarray((rows, k // 2), dtype=np.uint8, buffer=sc.buf)
        sf = np.ndarray((rows, k // sf_block), dtype=np.uint8, buffer=ss.buf)
        ids = np.arange(r0, r1)
        if kind == "nvfp4":
            (g,) = params
            c, s = O.quantize_with_scale(x[r0:r1], g)
            c = O.pack_codes(c)
        elif kind == "sr":
            a, seed, offset = params
            c, s, _, _ = S.quantize_sr(x[r0:r1], seed, offset, amax_value=a, row_ids=ids)
        elif kind == "hadamard":
            a, order = params
            c, s, _, _ = H.quantize_hadamard(x[r0:r1], order, amax_value=a)
        elif kind == "mx":
            c, s = MX.quantize_mx(x[r0:r1])
        elif kind == "hadamard_sr":
            a, order, seed, offset = params
            c, s, _, _ = H.quantize_hadamard_sr(x[r0:r1], order, seed, offset, amax_value=a, row_ids=ids)
        else:
            raise ValueError(kind)
        codes[r0:r1] = c
        sf[r0:r1] = s
        del x, codes, sf
    finally:
        si.close()
        sc.close()
        ss.close()


def _rotated_amax_rows(shm_in, rows, k, order, r0, r1):
    from multiprocessing import shared_memory
    si = shared_memory.SharedMemory(name=shm_in)
    try:
        x = np.ndarray((rows, k), dtype=np.uint16, buffer=si.buf)
        y = H.fwht_f32(O.bf16_to_f32(x[r0:r1]), order)
        m = np.float32(np.max(np.abs(y))) if y.size else np.float32(0.0)
        del x
        return m
    finally:
        si.close()


def _pool():
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    return ProcessPoolExecutor(max_workers=_workers(), mp_context=mp.get_context("spawn"))


def _by_rows(x_bits: np.ndarray, kind: str, params: tuple, sf_block: int = 16):
    """(packed codes [rows, k/2], row-major scales [rows, k/sf_block]) of the
    whole tensor, computed slice by slice."""
    from multiprocessing import shared_memory
    rows, k = x_bits.shape
    shms = [shared_memory.SharedMemory(create=True, size=max(1, n))
            for n in (x_bits.nbytes, rows * k // 2, rows * k // sf_block)]
    try:
        np.ndarray(x_bits.shape, dtype=np.uint16, buffer=shms[0].buf)[:] = x_bits
        with _pool() as ex:
            futs = [ex.submit(_quantize_rows, kind, shms[0].name, shms[1].name, shms[2].name, rows, k, sf_block,
                              params, r0, min(rows, r0 + _ROWS_PER_TASK))
                    for r0 in range(0, rows, _ROWS_PER_TASK)]
            for f in futs:
                f.result()
        codes = np.ndarray((rows, k // 2), dtype=np.uint8, buffer=shms[1].buf).copy()
        sf = np.ndarray((rows, k // sf_block), dtype=np.uint8, buffer=shms[2].buf).copy()
        return codes, sf
    finally:
        for s in shms:
            s.close()
            s.unlink()


def _small(x_bits: np.ndarray) -> bool:
    return x_bits.shape[0] <= _ROWS_PER_TASK or _workers() == 1


def quantize(x_bits: np.ndarray):
    """Same result as ``O.quantize(x_bits)``: (packed codes, row-major scales, g, amax)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    a = O.amax(x_bits)
    g = O.global_scale(a)
    if _small(x_bits):
        c, s = O.quantize_with_scale(x_bits, g)
        return O.pack_codes(c), s, g, a
    codes, sf = _by_rows(x_bits, "nvfp4", (g,))
    return codes, sf, g, a


def quantize_sr(x_bits: np.ndarray, seed: int, offset: int):
    """Same result as ``S.quantize_sr(x_bits, seed, offset)``."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if _small(x_bits):
        return S.quantize_sr(x_bits, seed, offset)
    a = O.amax(x_bits)
    codes, sf = _by_rows(x_bits, "sr", (a, seed, offset))
    return codes, sf, O.global_scale(a), a


def rotated_amax(x_bits: np.ndarray, order: int) -> np.float32:
    """max |x H| over the whole tensor, as ``H.quantize_hadamard`` takes it."""
    from multiprocessing import shared_memory
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, k = x_bits.shape
    if _small(x_bits):
        y = H.fwht_f32(O.bf16_to_f32(x_bits), order)
        return np.float32(np.max(np.abs(y))) if y.size else np.float32(0.0)
    shm = shared_memory.SharedMemory(create=True, size=max(1, x_bits.nbytes))
    try:
        np.ndarray(x_bits.shape, dtype=np.uint16, buffer=shm.buf)[:] = x_bits
        with _pool() as ex:
            futs = [ex.submit(_rotated_amax_rows, shm.name, rows, k, order, r0, min(rows, r0 + _ROWS_PER_TASK))
                    for r0 in range(0, rows, _ROWS_PER_TASK)]
            return np.float32(max(f.result() for f in futs))
    finally:
        shm.close()
        shm.unlink()


def quantize_hadamard(x_bits: np.ndarray, order: int):
    """Same result as ``H.quantize_hadamard(x_bits, order)``."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if _small(x_bits):
        return H.quantize_hadamard(x_bits, order)
    a = rotated_amax(x_bits, order)
    codes, sf = _by_rows(x_bits, "hadamard", (a, order))
    return codes, sf, O.global_scale(a), a


def quantize_hadamard_sr(x_bits: np.ndarray, order: int, seed: int, offset: int):
    """Same result as ``H.quantize_hadamard_sr(x_bits, order, seed, offset)``."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if _small(x_bits):
        return H.quantize_hadamard_sr(x_bits, order, seed, offset)
    a = rotated_amax(x_bits, order)
    codes, sf = _by_rows(x_bits, "hadamard_sr", (a, order, seed, offset))
    return codes, sf, O.global_scale(a), a


def quantize_mx(x_bits: np.ndarray):
    """Same result as ``MX.quantize_mx(x_bits)``: (packed codes, E8M0 scales)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if _small(x_bits):
        return MX.quantize_mx(x_bits)
    return _by_rows(x_bits, "mx", (), sf_block=MX.MX_BLOCK)


def gemm_ref_mx(a_packed, a_sf, b_packed, b_sf, cols_per_slice: int = 2048):
    """Same result as ``MX.gemm_ref_mx`` (D, S), over slices of B's rows."""
    n = b_packed.shape[0]
    ds, ss = [], []
    for c0 in range(0, n, cols_per_slice):
        d, s = MX.gemm_ref_mx(a_packed, a_sf, b_packed[c0:c0 + cols_per_slice], b_sf[c0:c0 + cols_per_slice])
        ds.append(d)
        ss.append(s)
    return np.concatenate(ds, axis=1), np.concatenate(ss, axis=1)


def gemm_ref(a_packed, a_sf, g_a, b_packed, b_sf, g_b, cols_per_slice: int = 2048):
    """Same result as ``O.gemm_ref`` (D, S, alpha), over slices of B's rows."""
    n = b_packed.shape[0]
    ds, ss = [], []
    alpha = None
    for c0 in range(0, n, cols_per_slice):
        d, s, alpha = O.gemm_ref(a_packed, a_sf, g_a, b_packed[c0:c0 + cols_per_slice],
                                 b_sf[c0:c0 + cols_per_slice], g_b)
        ds.append(d)
        ss.append(s)
    return np.concatenate(ds, axis=1), np.concatenate(ss, axis=1), alpha
