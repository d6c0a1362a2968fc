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
    and S are placed side by side.
Workers are started with ``spawn`` (safe after the process has used CUDA).
"""
from __future__ import annotations

import os

import numpy as np

from oracle import nvfp4_oracle as O

_ROWS_PER_TASK = 1024


def _workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _quantize_rows(shm_in, shm_codes, shm_sf, rows, k, g, r0, r1):
    from multiprocessing import shared_memory
    si = shared_memory.SharedMemory(name=shm_in)
    sc = shared_memory.SharedMemory(name=shm_codes)
    ss = shared_memory.SharedMemory(name=shm_sf)
    try:
        x = np.ndarray((rows, k), dtype=np.uint16, buffer=si.buf)
        codes = np.ndarray((rows, k // 2), dtype=np.uint8, buffer=sc.buf)
        sf = np.ndarray((rows, k // 16), dtype=np.uint8, buffer=ss.buf)
        c, s = O.quantize_with_scale(x[r0:r1], g)
        codes[r0:r1] = O.pack_codes(c)
        sf[r0:r1] = s
        del x, codes, sf
    finally:
        si.close()
        sc.close()
        ss.close()


def quantize(x_bits: np.ndarray):
    """Same result as ``O.quantize(x_bits)``: (packed codes, row-major scales, g, amax)."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    from multiprocessing import shared_memory

    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, k = x_bits.shape
    a = O.amax(x_bits)
    g = O.global_scale(a)
    if rows <= _ROWS_PER_TASK or _workers() == 1:
        c, s = O.quantize_with_scale(x_bits, g)
        return O.pack_codes(c), s, g, a
    shms = [shared_memory.SharedMemory(create=True, size=max(1, n))
            for n in (x_bits.nbytes, rows * k // 2, rows * k // 16)]
    try:
        np.ndarray(x_bits.shape, dtype=np.uint16, buffer=shms[0].buf)[:] = x_bits
        with ProcessPoolExecutor(max_workers=_workers(), mp_context=mp.get_context("spawn")) as ex:
            futs = [ex.submit(_quantize_rows, shms[0].name, shms[1].name, shms[2].name, rows, k, g,
                              r0, min(rows, r0 + _ROWS_PER_TASK))
                    for r0 in range(0, rows, _ROWS_PER_TASK)]
            for f in futs:
                f.result()
        codes = np.ndarray((rows, k // 2), dtype=np.uint8, buffer=shms[1].buf).copy()
        sf = np.ndarray((rows, k // 16), dtype=np.uint8, buffer=shms[2].buf).copy()
        return codes, sf, g, a
    finally:
        for s in shms:
            s.close()
            s.unlink()


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
