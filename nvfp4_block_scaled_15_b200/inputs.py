"""Seeded synthetic inputs for the NVFP4 workloads.

This module is the only code shared by the CUDA path's tests/benchmarks and
the CPU oracle.  It holds no NVFP4 arithmetic: it only draws random numbers
and rounds them to bf16.

Generator (counter based, so any slice can be regenerated independently):
  * splitmix64 of ``seed_word + (i + 1) * 0x9E3779B97F4A7C15`` gives 64 random
    bits for counter ``i``;
  * the top 53 bits give a uniform in (0, 1);
  * Box-Muller (cosine branch) turns two independent uniform streams into one
    standard normal;
  * the fp64 value is rounded to bf16 with round-to-nearest-even.

Workload shapes follow the pages' LLM-inference use (activations with a few
outlier channels, small-variance weights, SiLU-gated FFN activations); the
recipes are listed per function below.
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _seed_word(seed: int, stream: int) -> np.uint64:
    # distinct streams of one seed start from distinct splitmix64 states
    base = np.array([np.uint64(seed & 0xFFFFFFFFFFFFFFFF)], dtype=np.uint64)
    return _mix(base ^ np.uint64((0xD1B54A32D192ED03 * (stream + 1)) & 0xFFFFFFFFFFFFFFFF))[0]


def uniform01(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Uniforms in (0, 1) for counters ``start .. start+count-1`` (fp64)."""
    with np.errstate(over="ignore"):
        ctr = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = _mix(_seed_word(seed, stream) + ctr * _GOLDEN)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, start: int, count: int, stream: int = 0) -> np.ndarray:
    """Standard normals (fp64) for counters ``start .. start+count-1``."""
    u1 = uniform01(seed, 2 * stream, start, count)
    u2 = uniform01(seed, 2 * stream + 1, start, count)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def _f64_to_bf16_slow(x: np.ndarray) -> np.ndarray:
    mant, exp = np.frexp(x)                     # x = mant * 2**exp, 0.5 <= |mant| < 1
    exp = np.maximum(exp, -125)                 # bf16 subnormal quantum is 2**-133
    q = np.rint(np.ldexp(x, 8 - exp))           # 8 significant bits, ties to even
    with np.errstate(over="ignore"):
        y = np.ldexp(q, exp - 8).astype(np.float32)  # exact: y has <= 8 significant bits
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 (round-to-nearest-even, one rounding), as uint16 bits.

    Works on the fp64 bit pattern: keep 7 of the 52 fraction bits, round the
    other 45 to nearest-even, re-bias the exponent.  Values outside the bf16
    normal range (zero, subnormal, overflow) take a frexp-based path.
    """
    v = np.ascontiguousarray(v, dtype=np.float64)
    bits = v.view(np.uint64)
    sign = (bits >> np.uint64(63)).astype(np.uint16)
    exp = ((bits >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    frac = bits & np.uint64((1 << 52) - 1)
    keep = (frac >> np.uint64(45)).astype(np.int64)
    rest = frac & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rest > half) | ((rest == half) & ((keep & 1) == 1))
    keep = keep + up
    exp = exp + (keep >> 7)
    keep = keep & 127
    bexp = exp - 1023 + 127
    out = ((sign << np.uint16(15)) | (np.clip(bexp, 0, 255).astype(np.uint16) << np.uint16(7))
           | keep.astype(np.uint16))
    odd = (bexp <= 0) | (bexp >= 255)
    if np.any(odd):
        out[odd] = _f64_to_bf16_slow(v[odd])
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bits -> fp32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# Chunked generation.  Every element depends only on (seed, stream, index),
# so chunks can be produced in any order, serially or by a process pool.
# ---------------------------------------------------------------------------
_PARALLEL_MIN = 1 << 24        # elements; smaller tensors are generated serially


def _chunk_values(kind: str, params: tuple, start: int, count: int) -> np.ndarray:
    if kind == "gauss":
        seed, std, stream = params
        return f64_to_bf16_bits(std * normal(seed, start, count, stream))
    if kind == "outlier":
        seed, k, cols, factor = params
        z = normal(seed, start, count)
        is_out = np.zeros(k, dtype=bool)
        is_out[cols] = True
        col = np.arange(start, start + count, dtype=np.int64) % k
        z = np.where(is_out[col], z * factor, z)
        return f64_to_bf16_bits(z)
    if kind == "silu":
        seed_a, seed_b = params
        a = normal(seed_a, start, count).astype(np.float32)
        b = normal(seed_b, start, count).astype(np.float32)
        silu = b / (np.float32(1.0) + np.exp(-b))
        return f64_to_bf16_bits((a * silu).astype(np.float64))
    raise ValueError(kind)


def _worker_fill(shm_name: str, n: int, kind: str, params: tuple, start: int, count: int) -> None:
    from multiprocessing import shared_memory
    shm = shared_memory.SharedMemory(name=shm_name)
    try:
        out = np.ndarray((n,), dtype=np.uint16, buffer=shm.buf)
        out[start:start + count] = _chunk_values(kind, params, start, count)
        del out
    finally:
        shm.close()


def _generate(kind: str, params: tuple, n: int) -> np.ndarray:
    import os
    workers = int(os.environ.get("NVFP4_GEN_WORKERS", "0")) or min(32, os.cpu_count() or 1)
    if n < _PARALLEL_MIN or workers <= 1:
        out = np.empty(n, dtype=np.uint16)
        for s in range(0, n, _CHUNK):
            c = min(_CHUNK, n - s)
            out[s:s + c] = _chunk_values(kind, params, s, c)
        return out
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    from multiprocessing import shared_memory
    shm = shared_memory.SharedMemory(create=True, size=max(2, 2 * n))
    try:
        with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
            futs = [ex.submit(_worker_fill, shm.name, n, kind, params, s, min(_CHUNK, n - s))
                    for s in range(0, n, _CHUNK)]
            for f in futs:
                f.result()
        return np.ndarray((n,), dtype=np.uint16, buffer=shm.buf).copy()
    finally:
        shm.close()
        shm.unlink()


def gaussian_bf16(shape, seed: int, std: float = 1.0, stream: int = 0) -> np.ndarray:
    """bf16 bits of ``std * N(0, 1)`` in row-major ``shape``."""
    n = int(np.prod(shape))
    return _generate("gauss", (seed, float(std), stream), n).reshape(shape)


def outlier_columns(k: int, fraction: float, seed: int) -> np.ndarray:
    """Indices of ``round(fraction * k)`` columns chosen by a seeded Fisher-Yates shuffle."""
    n_out = int(round(fraction * k))
    perm = np.arange(k, dtype=np.int64)
    u = uniform01(seed, 97, 0, k)
    for i in range(k - 1, 0, -1):                   # classic Fisher-Yates, uniform j in [0, i]
        j = int(u[i] * (i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:n_out])


def activations_with_outliers(rows: int, k: int, seed: int, fraction: float,
                              factor: float) -> np.ndarray:
    """bf16 bits of N(0,1) activations whose outlier channels are scaled by ``factor``.

    The outlier columns are multiplied in fp64 before the single bf16 rounding.
    """
    cols = outlier_columns(k, fraction, seed)
    return _generate("outlier", (seed, k, cols, float(factor)), rows * k).reshape(rows, k)


def silu_gated_bf16(rows: int, k: int, seed_a: int, seed_b: int) -> np.ndarray:
    """bf16 bits of ``a * silu(b)`` with a, b ~ N(0,1); silu evaluated in fp32."""
    return _generate("silu", (seed_a, seed_b), rows * k).reshape(rows, k)


# --------------------------------------------------------------------------
# The five workloads (shapes, distributions and seeds)
# --------------------------------------------------------------------------
def tiny_end_to_end():
    """A bf16 [128,256] N(0,1) seed 1; W bf16 [256,256] N(0,1) seed 2."""
    return gaussian_bf16((128, 256), seed=1), gaussian_bf16((256, 256), seed=2)


def quantize_bandwidth(rows: int = 16384, k: int = 8192):
    """X bf16 [16384,8192] N(0,1) seed 3, 1% of columns x50 (outlier channels)."""
    return activations_with_outliers(rows, k, seed=3, fraction=0.01, factor=50.0)


def prefill_gemm(m: int = 8192, n: int = 8192, k: int = 8192):
    """A bf16 [8192,8192] N(0,1), 0.5% columns x30, seed 4; W bf16 [8192,8192] N(0,0.02) seed 5."""
    a = activations_with_outliers(m, k, seed=4, fraction=0.005, factor=30.0)
    w = gaussian_bf16((n, k), seed=5, std=0.02)
    return a, w


def decode_gemv(m: int, n: int = 28672, k: int = 8192):
    """W bf16 [28672,8192] N(0,0.02) seed 6; x bf16 [M,8192] N(0,1) seed 7."""
    w = gaussian_bf16((n, k), seed=6, std=0.02)
    x = gaussian_bf16((m, k), seed=7)
    return x, w


def long_k(m: int = 4096, n: int = 8192, k: int = 28672):
    """A bf16 [4096,28672] = a*silu(b), seeds 8/9; W bf16 [8192,28672] N(0,0.02) seed 10."""
    a = silu_gated_bf16(m, k, seed_a=8, seed_b=9)
    w = gaussian_bf16((n, k), seed=10, std=0.02)
    return a, w
