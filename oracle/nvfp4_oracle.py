"""NVFP4 oracle: a plain, slow, CPU statement of what the NVFP4 hot path computes.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
The library (``nvfp4_block_scaled_15_b200``) never imports it and has no CPU
fallback.  This file shares no code, table or constant with the CUDA path.

Pages cited (titles as printed; sections are the pages' own headings):
  [P1] "NVIDIA NVFP4 与 Micro-Scaling：Blackwell 推理 4-bit 浮点精度的深度工程实战" (ybb.press)
  [P2] "mxFP4/nvFP4 最小化知识" (10100.com)
  [P3] "Introducing NVFP4 for Efficient and Accurate Low-Precision Inference" (developer.nvidia.cn)
  [P4] "low-precision-floats" (july-h5kf3.github.io), section "FP4 / MXFP4 / NVFP4"
  [P5] "FP4" encyclopedia entry (newton.com.tw), section "技術原理"

Definition (fp32 operation order is part of the definition):
  1. amax = max |x| over the whole tensor (bf16 -> fp32 is exact)       [P1 §三 step 1; P4 NVFP4]
  2. g = 2688 / amax in fp32 (2688 = 6 * 448); g = 1 when amax == 0     [P4 NVFP4: s_global = amax/(6*448), g = 1/s_global]
  3. per 16 consecutive elements along K: ab = max |x|;
     s = e4m3_rne_satfinite((ab * g) / 6); sd = decode(s)              [P4 NVFP4: s_block = (block_amax/6)/s_global; P2 高精度scale]
  4. per element: code = e2m1_rne_sat((x * g) / sd); code = 0 if sd == 0 [P4 NVFP4: x_hat = s_nv * Q_E2M1(x / s_nv)]
  5. pack two codes per byte, first element in the low nibble            [P5 技術原理: ONNX FLOAT4E2M1 packing]
  6. D = alpha * (s_a (.) A)(s_b (.) W)^T with alpha = 1 / (g_a * g_b) in fp32,
     accumulated here in fp64                                            [P1 §三 scaled GEMM; P4 mixed-precision MMA]
  7. output scale g_d (optional outputs of the GEMM)                    [P1 §三: D = g_d * (...), "output dequant by g_d",
     v = fp32(alpha * acc) is the value the fp32 output holds;           the _scaled_mm example: scale_result=g_d,
     FP8 output: e4m3_rne_satfinite(fp32(v * g_d)), sign kept;           out_dtype=float8_e4m3fn]
     NVFP4 output: steps 3-5 on v with g := g_d (g_d is the output's
     encode scale, given by the caller); amax_d = max |v|

Where the pages are silent or disagree, each function below states the
reading it takes.

Pins (tests/test_oracle_pins.py) tie every function to the pages or to
mathematics outside this file.  ``swizzle_sf_tcgen05`` is a data layout the
pages do not describe: parity unpinned by the pages; it is pinned only on
hardware, by GEMMs whose result must equal ``gemm_ref`` computed from the
row-major scales.
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# Formats
# --------------------------------------------------------------------------
# E2M1 magnitudes for codes 0..7; code | 8 is the negative [P1 §二 value table;
# P2 "nvFP4的数据结构设计"; P4 "FP4 / MXFP4 / NVFP4"; P5 技術原理].
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0      # [P1 §二: "最大值只有 6.0"]
E4M3_MAX = 448.0    # [P4 NVFP4: "448 是 E4M3 的最大可表示值"]
BLOCK = 16          # elements per block scale along K [P1 §3.1; P3 "微块"; P5 技術原理]


class RangeError(ValueError):
    """The global scale 2688/amax is not a finite fp32 number."""


def e2m1_decode(codes) -> np.ndarray:
    """fp64 value of 4-bit E2M1 codes (sign in bit 3; -0 for code 8)."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def e2m1_encode(u) -> np.ndarray:
    """Round fp32 values to E2M1 codes: nearest magnitude, ties to the even code,
    magnitudes beyond 6 saturate to 6 [north_star "e2m1_rne_sat"].

    The sign bit follows the sign bit of ``u`` (so -0.1 gives code 8, "-0"), as
    the pages list -0 among the 16 values [P2; P1 §二].
    """
    u = np.asarray(u, dtype=np.float32)
    a = np.abs(u).astype(np.float64)
    lo = np.clip(np.searchsorted(E2M1_MAGNITUDES, a, side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    d_lo = a - E2M1_MAGNITUDES[lo]
    d_hi = E2M1_MAGNITUDES[hi] - a
    take_hi = (hi != lo) & ((d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0)))
    code = np.where(take_hi, hi, lo).astype(np.uint8)
    return code | np.where(np.signbit(u), np.uint8(8), np.uint8(0))


def e4m3_decode(b) -> np.ndarray:
    """fp32 value of E4M3 (float8_e4m3fn) bytes: bias 7, subnormals m*2^-9,
    0x7F/0xFF are NaN, no infinities."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 15
    m = b & 7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return np.where(s == 1, -val, val).astype(np.float32)


# the 127 non-negative finite E4M3 values, increasing with the code 0x00..0x7E
_E4M3_POS = e4m3_decode(np.arange(127)).astype(np.float64)


def e4m3_encode_satfinite(s) -> np.ndarray:
    """Round non-negative fp32 values to E4M3 bytes: nearest value, ties to the
    even code (even mantissa), values at or above 448 give 448 (0x7E)."""
    a = np.asarray(s, dtype=np.float32).astype(np.float64)
    if np.any(a < 0) or not np.all(np.isfinite(a)):
        raise ValueError("block scales are finite and non-negative by construction")
    lo = np.clip(np.searchsorted(_E4M3_POS, a, side="right") - 1, 0, 126)
    hi = np.minimum(lo + 1, 126)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    take_hi = (hi != lo) & ((d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0)))
    return np.where(take_hi, hi, lo).astype(np.uint8)


def bf16_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f64_to_bf16_rne(v) -> np.ndarray:
    """fp64 -> bf16 bits, a single round-to-nearest-even (overflow gives +-inf)."""
    v = np.asarray(v, dtype=np.float64)
    mant, exp = np.frexp(v)
    exp = np.maximum(exp, -125)
    q = np.rint(np.ldexp(v, 8 - exp))
    with np.errstate(over="ignore"):
        y = np.ldexp(q, exp - 8).astype(np.float32)
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# Quantization [P4 NVFP4 formulas; P1 §三 two-level scaling; P3 two-level strategy]
# --------------------------------------------------------------------------
def amax(x_bits) -> np.float32:
    """max |x| over the tensor, x given as bf16 bits."""
    x = bf16_to_f32(x_bits)
    return np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)


def global_scale(a) -> np.float32:
    """g = 2688 / amax in fp32 (encode direction: g = 1/s_global, s_global =
    amax/(6*448) [P4 NVFP4]).  amax == 0 gives g = 1 (pages silent).  A
    non-finite amax or g is an error (pages silent: the tensor has no
    finite two-level encoding)."""
    a = np.float32(a)
    if not np.isfinite(a):
        raise RangeError(f"amax is not finite ({float(a)!r})")
    if a == 0:
        return np.float32(1.0)
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        g = np.float32(2688.0) / a
    if not np.isfinite(g):
        raise RangeError(f"2688/amax is not finite for amax={float(a)!r}")
    return np.float32(g)


def quantize_with_scale(x_bits, g):
    """Steps 3-4 for a [rows, K] bf16 tensor and a given fp32 global scale g.

    Returns (codes [rows, K] uint8, one code per element, unpacked;
             sf [rows, K/16] uint8 E4M3 block scales, row-major).
    """
    return quantize_values_with_scale(bf16_to_f32(x_bits), g)


def quantize_values_with_scale(x, g):
    """Steps 3-4 for fp32 values x [rows, K] (any fp32, not only bf16 ones) and
    a given fp32 encode scale g; the same returns as quantize_with_scale."""
    x = np.asarray(x, dtype=np.float32)
    rows, k = x.shape
    if k % BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = np.float32(g)
    xb = x.reshape(rows, k // BLOCK, BLOCK)
    ab = np.max(np.abs(xb), axis=2)                                     # exact
    s_raw = (ab * g).astype(np.float32) / np.float32(6.0)               # two fp32 RN ops
    sf = e4m3_encode_satfinite(s_raw.astype(np.float32))
    sd = e4m3_decode(sf)
    t = (xb * g).astype(np.float32)                                     # fp32 RN
    zero_scale = (sd == 0)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.where(zero_scale, np.float32(0.0), t / np.where(zero_scale, np.float32(1.0), sd[:, :, None]))
    codes = e2m1_encode(u.astype(np.float32))
    codes = np.where(np.broadcast_to(zero_scale, codes.shape), np.uint8(0), codes)
    return codes.reshape(rows, k).astype(np.uint8), sf.astype(np.uint8)


def pack_codes(codes) -> np.ndarray:
    """Two 4-bit codes per byte, first element in the low nibble [P5 技術原理]."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


def quantize(x_bits, amax_value=None):
    """bf16 [rows, K] -> (packed codes [rows, K/2], sf [rows, K/16], g, amax).

    ``amax_value`` replaces step 1 when given (a caller-supplied amax).
    Raises RangeError when g is not finite.
    """
    a = amax(x_bits) if amax_value is None else np.float32(amax_value)
    g = global_scale(a)
    codes, sf = quantize_with_scale(x_bits, g)
    return pack_codes(codes), sf, g, a


def dequantize_blocks(packed, sf) -> np.ndarray:
    """s (.) q: E2M1 value times its decoded block scale, fp64, without the
    global scale (the GEMM folds 1/g into alpha) [P1 §三 scaled GEMM]."""
    q = e2m1_decode(unpack_codes(packed))
    rows, k = q.shape
    sd = e4m3_decode(sf).astype(np.float64)
    return (q.reshape(rows, k // BLOCK, BLOCK) * sd[:, :, None]).reshape(rows, k)


def dequantize(packed, sf, g) -> np.ndarray:
    """x_hat = s_global * s_block * q with s_global = 1/g [P4 NVFP4; P1 §三 还原]."""
    return dequantize_blocks(packed, sf) / np.float64(np.float32(g))


# --------------------------------------------------------------------------
# Block-scaled GEMM [P1 §三 scaled GEMM, §五 kernel data layout; P4 mixed-precision MMA]
# --------------------------------------------------------------------------
def gemm_alpha(g_a, g_b) -> np.float32:
    """alpha = 1 / (g_a * g_b), two fp32 RN operations."""
    return np.float32(np.float32(1.0) / (np.float32(g_a) * np.float32(g_b)))


def gemm_ref(a_packed, a_sf, g_a, b_packed, b_sf, g_b):
    """D = alpha * (s_a (.) A)(s_b (.) B)^T in fp64, plus S = sum_k |a_k b_k|.

    A is [M, K] and B is [N, K], both K-major.  Returns (D, S, alpha) with D and
    S of shape [M, N] (S without alpha).  The fp64 products of E2M1 values and
    E4M3 scales are exact; only the fp64 summation rounds (<= K * 2^-53 * S).
    """
    ad = dequantize_blocks(a_packed, a_sf)
    bd = dequantize_blocks(b_packed, b_sf)
    alpha = gemm_alpha(g_a, g_b)
    d = np.float64(alpha) * (ad @ bd.T)
    s = np.abs(ad) @ np.abs(bd).T
    return d, s, alpha


def gemm_ref_entries(a_packed, a_sf, g_a, b_packed, b_sf, g_b, rows, cols):
    """D[rows[i], cols[i]] and S for a list of output coordinates, one dot product each."""
    alpha = gemm_alpha(g_a, g_b)
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    d = np.empty(rows.size)
    s = np.empty(rows.size)
    for i, (r, c) in enumerate(zip(rows, cols)):
        ar = dequantize_blocks(a_packed[r:r + 1], a_sf[r:r + 1])[0]
        bc = dequantize_blocks(b_packed[c:c + 1], b_sf[c:c + 1])[0]
        d[i] = np.float64(alpha) * np.dot(ar, bc)
        s[i] = np.dot(np.abs(ar), np.abs(bc))
    return d, s, alpha


# --------------------------------------------------------------------------
# Output scale g_d [P1 §三: D = g_d * ((g_a s_a A)(g_b s_b W)), "输出反量化由
# g_d 完成（输出常以 FP8/FP16 落盘）", and the _scaled_mm example with
# scale_result=g_d, out_dtype=torch.float8_e4m3fn]
# --------------------------------------------------------------------------
def e4m3_encode_signed_satfinite(v) -> np.ndarray:
    """Signed fp32 values -> E4M3 bytes: the magnitude as e4m3_encode_satfinite
    (nearest, ties to the even code, >= 448 gives 448), the sign in bit 7
    (-0 gives 0x80)."""
    v = np.asarray(v, dtype=np.float32)
    if not np.all(np.isfinite(v)):
        raise ValueError("output values are finite")
    mag = e4m3_encode_satfinite(np.abs(v))
    return (mag | (np.signbit(v).astype(np.uint8) << 7)).astype(np.uint8)


def fp8_output(v, g_d) -> np.ndarray:
    """FP8 output bytes: e4m3_rne_satfinite(fp32(v * g_d))."""
    t = (np.asarray(v, dtype=np.float32) * np.float32(g_d)).astype(np.float32)
    return e4m3_encode_signed_satfinite(t)


def nvfp4_output(v, g_d):
    """NVFP4 output of fp32 values v [rows, N] under the given encode scale
    g_d: (packed codes [rows, N/2], E4M3 block scales [rows, N/16] row-major,
    amax = max |v|)."""
    v = np.asarray(v, dtype=np.float32)
    codes, sf = quantize_values_with_scale(v, g_d)
    return pack_codes(codes), sf, (np.float32(np.max(np.abs(v))) if v.size else np.float32(0.0))


# --------------------------------------------------------------------------
# Scale-factor layout read by the tensor core (not described by the pages)
# --------------------------------------------------------------------------
def sf_tcgen05_bytes(rows: int, k: int) -> int:
    """Size of the tensor-core scale layout: rows padded to 128, K-blocks to 4."""
    rp = -(-rows // 128) * 128
    kbp = -(-(k // BLOCK) // 4) * 4
    return rp * kbp


def swizzle_sf_tcgen05(sf) -> np.ndarray:
    """Row-major scales [rows, K/16] -> the 128-row x 4-block atom layout.

    Atom (i, j) covers rows 128i..128i+127 and blocks 4j..4j+3 and sits at byte
    512 * (i * KB4 + j) (KB4 = padded blocks / 4, atoms K-fastest).  Inside an
    atom, (row r, block b) is at (r % 32) * 16 + (r // 32) * 4 + b.  Padding is 0.
    Parity unpinned by the pages (pinned on hardware by the GEMM).
    """
    sf = np.asarray(sf, dtype=np.uint8)
    rows, kb = sf.shape
    rp = -(-rows // 128) * 128
    kbp = -(-kb // 4) * 4
    full = np.zeros((rp, kbp), dtype=np.uint8)
    full[:rows, :kb] = sf
    # index by (row_atom, row32, row_quarter, k_atom, block) -> byte address
    t = full.reshape(rp // 128, 4, 32, kbp // 4, 4)          # (i, r//32, r%32, j, b)
    t = t.transpose(0, 3, 2, 1, 4)                            # (i, j, r%32, r//32, b)
    return np.ascontiguousarray(t).reshape(-1)


def unswizzle_sf_tcgen05(flat, rows: int, k: int) -> np.ndarray:
    kb = k // BLOCK
    rp = -(-rows // 128) * 128
    kbp = -(-kb // 4) * 4
    t = np.asarray(flat, dtype=np.uint8).reshape(rp // 128, kbp // 4, 32, 4, 4)
    t = t.transpose(0, 3, 2, 1, 4).reshape(rp, kbp)
    return np.ascontiguousarray(t[:rows, :kb])


# --------------------------------------------------------------------------
# Output comparisons used by the parity tests
# --------------------------------------------------------------------------
def bf16_ordinal(bits) -> np.ndarray:
    """Monotone integer image of bf16 bit patterns (for ulp distances)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)
