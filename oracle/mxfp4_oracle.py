"""MXFP4 oracle: a plain, slow, CPU statement of MXFP4 quantization and its
block-scaled GEMM (the format NVFP4 is compared with on the pages).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
The library never imports it.  It shares no code with the CUDA path; it reuses
the E2M1 encoder, packing and the scale-layout helper of ``nvfp4_oracle``.

Pages cited:
  [P2] "mxFP4/nvFP4 最小化知识", sections nvFP4与mxFP4的核心差异解析 and
       (一) mxFP4的技术局限: 32 elements share one E8M0 (power-of-two) scale;
       an optimal scale of 0.9 becomes 1.0.
  [P3] "Introducing NVFP4 ...", 表 1: MXFP4 = E2M1 with one shared
       power-of-two scale per 32-value block.
  [P4] "low-precision-floats", section "FP4 / MXFP4 / NVFP4":
       x_hat = s_mx * Q_E2M1(x / s_mx), s_mx = 2^round(log2(A/6)) with A the
       block max |x|, and "TensorRT usually rounds up", which the page's bounds
       use (1 <= rho_mx = s_mx / (A/6) < 2, |e| <= s_mx, zero threshold
       0.25 s_mx between A/24 and A/12).

Definition (readings marked):
  1. per 32 consecutive elements along K: A = max |x| (bf16 -> fp32 exact);
  2. v = A / 6 in fp32 (RN); k = ceil(log2 v), exact, from v's bits
     [reading: rounded up, as the page says TensorRT does and as its bounds
     assume]; k is clamped to the E8M0 range [-127, 127]; A == 0 gives
     k = -127 [reading: the pages are silent; every code of such a block is 0
     whatever the scale];
  3. scale byte (E8M0) = k + 127;
  4. per element: code = e2m1_rne_sat(x * 2^-k) (fp32; the multiply by a power
     of two is exact unless the result underflows) - |x * 2^-k| <= 6 always;
  5. pack as NVFP4 (low nibble first);
  6. GEMM: D = sum_k (2^ka qa)(2^kb qb) in fp64, no global scale.
A block whose A is not finite raises RangeError [reading, as for NVFP4].
"""
import numpy as np

from oracle import nvfp4_oracle as NV

MX_BLOCK = 32          # elements per E8M0 scale [P2 (一); P3 表 1; P4 MXFP4]
E8M0_BIAS = 127


def e8m0_decode(b) -> np.ndarray:
    """fp64 value 2^(b - 127) of E8M0 scale bytes (0xFF, NaN, is never produced)."""
    b = np.asarray(b, dtype=np.int64)
    return np.ldexp(1.0, b - E8M0_BIAS)


def ceil_log2_f32(v) -> np.ndarray:
    """ceil(log2 v) for positive finite fp32 v, exactly (from the bits)."""
    v = np.asarray(v, dtype=np.float32)
    m, e = np.frexp(v.astype(np.float64))          # v = m 2^e, m in [0.5, 1)
    # v is a power of two exactly when m == 0.5: then log2 v = e - 1
    return np.where(m == 0.5, e - 1, e).astype(np.int64)


def mx_scale_exponent(block_amax) -> np.ndarray:
    """k = ceil(log2(fp32(A / 6))), clamped to [-127, 127]; -127 for A == 0."""
    a = np.asarray(block_amax, dtype=np.float32)
    if not np.all(np.isfinite(a)):
        raise NV.RangeError("non-finite block amax")
    v = (a / np.float32(6.0)).astype(np.float32)
    k = np.where(v > 0, ceil_log2_f32(np.where(v > 0, v, np.float32(1.0))), -E8M0_BIAS)
    return np.clip(k, -E8M0_BIAS, E8M0_BIAS)


def quantize_mx(x_bits):
    """bf16 [rows, K] -> (packed codes [rows, K/2], E8M0 scales [rows, K/32])."""
    x = NV.bf16_to_f32(x_bits)
    rows, k = x.shape
    assert k % MX_BLOCK == 0
    blocks = x.reshape(rows, k // MX_BLOCK, MX_BLOCK)
    a = np.max(np.abs(blocks), axis=2)
    e = mx_scale_exponent(a)
    inv = np.ldexp(np.float32(1.0), -e).astype(np.float32)       # 2^-k, exact in fp32
    u = (blocks * inv[:, :, None]).astype(np.float32)
    codes = NV.e2m1_encode(u).reshape(rows, k)
    return NV.pack_codes(codes), (e + E8M0_BIAS).astype(np.uint8)


def dequantize_mx(packed, sf) -> np.ndarray:
    """x_hat = 2^k * E2M1[code] in fp64 [P4 MXFP4]."""
    q = NV.e2m1_decode(NV.unpack_codes(packed))
    rows, k = q.shape
    s = e8m0_decode(sf)
    return (q.reshape(rows, k // MX_BLOCK, MX_BLOCK) * s[:, :, None]).reshape(rows, k)


def gemm_ref_mx(a_packed, a_sf, b_packed, b_sf):
    """D = (s_a (.) A)(s_b (.) B)^T in fp64 and S = sum_k |a_k b_k| (no alpha)."""
    ad = dequantize_mx(a_packed, a_sf)
    bd = dequantize_mx(b_packed, b_sf)
    return ad @ bd.T, np.abs(ad) @ np.abs(bd).T


def gemm_ref_mx_entries(a_packed, a_sf, b_packed, b_sf, rows, cols):
    """D[rows[i], cols[i]] and S for a list of coordinates, one dot product each."""
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    d = np.empty(rows.size)
    s = np.empty(rows.size)
    for i, (r, c) in enumerate(zip(rows, cols)):
        ar = dequantize_mx(a_packed[r:r + 1], a_sf[r:r + 1])[0]
        bc = dequantize_mx(b_packed[c:c + 1], b_sf[c:c + 1])[0]
        d[i] = np.dot(ar, bc)
        s[i] = np.dot(np.abs(ar), np.abs(bc))
    return d, s


def sf_tcgen05_bytes_mx(rows: int, k: int) -> int:
    """Tensor-core layout of MX scales: rows padded to 128, K/32 scales to 4
    (an atom of 128 rows x 4 scales covers 128 of K)."""
    return (-(-rows // 128) * 128) * (-(-(k // MX_BLOCK) // 4) * 4)
