"""Stochastic-rounding NVFP4 quantization oracle: a plain, slow, CPU statement.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
The library never imports it.  It shares no code with the CUDA path; it reuses
the format functions of ``nvfp4_oracle`` (E2M1 table, E4M3 encoder, global
scale, packing).

Page cited:
  [P5] "FP4" encyclopedia entry (newton.com.tw), section 技術原理: NVFP4's
       quantization uses stochastic rounding instead of plain truncation
       (and a Hadamard transform before it).

Definition (readings marked; the pages give no further detail):
  1-3. amax, g = 2688 / amax and the E4M3 block scales exactly as the
       deterministic quantizer (round to nearest even; scales are not drawn)
       [reading: only the element values are rounded stochastically];
  4. u = fp32(fp32(x * g) / sd) as in the deterministic quantizer; with
     a = |u| between adjacent E2M1 magnitudes lo <= a < hi (step hi - lo of
     0.5, 1 or 2), f = (a - lo) / (hi - lo), and R a 16-bit random integer,
     the magnitude is hi when R < f * 2^16, else lo; a >= 6 gives 6; the code
     keeps u's sign bit (a negative u that rounds to 0 gives code 8, -0); a
     block whose scale decodes to 0 gets zero codes
     [reading: rounding up with probability ceil(f * 2^16) / 2^16, which is
     f to within 2^-16 of a step, so E[x_hat] = x to within that];
  5. R comes from Philox4x32-10 (J. Salmon, M. Moraes, R. Dror, D. Shaw,
     "Parallel random numbers: as easy as 1, 2, 3", SC 2011): key =
     (seed mod 2^32, seed div 2^32); for row r and 16-element block b the
     counters (2b + h, r, offset mod 2^32, offset div 2^32), h = 0, 1, give
     words w0..w3; element 8h + 2i + m of the block takes bits 16m..16m+15
     of w_i [reading: a counter-based layout, so any element's bits can be
     regenerated on their own].
"""
import numpy as np

from oracle import nvfp4_oracle as NV

# Philox4x32 constants from the paper (round multipliers and Weyl key increments)
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)
SR_BITS = 16


def philox4x32_10(counter, key) -> np.ndarray:
    """Philox4x32 with 10 rounds: uint32 counters [..., 4] and keys [..., 2]
    (broadcast) -> uint32 [..., 4].  One round maps (c0, c1, c2, c3) with key
    (k0, k1) to (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0));
    the key grows by (W0, W1) between rounds."""
    c = np.asarray(counter, dtype=np.uint64)
    k = np.asarray(key, dtype=np.uint64)
    c0, c1, c2, c3 = c[..., 0], c[..., 1], c[..., 2], c[..., 3]
    k0, k1 = k[..., 0], k[..., 1]
    for rnd in range(10):
        if rnd:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK
        p0 = np.uint64(PHILOX_M0) * c0
        p1 = np.uint64(PHILOX_M1) * c2
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & _MASK,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & _MASK)
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def random16(rows: int, k: int, seed: int, offset: int, row_ids=None) -> np.ndarray:
    """The 16-bit random integers R [rows, k] of definition step 5 (for the
    tensor rows ``row_ids`` when given, else rows 0 .. rows-1)."""
    if k % NV.BLOCK:
        raise ValueError("K must be a multiple of 16")
    kb = k // NV.BLOCK
    ids = np.arange(rows) if row_ids is None else np.asarray(row_ids)
    r = ids.astype(np.uint64)[:, None, None]
    b = np.arange(kb, dtype=np.uint64)[None, :, None]
    h = np.arange(2, dtype=np.uint64)[None, None, :]
    ctr = np.empty((rows, kb, 2, 4), dtype=np.uint64)
    ctr[..., 0] = 2 * b + h
    ctr[..., 1] = r
    ctr[..., 2] = offset & 0xFFFFFFFF
    ctr[..., 3] = (offset >> 32) & 0xFFFFFFFF
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    w = philox4x32_10(ctr, key)                                   # [rows, kb, 2, 4]
    halves = np.stack([w & np.uint32(0xFFFF), w >> np.uint32(16)], axis=-1)   # [rows, kb, 2, 4, 2]
    return halves.reshape(rows, k).astype(np.uint16)


def e2m1_encode_sr(u, r16) -> np.ndarray:
    """Stochastic rounding of fp32 values to E2M1 codes (definition step 4)."""
    u = np.asarray(u, dtype=np.float32)
    a = np.abs(u).astype(np.float64)
    r = np.asarray(r16, dtype=np.uint16).astype(np.float64)
    lo = np.clip(np.searchsorted(NV.E2M1_MAGNITUDES, a, side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    step = NV.E2M1_MAGNITUDES[hi] - NV.E2M1_MAGNITUDES[lo]
    with np.errstate(invalid="ignore", divide="ignore"):
        f = np.where(step > 0, (a - NV.E2M1_MAGNITUDES[lo]) / np.where(step > 0, step, 1.0), 0.0)
    up = r < f * 2.0 ** SR_BITS
    code = np.where(a >= NV.E2M1_MAX, 7, np.where(up, hi, lo)).astype(np.uint8)
    return code | np.where(np.signbit(u), np.uint8(8), np.uint8(0))


def quantize_values_sr(y, g, seed: int, offset: int, row_ids=None):
    """Steps 3-5 for fp32 values y [rows, K] under a given encode scale g:
    (codes [rows, K] unpacked, row-major scales [rows, K/16])."""
    y = np.asarray(y, dtype=np.float32)
    rows, k = y.shape
    g = np.float32(g)
    yb = y.reshape(rows, k // NV.BLOCK, NV.BLOCK)
    ab = np.max(np.abs(yb), axis=2) if k else np.zeros((rows, 0), dtype=np.float32)
    s_raw = (ab * g).astype(np.float32) / np.float32(6.0)
    sf = NV.e4m3_encode_satfinite(s_raw.astype(np.float32))
    sd = NV.e4m3_decode(sf)
    t = (yb * g).astype(np.float32)
    zero = (sd == 0)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.where(zero, np.float32(0.0), t / np.where(zero, np.float32(1.0), sd[:, :, None])).astype(np.float32)
    r16 = random16(rows, k, seed, offset, row_ids).reshape(rows, k // NV.BLOCK, NV.BLOCK)
    codes = e2m1_encode_sr(u, r16)
    codes = np.where(np.broadcast_to(zero, codes.shape), np.uint8(0), codes)
    return codes.reshape(rows, k).astype(np.uint8), sf.astype(np.uint8)


def quantize_sr(x_bits, seed: int, offset: int, amax_value=None, row_ids=None):
    """bf16 [rows, K] -> (packed codes [rows, K/2], row-major scales [rows, K/16], g, amax).
    ``row_ids``: the tensor rows x_bits holds (a sample of a larger tensor, whose
    amax is then given), which select the random integers."""
    a = NV.amax(x_bits) if amax_value is None else np.float32(amax_value)
    g = NV.global_scale(a)
    codes, sf = quantize_values_sr(NV.bf16_to_f32(x_bits), g, seed, offset, row_ids)
    return NV.pack_codes(codes), sf, g, a
