"""Hadamard-rotated NVFP4 quantization oracle: a plain, slow, CPU statement.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
The library never imports it.  It shares no code with the CUDA path; it reuses
the NVFP4 quantization steps of ``nvfp4_oracle``.

Page cited:
  [P1] "NVIDIA NVFP4 与 Micro-Scaling", section 4.1 旋转/阿达玛变换: before
       quantization the activations are rotated, x @ H with H an orthogonal
       [C, C] matrix (H H^T = I), a fast Walsh-Hadamard transform or a random
       rotation, which spreads outlier channels over all channels; the same
       rotation is absorbed into the adjacent weights, so the layer's product
       is unchanged.

Definition (readings marked):
  1. H = blockdiag(H_b, ..., H_b) / sqrt(b), H_b the Sylvester-ordered
     Walsh-Hadamard matrix of order b (a power of two): an orthogonal [C, C]
     matrix [reading: the block-diagonal form, b dividing C, so one operand
     row needs no more than b elements together; b = C is the page's full
     transform when C is a power of two];
  2. y = x H computed by the fast Walsh-Hadamard transform in fp32, per
     b-element segment: stages h = 1, 2, 4, ..., b/2, each pair (i, i + h)
     with bit h of i clear becoming (fp32(y_i + y_{i+h}), fp32(y_i - y_{i+h}));
     then y = fp32(y * c_b), c_b = fp32(1 / sqrt(b)) [reading: the rounding
     of the transform is fixed by this order, which the kernel follows];
  3. y is quantized to NVFP4 like any fp32 tensor (steps 1-5 of
     nvfp4_oracle, the amax taken over y);
  4. with stochastic rounding ("FP4" encyclopedia entry, 技術原理, names the
     rotation and stochastic rounding together): step 3 with the element
     rounding of stochastic_oracle, its random integers indexed by the
     position in y.
"""
import numpy as np

from oracle import nvfp4_oracle as NV
from oracle import stochastic_oracle as SR


def norm_constant(b: int) -> np.float32:
    """c_b = fp32(1 / sqrt(b)) (exact for b a power of four)."""
    return np.float32(1.0 / np.sqrt(np.float64(b)))


def fwht_f32(x, b: int) -> np.ndarray:
    """y = x H (definition step 2) for fp32 x [rows, C], C % b == 0."""
    x = np.asarray(x, dtype=np.float32)
    rows, c = x.shape
    if b < 1 or (b & (b - 1)) or c % b:
        raise ValueError("b must be a power of two dividing C")
    y = x.reshape(rows, c // b, b).copy()
    h = 1
    while h < b:
        z = y.reshape(rows, c // b, b // (2 * h), 2, h)
        u = z[:, :, :, 0, :].copy()
        v = z[:, :, :, 1, :].copy()
        z[:, :, :, 0, :] = (u + v).astype(np.float32)
        z[:, :, :, 1, :] = (u - v).astype(np.float32)
        h *= 2
    y = (y * norm_constant(b)).astype(np.float32)
    return y.reshape(rows, c)


def quantize_hadamard(x_bits, b: int, amax_value=None):
    """bf16 [rows, C] -> rotated NVFP4: (packed codes, row-major scales, g, amax of y)."""
    y = fwht_f32(NV.bf16_to_f32(x_bits), b)
    if amax_value is not None:
        a = np.float32(amax_value)
    else:                                   # an empty tensor has amax 0, so g = 1
        a = np.float32(np.max(np.abs(y))) if y.size else np.float32(0.0)
    g = NV.global_scale(a)
    codes, sf = NV.quantize_values_with_scale(y, g)
    return NV.pack_codes(codes), sf, g, a


def quantize_hadamard_sr(x_bits, b: int, seed: int, offset: int, amax_value=None, row_ids=None):
    """bf16 [rows, C] -> rotated NVFP4 with stochastic rounding (definition step 4):
    (packed codes, row-major scales, g, amax of y)."""
    y = fwht_f32(NV.bf16_to_f32(x_bits), b)
    if amax_value is not None:
        a = np.float32(amax_value)
    else:
        a = np.float32(np.max(np.abs(y))) if y.size else np.float32(0.0)
    g = NV.global_scale(a)
    codes, sf = SR.quantize_values_sr(y, g, seed, offset, row_ids)
    return NV.pack_codes(codes), sf, g, a
