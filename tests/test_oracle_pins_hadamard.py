"""Pins of the Hadamard-rotation oracle (CPU only).

[P1] "NVIDIA NVFP4 与 Micro-Scaling", section 4.1: x @ H with H orthogonal
     (H H^T = I), a fast Walsh-Hadamard transform; outlier channels are spread
     over all channels; the rotation absorbed into the weights leaves the
     layer's product unchanged.
The Walsh-Hadamard matrix itself is pinned against scipy.linalg.hadamard.
"""
import numpy as np
import pytest
import scipy.linalg

from oracle import hadamard_oracle as H
from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs

SIZES = [16, 32, 64, 128, 256, 512]


def _x(rows, c, seed, outliers=True):
    if outliers:
        return inputs.activations_with_outliers(rows, c, seed=seed, fraction=0.01, factor=30.0)
    return inputs.gaussian_bf16((rows, c), seed=seed)


def check_matrix_is_sylvester_hadamard():
    """Rows of the identity map to the rows of H_b / sqrt(b), exactly (every
    partial sum is a small integer), segment by segment."""
    for b in SIZES:
        eye = np.eye(b, dtype=np.float32)
        want = (scipy.linalg.hadamard(b).astype(np.float32) * H.norm_constant(b)).astype(np.float32)
        assert np.array_equal(H.fwht_f32(eye, b), want), b
    # block diagonal: a unit vector in segment 1 of C = 2b leaves segment 0 at zero
    b = 64
    e = np.zeros((1, 2 * b), dtype=np.float32)
    e[0, b + 5] = 1.0
    y = H.fwht_f32(e, b)
    assert not y[0, :b].any()
    assert np.array_equal(y[0, b:], (scipy.linalg.hadamard(b)[5] * H.norm_constant(b)).astype(np.float32))


def check_close_to_exact_product():
    """fp32 transform within (log2 b + 1) 2^-23 c_b sum|x_seg| of the exact x H."""
    x = O.bf16_to_f32(_x(8, 1024, 3)).astype(np.float64)
    for b in SIZES:
        hm = scipy.linalg.hadamard(b).astype(np.float64) / np.sqrt(b)
        exact = (x.reshape(8, -1, b) @ hm).reshape(8, -1)
        got = H.fwht_f32(x.astype(np.float32), b).astype(np.float64)
        l1 = np.repeat(np.abs(x).reshape(8, -1, b).sum(axis=2), b, axis=1)
        lim = (np.log2(b) + 1) * 2.0 ** -23 * float(H.norm_constant(b)) * l1
        assert np.all(np.abs(got - exact) <= lim), b


def check_orthogonal():
    """H H^T = I: the transform keeps each segment's energy and is its own inverse."""
    x = O.bf16_to_f32(_x(4, 2048, 5)).astype(np.float32)
    for b in SIZES:
        y = H.fwht_f32(x, b)
        ex = (x.astype(np.float64) ** 2).reshape(4, -1, b).sum(axis=2)
        ey = (y.astype(np.float64) ** 2).reshape(4, -1, b).sum(axis=2)
        assert np.allclose(ey, ex, rtol=1e-5), b
        back = H.fwht_f32(y, b)
        assert np.allclose(back, x, rtol=0, atol=1e-5 * np.max(np.abs(x))), b


def check_layer_product_unchanged():
    """(x H)(w H)^T = x w^T (the rotation absorbed into the weights)."""
    x = O.bf16_to_f32(_x(16, 1024, 7)).astype(np.float32)
    w = O.bf16_to_f32(inputs.gaussian_bf16((24, 1024), seed=8, std=0.02)).astype(np.float32)
    want = x.astype(np.float64) @ w.astype(np.float64).T
    for b in (16, 128, 512):
        got = H.fwht_f32(x, b).astype(np.float64) @ H.fwht_f32(w, b).astype(np.float64).T
        scale = np.abs(x).astype(np.float64) @ np.abs(w).astype(np.float64).T
        assert np.all(np.abs(got - want) <= 1e-5 * scale), b


def check_outliers_spread():
    """P1 4.1: after the rotation the channels' variances are closer (the
    spread of per-channel rms falls) and a block's absmax is no longer set by
    a single outlier channel (the largest and the mean share of a 16-element
    block's energy held by one element fall)."""
    x = O.bf16_to_f32(_x(64, 2048, 11)).astype(np.float64)

    def chan_spread(t):
        r = np.sqrt(np.mean(t ** 2, axis=0))
        return r.std() / r.mean()

    def shares(t):
        e = (t ** 2).reshape(64, -1, 16)
        s = e.max(axis=2) / e.sum(axis=2)
        return s.max(), s.mean()

    for b in (16, 64, 512):
        y = H.fwht_f32(x.astype(np.float32), b).astype(np.float64)
        assert chan_spread(y) < 0.6 * chan_spread(x), b
        (mx, mn), (my, ny) = shares(x), shares(y)
        assert my < 0.8 * mx and ny < 0.8 * mn, b


def check_order_one_is_plain_quantize():
    """b = 1 is the identity: the rotated quantizer equals the plain one."""
    x_bits = _x(8, 256, 13)
    p1, s1, g1, a1 = H.quantize_hadamard(x_bits, 1)
    p0, s0, g0, a0 = O.quantize(x_bits)
    assert np.array_equal(p1, p0) and np.array_equal(s1, s0) and g1 == g0 and a1 == a0


def check_amax_of_rotated_tensor():
    """The global scale comes from the rotated tensor: its amax block gets the
    largest scale 448 and its amax element code +-6."""
    x_bits = _x(8, 512, 17)
    p, s, g, a = H.quantize_hadamard(x_bits, 128)
    y = H.fwht_f32(O.bf16_to_f32(x_bits), 128)
    assert a == np.float32(np.max(np.abs(y)))
    r, c = np.unravel_index(np.argmax(np.abs(y)), y.shape)
    assert s[r, c // 16] == 0x7E
    assert O.unpack_codes(p)[r, c] & 7 == 7


CHECKS = [check_matrix_is_sylvester_hadamard, check_close_to_exact_product, check_orthogonal,
          check_layer_product_unchanged, check_outliers_spread, check_order_one_is_plain_quantize,
          check_amax_of_rotated_tensor]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_hadamard_pin(check):
    check()


# --------------------------------------------------------------------------
# Planted mistakes
# --------------------------------------------------------------------------
def _mut_no_norm(mp):
    mp.setattr(H, "norm_constant", lambda b: np.float32(1.0))


def _mut_norm_1_over_b(mp):
    mp.setattr(H, "norm_constant", lambda b: np.float32(1.0 / b))


def _mut_swapped_difference(mp):
    real = H.fwht_f32
    def f(x, b):
        # (v - u) instead of (u - v) in every stage: negate, transform, fix the sum
        x = np.asarray(x, dtype=np.float32)
        rows, c = x.shape
        y = x.reshape(rows, c // b, b).copy()
        h = 1
        while h < b:
            z = y.reshape(rows, c // b, b // (2 * h), 2, h)
            u = z[:, :, :, 0, :].copy()
            v = z[:, :, :, 1, :].copy()
            z[:, :, :, 0, :] = u + v
            z[:, :, :, 1, :] = v - u
            h *= 2
        return (y * H.norm_constant(b)).astype(np.float32).reshape(rows, c)
    mp.setattr(H, "fwht_f32", f)


def _mut_shifted_segments(mp):
    real = H.fwht_f32
    def f(x, b):
        x = np.asarray(x, dtype=np.float32)
        return np.roll(real(np.roll(x, b // 2, axis=1), b), -(b // 2), axis=1)
    mp.setattr(H, "fwht_f32", f)


def _mut_amax_of_input(mp):
    real = H.quantize_hadamard
    mp.setattr(H, "quantize_hadamard", lambda x, b, amax_value=None: real(x, b, O.amax(x)))


MUTATIONS = [_mut_no_norm, _mut_norm_1_over_b, _mut_swapped_difference, _mut_shifted_segments, _mut_amax_of_input]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_planted_mistakes(mutate, monkeypatch):
    mutate(monkeypatch)
    caught = False
    for check in CHECKS:
        try:
            check()
        except AssertionError:
            caught = True
            break
    assert caught, f"no pin catches {mutate.__name__}"


def test_rotated_stochastic_composition():
    """Rotation followed by stochastic rounding: order 1 is the plain stochastic
    quantizer; scales, g and amax are the rotated quantizer's; every code is a
    neighbour of the rotated u; averaged over offsets, the dequantized values
    approach y = x H (unbiased in the rotated domain)."""
    from oracle import stochastic_oracle as S
    x = _x(8, 256, 41)
    assert all(np.array_equal(u, v) for u, v in zip(H.quantize_hadamard_sr(x, 1, 5, 6), S.quantize_sr(x, 5, 6)))
    for b in (16, 128):
        p, sf, g, a = H.quantize_hadamard_sr(x, b, 5, 6)
        p2, sf2, g2, a2 = H.quantize_hadamard(x, b)
        assert np.array_equal(sf, sf2) and g == g2 and a == a2
        d_rn = np.abs(O.e2m1_decode(O.unpack_codes(p)) - O.e2m1_decode(O.unpack_codes(p2)))
        assert np.all(d_rn <= 2.0)                                   # at most one grid step apart
    y = H.fwht_f32(O.bf16_to_f32(x), 16).astype(np.float64)
    acc = np.zeros_like(y)
    for off in range(48):
        p, sf, g, _ = H.quantize_hadamard_sr(x, 16, 9, off)
        acc += O.dequantize(p, sf, g)
    p2, sf2, g2, _ = H.quantize_hadamard(x, 16)
    assert np.abs(acc / 48 - y).mean() < 0.4 * np.abs(O.dequantize(p2, sf2, g2) - y).mean()
