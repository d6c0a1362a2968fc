"""The parallel driver of the oracle (tests/oracle_pool.py) returns exactly
what the oracle returns when called on the whole problem."""
import numpy as np

import oracle_pool
from oracle import hadamard_oracle as H
from oracle import mxfp4_oracle as MX
from oracle import nvfp4_oracle as O
from oracle import stochastic_oracle as S
from nvfp4_block_scaled_15_b200 import inputs


def test_pool_quantize_equals_oracle():
    x = inputs.activations_with_outliers(2600, 256, seed=44, fraction=0.02, factor=40.0)   # > 1 task of rows
    got = oracle_pool.quantize(x)
    want = O.quantize(x)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
    assert got[2] == want[2] and got[3] == want[3]


def test_pool_gemm_ref_equals_oracle():
    xa = inputs.gaussian_bf16((5, 128), seed=45)
    xb = inputs.gaussian_bf16((300, 128), seed=46, std=0.02)
    pa, sa, ga, _ = O.quantize(xa)
    pb, sb, gb, _ = O.quantize(xb)
    d, s, alpha = O.gemm_ref(pa, sa, ga, pb, sb, gb)
    d2, s2, alpha2 = oracle_pool.gemm_ref(pa, sa, ga, pb, sb, gb, cols_per_slice=64)
    assert alpha2 == alpha
    assert np.all(np.abs(d2 - d) <= 1e-13 * float(alpha) * s)
    assert np.all(np.abs(s2 - s) <= 1e-13 * s)


def _same(got, want):
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
    assert got[2] == want[2] and got[3] == want[3]


def test_pool_stochastic_equals_oracle():
    """Rows in several tasks draw the random integers of their own indices."""
    x = inputs.activations_with_outliers(2600, 128, seed=47, fraction=0.02, factor=40.0)
    _same(oracle_pool.quantize_sr(x, 0x1234_5678_9ABC, 5), S.quantize_sr(x, 0x1234_5678_9ABC, 5))


def test_pool_rotated_equals_oracle():
    """The amax of y from the slices' maxima, then the rows by slices."""
    x = inputs.activations_with_outliers(2600, 256, seed=48, fraction=0.02, factor=40.0)
    assert oracle_pool.rotated_amax(x, 64) == np.float32(np.max(np.abs(H.fwht_f32(O.bf16_to_f32(x), 64))))
    _same(oracle_pool.quantize_hadamard(x, 64), H.quantize_hadamard(x, 64))
    _same(oracle_pool.quantize_hadamard_sr(x, 32, 9, 3), H.quantize_hadamard_sr(x, 32, 9, 3))


def test_pool_mxfp4_equals_oracle():
    x = inputs.activations_with_outliers(2600, 128, seed=49, fraction=0.02, factor=40.0)
    got, want = oracle_pool.quantize_mx(x), MX.quantize_mx(x)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
    pa, sa = MX.quantize_mx(inputs.gaussian_bf16((5, 128), seed=50))
    pb, sb = want
    d, s = MX.gemm_ref_mx(pa, sa, pb[:300], sb[:300])
    d2, s2 = oracle_pool.gemm_ref_mx(pa, sa, pb[:300], sb[:300], cols_per_slice=64)
    assert np.all(np.abs(d2 - d) <= 1e-13 * s) and np.all(np.abs(s2 - s) <= 1e-13 * s)
