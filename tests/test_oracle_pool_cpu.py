"""The parallel driver of the oracle (tests/oracle_pool.py) returns exactly
what the oracle returns when called on the whole problem."""
import numpy as np

import oracle_pool
from oracle import nvfp4_oracle as O
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
