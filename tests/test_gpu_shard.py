"""The split over ranks (nvfp4_block_scaled_15_b200.shard) on one GPU.

A rank's share of the work is an ordinary library call on a slice: the
weight slice of ``shard.slice_weight`` (codes rows and whole 128-row scale
atoms of a weight quantized whole) must give exactly the columns of the
unsplit GEMM and GEMV, and ``quantize_row_sharded`` (amax pass, the
exchange, quantize pass with the amax given) exactly ``quantize`` when one
rank holds all rows.  The exchange itself is tested on two gloo ranks
(tests/test_shard_cpu.py)."""
import numpy as np
import pytest
import torch

from nvfp4_block_scaled_15_b200 import inputs, shard
from parity import dev_bf16, host_u8

pytestmark = pytest.mark.gpu


def test_quantize_row_sharded_single_rank_equals_quantize(lib):
    x = dev_bf16(inputs.activations_with_outliers(300, 512, seed=81, fraction=0.01, factor=30.0))
    q1 = shard.quantize_row_sharded(x)
    q2 = lib.quantize(x, lib.SF_TCGEN05)
    torch.cuda.synchronize()
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.sf, q2.sf)
    assert torch.equal(q1.g, q2.g) and torch.equal(q1.amax, q2.amax)


@pytest.mark.parametrize("world", [2, 3])
def test_weight_slices_give_the_columns_of_the_whole(lib, world):
    m, n, k = 256, 1000, 1024
    a = lib.quantize(dev_bf16(inputs.gaussian_bf16((m, k), seed=82)), lib.SF_TCGEN05)
    w = lib.quantize(dev_bf16(inputs.gaussian_bf16((n, k), seed=83, std=0.02)), lib.SF_TCGEN05)
    x = dev_bf16(inputs.gaussian_bf16((4, k), seed=84))
    d_full = lib.gemm(a, w)
    y_full = lib.gemv_batched(x, w)
    for rank in range(world):
        ws, (c0, c1) = shard.slice_weight(w, world, rank)
        d = lib.gemm(a, ws)
        y = lib.gemv_batched(x, ws)
        torch.cuda.synchronize()
        assert lib.nvfp4_check_device_status() == lib.OK
        assert torch.equal(d.view(torch.int16), d_full[:, c0:c1].view(torch.int16))
        assert torch.equal(y.view(torch.int16), y_full[:, c0:c1].view(torch.int16))
