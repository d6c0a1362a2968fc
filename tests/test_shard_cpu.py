"""The hot path split over ranks (nvfp4_block_scaled_15_b200.shard), on CPU.

Two gloo ranks on 127.0.0.1 run the split exactly as GPU ranks would, with
the oracle doing each rank's arithmetic (the library needs a GPU) and the
shard module doing the split and the exchange:
  * activations split by rows: each rank's amax, the all-reduce(max) of
    shard.all_reduce_amax_, then the quantization of its rows under the
    resulting g.  Both ranks' g must equal the unsharded g bit for bit, and
    the ranks' codes and scales, put together, the unsharded oracle's;
  * weights split by rows (the output columns): each rank computes D for its
    columns; shard.gather_columns assembles D, which must equal the
    unsharded reference.
A tensor whose amax sits on one rank only, and one holding a NaN, check that
the exchange keeps the unsharded result (g, or the range error) everywhere.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    from oracle import nvfp4_oracle as O
    from nvfp4_block_scaled_15_b200 import inputs, shard
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    res = {}
    try:
        # activations [300, 256] split by rows (ragged: 128-row units, 300 rows)
        x = inputs.activations_with_outliers(300, 256, seed=70, fraction=0.02, factor=50.0)
        r0, r1 = shard.row_range(x.shape[0], world, rank)
        amax = torch.tensor([O.amax(x[r0:r1])], dtype=torch.float32)
        shard.all_reduce_amax_(amax)
        g = O.global_scale(np.float32(amax.item()))
        codes, sf = O.quantize_with_scale(x[r0:r1], g)
        res["g"] = float(g)
        res["rows"] = (r0, r1)
        res["codes"] = O.pack_codes(codes)
        res["sf"] = sf
        # the tensor amax on the last rank's rows only
        y = inputs.gaussian_bf16((256, 64), seed=71)
        y[250, 5] = 0x4480                                    # 1024.0, far above the rest
        q0, q1 = shard.row_range(256, world, rank)
        a2 = torch.tensor([O.amax(y[q0:q1])], dtype=torch.float32)
        shard.all_reduce_amax_(a2)
        res["g_peak"] = float(O.global_scale(np.float32(a2.item())))
        # a NaN on rank 0's rows: every rank must see a non-finite amax
        z = inputs.gaussian_bf16((256, 64), seed=72)
        z[3, 3] = 0x7FC0
        a3 = torch.tensor([O.amax(z[slice(*shard.row_range(256, world, rank))])], dtype=torch.float32)
        shard.all_reduce_amax_(a3)
        res["nan_amax"] = bool(np.isnan(a3.item()))
        # weights [520, 256] split by rows -> D's columns
        w = inputs.gaussian_bf16((520, 256), seed=73, std=0.02)
        pa, sa, ga, _ = O.quantize(x)
        pw, sw, gw, _ = O.quantize(w)
        c0, c1 = shard.row_range(w.shape[0], world, rank)
        d_local, _, _ = O.gemm_ref(pa, sa, ga, pw[c0:c1], sw[c0:c1], gw)
        d = shard.gather_columns(torch.from_numpy(d_local), w.shape[0])
        res["d"] = d.numpy()
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_two_rank_split_equals_unsharded():
    from oracle import nvfp4_oracle as O
    from nvfp4_block_scaled_15_b200 import inputs
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    x = inputs.activations_with_outliers(300, 256, seed=70, fraction=0.02, factor=50.0)
    p, s, g, _ = O.quantize(x)
    assert out[0]["g"] == out[1]["g"] == float(g)
    assert out[0]["rows"] == (0, 128) and out[1]["rows"] == (128, 300)
    assert np.array_equal(np.concatenate([out[0]["codes"], out[1]["codes"]]), p)
    assert np.array_equal(np.concatenate([out[0]["sf"], out[1]["sf"]]), s)
    y = inputs.gaussian_bf16((256, 64), seed=71)
    y[250, 5] = 0x4480
    assert out[0]["g_peak"] == out[1]["g_peak"] == float(O.global_scale(O.amax(y)))
    assert out[0]["nan_amax"] and out[1]["nan_amax"]
    w = inputs.gaussian_bf16((520, 256), seed=73, std=0.02)
    pw, sw, gw, _ = O.quantize(w)
    d_ref, s_ref, alpha = O.gemm_ref(p, s, g, pw, sw, gw)
    for r in range(world):
        d = out[r]["d"]
        assert d.shape == d_ref.shape
        assert np.all(np.abs(d - d_ref) <= 1e-12 * float(alpha) * s_ref)


def test_row_range_partitions():
    from nvfp4_block_scaled_15_b200 import shard
    for rows in (0, 1, 127, 128, 129, 300, 28672, 28672 + 40):
        for world in (1, 2, 3, 4, 8):
            spans = [shard.row_range(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0 and a0 <= a1
            assert all(s0 % 128 == 0 for s0, _ in spans)
            units = [-(-(s1 - s0) // 128) for s0, s1 in spans]
            assert max(units) - min(units) <= 1
    with pytest.raises(ValueError):
        shard.row_range(10, 2, 2)
