"""The GEMV's workspace contract, at the decode workload's full size.

The stream-K fix-up counters of the one-kernel path (M <= 8) are never
cleared by a separate step: each carries a per-launch tag, and each launch returns the
counters it used to zero.  These tests check, against the oracle on every
output, that
  * the first launches of a fresh process are right on a workspace whose
    bytes start as stale int32 counts of 1, and so are interleaved calls of
    the no-allocation entry point that share the library's scratch;
  * a CUDA graph that replays one GEMV launch (one tag for all replays) gives
    the right answer on every replay, for new activations each time.
W [28672, 8192] puts 224 weight tiles on the 148 CTAs, so tiles are split
between CTAs and their partial sums meet through the counters.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle_pool
from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import check_bf16, dev_bf16, host_bf16_bits, host_u8

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def decode_w():
    """The decode weights and their oracle quantization (every row)."""
    x_a, w = inputs.decode_gemv(20)
    x_b = inputs.gaussian_bf16((20, w.shape[1]), seed=17)
    pw, sw, gw, _ = oracle_pool.quantize(w)
    return {"w": w, "x_a": x_a, "x_b": x_b, "pw": pw, "sw": sw, "gw": gw}


def _check_all_columns(y_bits, x_bits, ref):
    px, sx, gx, _ = O.quantize(x_bits)
    d_ref, s_ref, alpha = oracle_pool.gemm_ref(px, sx, gx, ref["pw"], ref["sw"], ref["gw"])
    assert y_bits.shape == d_ref.shape
    check_bf16(y_bits, d_ref, s_ref, alpha)


def test_fresh_process_stale_workspace_and_shared_scratch(decode_w, tmp_path):
    out = tmp_path / "gemv_fresh.npz"
    env = dict(os.environ)
    proc = subprocess.run([sys.executable, os.path.join(HERE, "gemv_fresh_process_child.py"), str(out)],
                          env=env, capture_output=True, text=True, timeout=900)
    assert proc.returncode == 0, proc.stdout[-2000:] + proc.stderr[-4000:]
    res = np.load(out)
    assert int(res["status"]) == 0
    names = [k for k in res.files if k != "status"]
    assert len(names) == 11
    for name in names:
        src, m = name.split("_")[-2], int(name.split("_")[-1])
        x = decode_w["x_" + src][:m]
        _check_all_columns(res[name], x, decode_w)


@pytest.mark.parametrize("m", [1, 4, 8, 16, 20])
def test_graph_replays_one_launch(lib, decode_w, m):
    """Capture one nvfp4_gemv_batched call, replay it three times with new
    activations copied into the captured input; every replay is checked."""
    w = decode_w["w"]
    n, k = w.shape
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    if m == 1:      # the decode weights themselves, every byte
        assert np.array_equal(host_u8(qw.codes), decode_w["pw"])
        assert np.array_equal(host_u8(qw.sf), O.swizzle_sf_tcgen05(decode_w["sw"]))
    x_static = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    y_static = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(lib.nvfp4_workspace_bytes(lib.OP_GEMV_BATCHED, m, n, k), dtype=torch.uint8, device="cuda")
    lib.gemv_batched(x_static, qw, out=y_static, workspace=ws)        # loads the kernels before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        lib.gemv_batched(x_static, qw, out=y_static, workspace=ws)
    for seed in (31, 32, 33):
        x = inputs.gaussian_bf16((m, k), seed=seed)
        x_static.copy_(dev_bf16(x))
        graph.replay()
        torch.cuda.synchronize()
        assert lib.nvfp4_check_device_status() == lib.OK
        _check_all_columns(host_bf16_bits(y_static), x, decode_w)
    del graph
