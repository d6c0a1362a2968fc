"""Child process of tests/test_gpu_gemv_workspace.py (not collected by pytest).

Runs the first GEMV launches of a fresh process on the decode workload
(W [28672, 8192], tiles split between CTAs) with workspace bytes that do not
start at zero, and saves every output's bf16 bits for the parent to check
against the oracle:
  * nvfp4_gemv_batched, M = 1, 4, 8 and 20, each on a workspace whose int32
    words are all 1 (stale small counts) before the call;
  * nvfp4_gemv_batched_noalloc, M = 1, 4, 8, 20, 1, 16, 4 interleaved: the
    library's fixed scratch, which each call leaves to the next (an M = 20
    or M = 16 call, two kernels, leaves 32-bit counts where the M <= 8
    kernel keeps its 64-bit tagged counters).
Usage: python gemv_fresh_process_child.py OUT.npz
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def main(out_path: str) -> None:
    import numpy as np
    import torch

    from nvfp4_block_scaled_15_b200 import inputs
    from nvfp4_block_scaled_15_b200 import nvfp4 as lib
    from parity import dev_bf16, host_bf16_bits

    x_a, w = inputs.decode_gemv(20)
    x_b = inputs.gaussian_bf16((20, w.shape[1]), seed=17)
    qw = lib.quantize(dev_bf16(w), lib.SF_TCGEN05)
    xa, xb = dev_bf16(x_a), dev_bf16(x_b)
    n, k = w.shape
    out = {}
    for m in (1, 4, 8, 20):                  # the workspace entry point, stale counts of 1
        ws = torch.empty(lib.nvfp4_workspace_bytes(lib.OP_GEMV_BATCHED, m, n, k), dtype=torch.uint8, device="cuda")
        ws.view(torch.int32).fill_(1)
        y = lib.gemv_batched(xa[:m], qw, workspace=ws)
        out[f"ws_a_{m}"] = host_bf16_bits(y)
    for i, (m, src, name) in enumerate([(1, xa, "a"), (4, xb, "b"), (8, xa, "a"), (20, xb, "b"), (1, xb, "b"),
                                        (16, xa, "a"), (4, xa, "a")]):
        x = src[:m]
        y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        lib.nvfp4_gemv_batched_noalloc(x, m, x.stride(0), qw.codes, qw.sf, qw.g, n, k, y, y.stride(0))
        out[f"noalloc{i}_{name}_{m}"] = host_bf16_bits(y)
    torch.cuda.synchronize()
    status = lib.nvfp4_check_device_status()
    np.savez(out_path, status=np.array(status), **out)


if __name__ == "__main__":
    main(sys.argv[1])
