"""The hot path split over ranks (one process per GPU, torch.distributed).

The work partitions without a data-path exchange except in one place:
  * GEMM and GEMV: the weight rows (the output columns n of D = A W^T) are
    split into contiguous ranges of whole 128-row tiles.  Each rank holds its
    slice of W's codes and tensor-core scales (both contiguous for such a
    range) under W's one global scale, and computes D[:, its columns] with
    no collective.  ``gather_columns`` assembles the whole D where a caller
    needs it (an all-gather).
  * Quantization of activations split by rows: the global encode scale
    g = 2688/amax needs the amax of the WHOLE tensor ("low-precision-floats",
    FP4 / MXFP4 / NVFP4: s_global from the tensor's amax).  The one exchange
    is an all-reduce(max) of the ranks' amax values, taken on their fp32 bit
    patterns as int32 (an amax is >= 0, and a NaN's pattern lies above
    infinity's), so every rank's g equals the unsharded g bit for bit.
Nothing here computes any of the method's arithmetic: the quantization and
the products run in the CUDA library (``nvfp4``), the exchange in
torch.distributed (NCCL on GPUs, gloo on the host).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

TILE_ROWS = 128          # rows of one tensor-core scale atom and one weight tile


def row_range(rows: int, world: int, rank: int, align: int = TILE_ROWS):
    """[start, stop) of ``rank``'s rows: contiguous, in whole ``align``-row
    units (the last unit may be short), sizes differing by one unit at most."""
    if world < 1 or not 0 <= rank < world or rows < 0 or align < 1:
        raise ValueError("bad split")
    units = -(-rows // align)
    u0 = units * rank // world
    u1 = units * (rank + 1) // world
    return min(rows, u0 * align), min(rows, u1 * align)


def _world(group):
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def all_reduce_amax_(amax: torch.Tensor, group=None) -> torch.Tensor:
    """In place: each rank's fp32 amax (one element) becomes the maximum over
    the ranks, compared as int32 bit patterns."""
    if amax.dtype != torch.float32 or amax.numel() != 1:
        raise ValueError("amax is one fp32 value")
    if _world(group) > 1:
        dist.all_reduce(amax.view(torch.int32), op=dist.ReduceOp.MAX, group=group)
    return amax


def quantize_row_sharded(x_local: torch.Tensor, group=None, layout=None):
    """Quantize this rank's rows of an activation tensor split by rows, under
    the global scale of the whole tensor: the amax pass on the local rows,
    the all-reduce(max), then the quantize pass with that amax given."""
    from . import nvfp4 as nv
    layout = nv.SF_TCGEN05 if layout is None else layout
    rows, k = x_local.shape
    q = nv.empty_quantized(rows, k, layout, x_local.device)
    nv.nvfp4_amax(x_local, rows, k, x_local.stride(0), q.amax)
    all_reduce_amax_(q.amax, group)
    nv.nvfp4_quantize(x_local, rows, k, x_local.stride(0), q.codes, q.sf, layout, q.g, q.amax, 1)
    return q


def slice_weight(w, world: int, rank: int):
    """``rank``'s rows of an NVFP4 weight quantized whole (tensor-core scale
    layout): views of its codes and scale atoms, W's global scale shared.
    Returns (Quantized view, (start, stop))."""
    from . import nvfp4 as nv
    if w.layout != nv.SF_TCGEN05:
        raise ValueError("weights in the tensor-core scale layout")
    r0, r1 = row_range(w.rows, world, rank)
    atom_row_bytes = nv.nvfp4_sf_bytes(TILE_ROWS, w.k, nv.SF_TCGEN05)     # one 128-row group of atoms
    sf = w.sf[(r0 // TILE_ROWS) * atom_row_bytes:(-(-r1 // TILE_ROWS)) * atom_row_bytes]
    return nv.Quantized(w.codes[r0:r1], sf, w.g, w.amax, r1 - r0, w.k, w.layout), (r0, r1)


def gather_columns(d_local: torch.Tensor, n_total: int, group=None) -> torch.Tensor:
    """The whole D [M, n_total] from each rank's columns (split by row_range):
    an all-gather of the column slices, padded to the widest slice."""
    world = _world(group)
    if world == 1:
        return d_local
    rank = dist.get_rank(group)
    widths = [row_range(n_total, world, r)[1] - row_range(n_total, world, r)[0] for r in range(world)]
    if d_local.shape[1] != widths[rank]:
        raise ValueError("local columns do not match this rank's range")
    w_max = max(widths)
    send = torch.zeros((d_local.shape[0], w_max), dtype=d_local.dtype, device=d_local.device)
    send[:, :widths[rank]] = d_local
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send.contiguous(), group=group)
    return torch.cat([p[:, :w] for p, w in zip(parts, widths)], dim=1)
