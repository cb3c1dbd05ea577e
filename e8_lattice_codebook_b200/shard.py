"""Row-parallel GLQ linear layer over several GPUs (one process per GPU,
torch.distributed for the collective).

The layer y = S_out . H_m . W^ . H_n . (S_in . x) is split over its input
columns: rank r holds the index columns of its column range, rotates the
whole (replicated) input x, and computes its part of the output in fp32 with
the library's kernels (glq_layer_create_shard); H_m and S_out are linear, so
one all-reduce (sum) of the parts' y over the ranks -- NCCL over NVLink on
GPUs -- gives the layer's y, which glq_cast rounds to the model's dtype.
Column ranges are whole 128-column chunks, dealt out as evenly as possible.
"""
from __future__ import annotations

import numpy as np

from . import _stream_ptr, dtype_code, glq_cast, glq_layer_create_shard, glq_layer_destroy, glq_linear

CHUNK = 128


def shard_ranges(n: int, world: int) -> list:
    """Input-column ranges [k0, k1) of `world` ranks: whole 128-column chunks
    (the last range ends at n), as even as possible, none empty."""
    chunks = -(-n // CHUNK)
    if world < 1 or world > chunks:
        raise ValueError(f"cannot split {chunks} chunks over {world} ranks")
    out = []
    for r in range(world):
        c0, c1 = chunks * r // world, chunks * (r + 1) // world
        out.append((c0 * CHUNK, min(c1 * CHUNK, n)))
    return out


class RowParallelLinear:
    """This rank's shard of one layer and the all-reduce of its output."""

    def __init__(self, m, n, bpw, idx1, idx_res, primary, residual, weight_scale, resid_scales, s_in, s_out,
                 rank: int, world: int, group=None):
        self.m, self.n, self.bpw = int(m), int(n), int(bpw)
        self.rank, self.world, self.group = rank, world, group
        self.k0, self.k1 = shard_ranges(self.n, world)[rank]
        self._cbs = (primary, residual)  # keep the codebooks alive
        if self.bpw <= 4:  # the two-stage argument form
            idx_res = [] if idx_res is None else [idx_res]
            resid_scales = [] if self.bpw == 2 else [resid_scales]
        self.handle = glq_layer_create_shard(self.m, self.n, self.bpw, idx1, idx_res, primary.handle,
                                             0 if residual is None else residual.handle, weight_scale,
                                             resid_scales, s_in, s_out, self.k0, self.k1)

    def partial(self, x, out=None, stream=None):
        """This rank's fp32 part of y (before the all-reduce)."""
        import torch
        y = out if out is not None else torch.empty((x.shape[0], self.m), dtype=torch.float32, device=x.device)
        glq_linear(self.handle, x.data_ptr(), dtype_code(x.dtype), y.data_ptr(), dtype_code(torch.float32),
                   x.shape[0], _stream_ptr(stream))
        return y

    def __call__(self, x, out_dtype=None, stream=None):
        """y of the whole layer on every rank: partial, all-reduce, cast."""
        import torch
        import torch.distributed as dist
        y32 = self.partial(x, stream=stream)
        if self.world > 1:
            dist.all_reduce(y32, op=dist.ReduceOp.SUM, group=self.group)
        odt = out_dtype or x.dtype
        if odt == torch.float32:
            return y32
        y = torch.empty(y32.shape, dtype=odt, device=y32.device)
        glq_cast(y32.data_ptr(), y.data_ptr(), dtype_code(odt), y32.numel(), _stream_ptr(stream))
        return y

    def close(self):
        if self.handle:
            glq_layer_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
