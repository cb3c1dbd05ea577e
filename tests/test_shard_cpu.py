"""Row-parallel shards of the layer (a layer split over its input columns,
one all-reduce of the parts' outputs), host side, without a GPU:

* the column ranges the ranks take: whole 128-column chunks, covering
  [0, n) exactly, in order, as even as possible;
* the identity the shards rely on, checked with the fp64 oracle: the output
  of the layer with every column outside a range zeroed (index 0 is the E8
  origin in every 16-bit stage), summed over the ranges, equals the layer's
  output (H_m and S_out are linear, and W^ xr splits over columns);
* the collective step of RowParallelLinear on two gloo ranks (127.0.0.1): each
  rank's fp32 part, summed by the all-reduce, gives every rank the layer's
  output.
"""
import os
import socket
import sys

import numpy as np
import pytest

import glq_inputs as gi
from oracle import glq_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shard_ranges_cover_and_balance():
    from e8_lattice_codebook_b200.shard import shard_ranges
    for n in (960, 2048, 2560, 5120, 11008, 14336, 32768):
        for world in (1, 2, 3, 4, 8):
            if world > -(-n // 128):
                continue
            rs = shard_ranges(n, world)
            assert len(rs) == world and rs[0][0] == 0 and rs[-1][1] == n
            for (a0, a1), (b0, _) in zip(rs, rs[1:]):
                assert a1 == b0
            sizes = [k1 - k0 for k0, k1 in rs]
            assert all(k0 % 128 == 0 for k0, _ in rs) and min(sizes) > 0
            assert max(-(-s // 128) for s in sizes) - min(-(-s // 128) for s in sizes) <= 1
    with pytest.raises(ValueError):
        shard_ranges(256, 3)


def _masked(L, k0, k1):
    """The layer with every input column outside [k0, k1) zeroed (origin index)."""
    g0, g1 = k0 // 8, k1 // 8
    keep = np.zeros(L.n // 8, dtype=bool)
    keep[g0:g1] = True
    idx1 = np.where(keep[None, :], L.idx1, 0).astype(np.uint16)
    res, _ = L.stages()
    res = [np.where(keep[None, :], a, 0).astype(a.dtype) for a in res]
    idx2 = None if not res else (res[0] if L.bpw <= 4 else res)
    return idx1, idx2


def _partial(L, xb, k0, k1):
    idx1, idx2 = _masked(L, k0, k1)
    return orc.linear(L.m, L.n, L.bpw, idx1, idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb, True)


@pytest.mark.parametrize("m,n,bpw,world", [(64, 512, 4, 2), (40, 960, 2, 3), (72, 1280, 6, 4), (16, 384, 8, 3)])
def test_parts_sum_to_the_layer(m, n, bpw, world):
    from e8_lattice_codebook_b200.shard import shard_ranges
    L = gi.make_layer(m + n, 6, m, n, bpw)
    xb = gi.make_x(m + n, 6, 3, n, "bf16")
    full = orc.linear(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb, True)
    parts = [_partial(L, xb, k0, k1) for k0, k1 in shard_ranges(n, world)]
    np.testing.assert_allclose(sum(parts), full, rtol=0, atol=1e-9 * (np.abs(full).max() + 1))
    assert all(np.abs(p).max() > 0 for p in parts)  # each part contributes


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from e8_lattice_codebook_b200.shard import RowParallelLinear, shard_ranges
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m, n, bpw = 48, 768, 4
        L = gi.make_layer(9, 1, m, n, bpw)
        xb = gi.make_x(9, 1, 2, n, "bf16")
        k0, k1 = shard_ranges(n, world)[rank]
        # the collective step of the class, with this rank's part from the
        # oracle in place of the GPU kernels (no GPU here)
        lay = object.__new__(RowParallelLinear)
        lay.m, lay.n, lay.bpw, lay.rank, lay.world, lay.group = m, n, bpw, rank, world, None
        lay.handle = 0
        part = torch.from_numpy(_partial(L, xb, k0, k1).astype(np.float32))
        lay.partial = lambda x, out=None, stream=None: part.clone()
        y = lay(torch.zeros((2, n), dtype=torch.float32), out_dtype=torch.float32)
        q.put((rank, y.numpy().astype(np.float64)))
    finally:
        dist.destroy_process_group()


def test_rowparallel_allreduce_on_two_gloo_ranks():
    torch = pytest.importorskip("torch")
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    L = gi.make_layer(9, 1, 48, 768, 4)
    xb = gi.make_x(9, 1, 2, 768, "bf16")
    full = orc.linear(48, 768, 4, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb, True)
    for r in range(world):
        np.testing.assert_allclose(got[r], full, rtol=0, atol=1e-4 * (np.abs(full).max() + 1))
    np.testing.assert_array_equal(got[0], got[1])
