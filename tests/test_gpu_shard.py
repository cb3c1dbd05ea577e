"""Row-parallel shards on the GPU (glq_layer_create_shard, glq_cast), through
the C ABI.  The test holds every part of a layer on the one GPU of the test
and sums their fp32 outputs (the all-reduce of a multi-GPU run, which needs
no kernel of the library); the sum must match the fp64 oracle within the
parity bound, on the decode path (separate transforms, the exact per-shard
row sums) and the tensor-core path (W reconstructed per shard), for whole
and ragged column ranges, an 8-bit stage and rows above 16384 values.  Each
shard's dequantised columns are bit-exact, and glq_cast rounds to nearest.
"""
import numpy as np
import pytest

import glq_inputs as gi
from gpu_helpers import Device, to_torch_x, tolerance
from oracle import glq_oracle as orc

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Device()


def _shard(dev, L, k0, k1):
    import e8_lattice_codebook_b200 as glq
    res, rs = L.stages()
    resid = glq.Codebook(L.cb2_f16.reshape(256, 8)) if L.bpw % 2 else None
    h = glq.glq_layer_create_shard(L.m, L.n, L.bpw, L.idx1, res, dev.e8.handle, 0 if resid is None else resid.handle,
                                   L.weight_scale, rs, L.s_in, L.s_out, k0, k1)
    return h, resid


CASES = [  # m, n, bpw, world, B, x dtype
    (2048, 2048, 4, 2, 1, "bf16"), (960, 2560, 3, 3, 9, "f16"), (5120, 32768, 4, 4, 2, "bf16"),
    (1024, 4096, 5, 3, 16, "bf16"), (2048, 2048, 4, 2, 300, "bf16"), (1000, 968, 6, 2, 600, "f16"),
]


@pytest.mark.parametrize("m,n,bpw,world,B,xdt", CASES)
def test_parts_sum_to_the_oracle(dev, m, n, bpw, world, B, xdt):
    import e8_lattice_codebook_b200 as glq
    from e8_lattice_codebook_b200.shard import shard_ranges
    L = gi.make_layer(m + n + world, 12, m, n, bpw)
    xb = gi.make_x(m + n + world, 12, B, n, xdt)
    x = to_torch_x(xb, xdt)
    stream = torch.cuda.current_stream().cuda_stream
    total = torch.zeros((B, m), dtype=torch.float32, device="cuda")
    keep = []
    for k0, k1 in shard_ranges(n, world):
        h, resid = _shard(dev, L, k0, k1)
        keep.append((h, resid))
        part = torch.empty((B, m), dtype=torch.float32, device="cuda")
        glq.glq_linear(h, x.data_ptr(), glq.dtype_code(x.dtype), part.data_ptr(), glq.GLQ_F32, B, stream)
        total += part
        w = torch.empty((m, k1 - k0), dtype=torch.float32, device="cuda")
        glq.glq_dequant_reference(h, w.data_ptr(), stream)
        ref_w = orc.decode_rows(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, 0, 8, cb2=L.cb2_f16)
        np.testing.assert_array_equal(w[:8].cpu().numpy().astype(np.float64), ref_w[:, k0:k1])
    sample = list(range(B)) if B <= 16 else [0, 1, B // 2, B - 1]
    ref = orc.linear(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb[sample],
                     xdt == "bf16", cb2=L.cb2_f16, threads=0)
    y = total.cpu().numpy().astype(np.float64)[sample]
    err = np.max(np.abs(y - ref))
    print(f"\nSHARD {m}x{n} bpw {bpw} x{world} B={B}: err {err:.3e} tol {tolerance(ref):.3e}")
    assert err <= tolerance(ref)
    for h, _ in keep:
        glq.glq_layer_check(h, stream)
        glq.glq_layer_destroy(h)


def test_shard_rejects_bad_ranges_and_dtypes(dev):
    import e8_lattice_codebook_b200 as glq
    L = gi.make_layer(1, 1, 64, 512, 4)
    for k0, k1 in ((64, 512), (0, 200), (256, 256), (0, 640)):
        with pytest.raises(glq.GlqError) as e:
            _shard(dev, L, k0, k1)
        assert e.value.status == 2  # GLQ_ERR_SHAPE
    h, _ = _shard(dev, L, 128, 512)
    x = torch.zeros((1, 512), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(glq.GlqError) as e:
        glq.glq_linear(h, x.data_ptr(), glq.GLQ_BF16, y.data_ptr(), glq.GLQ_BF16, 1,
                       torch.cuda.current_stream().cuda_stream)
    assert e.value.status == 3  # GLQ_ERR_DTYPE: a part's output stays fp32
    with pytest.raises(glq.GlqError):
        glq.glq_layer_set_batch_invariant(h, True)
    glq.glq_layer_destroy(h)


def test_cast_rounds_to_nearest_even(dev):
    import e8_lattice_codebook_b200 as glq
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(100003) * 50).astype(np.float32)
    src = torch.from_numpy(v).cuda()
    for dt, code in ((torch.bfloat16, glq.GLQ_BF16), (torch.float16, glq.GLQ_F16)):
        out = torch.empty(v.size, dtype=dt, device="cuda")
        glq.glq_cast(src.data_ptr(), out.data_ptr(), code, v.size, torch.cuda.current_stream().cuda_stream)
        assert torch.equal(out, src.to(dt))


def test_rowparallel_single_rank_nccl(dev):
    """The RowParallelLinear wrapper with a one-rank NCCL group (one GPU
    here): the whole layer as its own shard, cast to bf16, equals glq_linear."""
    import os
    import socket
    import torch.distributed as dist
    from e8_lattice_codebook_b200.shard import RowParallelLinear
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        L = gi.make_layer(5, 2, 1024, 2048, 4)
        xb = gi.make_x(5, 2, 4, 2048, "bf16")
        x = to_torch_x(xb, "bf16")
        rp = RowParallelLinear(L.m, L.n, L.bpw, L.idx1, L.idx2, dev.e8, dev.e8, L.weight_scale, L.resid_scale,
                               L.s_in, L.s_out, rank=0, world=1)
        y = rp(x)
        ref = dev.layer(L)(x, out_dtype=torch.float32)
        assert torch.equal(y, ref.to(torch.bfloat16))
        rp.close()
    finally:
        dist.destroy_process_group()
