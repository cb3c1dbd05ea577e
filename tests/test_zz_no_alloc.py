"""glq_linear_noalloc: the decode path for callers that cannot allocate
device memory at call time (graph capture, host callbacks, frameworks that
own every allocation).  Through the C ABI, its output must match
glq_linear's within the parity tolerance, on two calls in a row (the fixed
device scratch array keeps the previous call's contents).  One layer is set
up so that glq_linear's split-K partial sums cannot fit the array: the
noalloc call must narrow its split count (the test checks the arithmetic of
that plan through glq_decode_plan) and still match glq_linear and the oracle.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test."""
import numpy as np
import pytest

import glq_inputs as gi
from gpu_helpers import Device, to_torch_x, tolerance

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Device()


def _noalloc(glq, lay, x, y):
    glq.glq_linear_noalloc(lay.handle, x.data_ptr(), glq.dtype_code(x.dtype), y.data_ptr(),
                           glq.dtype_code(y.dtype), x.shape[0],
                           torch.cuda.current_stream().cuda_stream)


CASES = [  # (workload, layer, B): 4 bpw layers, a 3 bpw layer, a 2 bpw layer
    ("24b-decode-4bpw", 0, 16), ("smollm2-360m-3bpw", 2, 3), ("24b-decode-4bpw", 2, 16),
    ("single-1024-2bpw", 0, 1),
]

SCRATCH = 8 << 20  # GLQ_NOALLOC_SCRATCH_BYTES


def test_noalloc_matches_glq_linear_two_calls(dev):
    import e8_lattice_codebook_b200 as glq
    layers = []
    for key, li, B in CASES:
        wl = gi.WORKLOADS[key]
        L = gi.workload_layer(wl, li)
        lay = dev.layer(L)
        x = to_torch_x(gi.workload_x(wl, li, B), wl.x_dtype)
        ref = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
        layers.append((lay, x, ref))
    for rnd in range(2):  # two calls in a row on every layer
        for lay, x, ref in layers:
            y = torch.full((x.shape[0], lay.m), float("nan"), dtype=torch.float32, device="cuda")
            _noalloc(glq, lay, x, y)
            got = y.cpu().numpy().astype(np.float64)
            err = np.max(np.abs(got - ref))
            assert np.all(np.isfinite(got))
            assert err <= tolerance(ref), (rnd, lay.m, lay.n, err, tolerance(ref))
    # production dtype output as well
    lay, x, ref = layers[0]
    yb = torch.empty((x.shape[0], lay.m), dtype=x.dtype, device="cuda")
    _noalloc(glq, lay, x, yb)
    yl = lay(x)
    assert torch.allclose(yb.float(), yl.float(), rtol=2 ** -7, atol=tolerance(ref))
    lay.check()


def test_noalloc_rejects_large_batches(dev):
    import e8_lattice_codebook_b200 as glq
    L = gi.make_layer(9, 0, 64, 64, 2)
    lay = dev.layer(L)
    x = torch.zeros((17, 64), dtype=torch.float16, device="cuda")
    y = torch.zeros((17, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(glq.GlqError) as e:
        _noalloc(glq, lay, x, y)
    assert e.value.status == 2  # GLQ_ERR_SHAPE


def test_noalloc_narrows_a_plan_whose_partials_do_not_fit(dev):
    """32768 x 2048 at 4 bpw, 16 tokens, with the input transform fused on
    request and the cluster reduction off: glq_linear's plan splits K into
    power-of-two ranges whose fp64 partial sums (splits x 16 x 32768 x 8
    bytes) exceed the scratch array, so the noalloc call has to take a
    narrower plan (here one split, the separate transform).  Its output must
    still match glq_linear and the oracle, twice in a row."""
    import e8_lattice_codebook_b200 as glq
    from oracle import glq_oracle as orc
    m, n, B = 32768, 2048, 16
    L = gi.make_layer(77, 1, m, n, 4)
    lay = dev.layer(L)
    lay.set_fusion(1)  # GLQ_FUSE_INPUT, no cluster reduction
    plan = lay.decode_plan(B)
    per_split = B * m * 8
    fixed = B * m * 4 + B * n * 2
    assert plan["fused_input"] == 1 and plan["cluster"] == 0 and plan["splits"] > 1, plan
    assert plan["splits"] * per_split > SCRATCH - fixed, plan  # glq_linear's plan cannot fit
    xb = gi.make_x(77, 1, B, n, "bf16")
    x = to_torch_x(xb, "bf16")
    ref_lin = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    ref = orc.linear(m, n, 4, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb, True,
                     threads=0)
    for rnd in range(2):
        y = torch.full((B, m), float("nan"), dtype=torch.float32, device="cuda")
        _noalloc(glq, lay, x, y)
        got = y.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref_lin)) <= tolerance(ref_lin), rnd
        assert np.max(np.abs(got - ref)) <= tolerance(ref), rnd
    lay.check()
