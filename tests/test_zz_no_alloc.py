"""glq_linear_noalloc: the decode path for callers that cannot allocate
device memory at call time (graph capture, host callbacks, frameworks that
own every allocation).  Through the C ABI, its output must match
glq_linear's within the parity tolerance, on two calls in a row (the fixed
device scratch array keeps the previous call's contents), including a layer
whose split-K plan has to be narrowed to fit the array.

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


CASES = [  # (workload, layer, B): a 4 bpw layer, a 3 bpw layer, and the
           # 32768x5120 layer whose partial sums at B=16 exceed the array
    ("24b-decode-4bpw", 0, 16), ("smollm2-360m-3bpw", 2, 3), ("24b-decode-4bpw", 2, 16),
    ("single-1024-2bpw", 0, 1),
]


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
