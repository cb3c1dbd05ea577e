"""Failure detection in the device waits, on the GPU, without a fault.

Every wait in the layer's kernels is bounded: after its limit it reports
GLQ_DEVERR_TIMEOUT through the layer's device error word, which
glq_layer_check turns into GLQ_ERR_TIMEOUT, and the kernel returns.  Here
each of the three wait helpers runs (glq_layer_selftest_wait) on a barrier
that only one of its two expected arrivals reaches, a flag that nothing sets,
with a short limit: the wait must run out within milliseconds and report
the timeout, the same wait on a completed barrier must not, and the context
must stay usable (a layer call afterwards matches the fp64 oracle).
"""
import time

import numpy as np
import pytest

import glq_inputs as gi
from gpu_helpers import Device, to_torch_x, tolerance
from oracle import glq_oracle as orc

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

GLQ_ERR_TIMEOUT = 9
KINDS = [(0, 2_000_000), (1, 2_000_000), (2, 200_000)]  # (kind, limit: cycles, cycles, polls)


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Device()


@pytest.mark.parametrize("kind,limit", KINDS)
def test_wait_runs_out_and_reports(dev, kind, limit):
    import e8_lattice_codebook_b200 as glq
    L = gi.make_layer(77, 0, 64, 256, 2)
    lay = dev.layer(L)
    lay.check()  # clean start
    t0 = time.time()
    lay.selftest_wait(kind, 1, limit)
    with pytest.raises(glq.GlqError) as ei:
        lay.check()
    assert ei.value.status == GLQ_ERR_TIMEOUT
    assert time.time() - t0 < 2.0
    lay.check()  # the check cleared the word
    lay.selftest_wait(kind, 2, limit)  # both arrivals: the wait completes
    lay.check()
    # the context stays usable
    xb = gi.make_x(77, 0, 3, L.n, "bf16")
    y = lay(to_torch_x(xb, "bf16"), out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    ref = orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb, True)
    assert np.max(np.abs(y - ref)) <= tolerance(ref)
    lay.check()


def test_selftest_rejects_bad_arguments(dev):
    import e8_lattice_codebook_b200 as glq
    lay = dev.layer(gi.make_layer(78, 0, 16, 64, 2))
    for kind, arrivals, limit in ((3, 1, 10), (0, 0, 10), (0, 3, 10), (0, 1, 0), (2, 1, 1 << 33)):
        with pytest.raises(glq.GlqError) as ei:
            lay.selftest_wait(kind, arrivals, limit)
        assert ei.value.status == 1  # GLQ_ERR_INVALID_ARG
