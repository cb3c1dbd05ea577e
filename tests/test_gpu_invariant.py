"""The batch-invariant mode (glq_layer_set_batch_invariant): a token's
output is the same bits whatever the batch it arrives in (B = 1, 8, 17 and
512, i.e. one-token decode, a decode batch, and batches the default mode
runs on the tensor cores) and wherever in the batch it sits; the results are
within the oracle bound and reproducible run to run.  Layers cover every
kind of stage (16-bit E8 stages, the fp16-table 8-bit stage of an odd bpw)
and both transform kernels (rows up to 16384 values and the clustered
kernel for longer rows), through the C ABI.  (The pages' claim: glq 0.5.1
PyPI page, "Inference kernels", "Bit-exact determinism".)"""
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


LAYERS = [  # m, n, bpw, x dtype
    (2048, 2048, 4, "bf16"), (960, 2560, 3, "f16"), (1024, 2048, 7, "bf16"),
    (20480, 1024, 2, "f16"), (1024, 20480, 4, "bf16"),
]


@pytest.mark.parametrize("m,n,bpw,xdt", LAYERS)
def test_tokens_bitwise_independent_of_batch_and_path(dev, m, n, bpw, xdt):
    L = gi.make_layer(m + 2 * n + bpw, 11, m, n, bpw)
    lay = dev.layer(L)
    xb = gi.make_x(m + 2 * n + bpw, 11, 512, n, xdt)
    x = to_torch_x(xb, xdt)
    # the default mode: B = 1 decode and B = 512 tensor-core results differ
    # in their rounding (different arithmetic); the mode removes that
    lay.set_batch_invariant(True)
    try:
        y512 = lay(x, out_dtype=torch.float32)
        assert torch.equal(y512, lay(x, out_dtype=torch.float32))  # run to run
        for B in (1, 8, 17):
            yb = lay(x[:B].contiguous(), out_dtype=torch.float32)
            assert torch.equal(yb, y512[:B]), B
        yw = lay(x[5:22].contiguous(), out_dtype=torch.float32)  # 17 tokens, shifted
        assert torch.equal(yw, y512[5:22])
        y16 = lay(x[:512].contiguous())  # production dtype, same rule
        assert torch.equal(lay(x[:8].contiguous()), y16[:8])
        sample = [0, 1, 16, 17, 511]
        ref = orc.linear(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out,
                         xb[sample], xdt == "bf16", cb2=L.cb2_f16, threads=0)
        err = np.max(np.abs(y512.cpu().numpy().astype(np.float64)[sample] - ref))
        print(f"\nINVARIANT {m}x{n} bpw {bpw}: err {err:.3e} tol {tolerance(ref):.3e}")
        assert err <= tolerance(ref)
        plan = lay.decode_plan(1)
        for B in (8, 9, 16):
            assert lay.decode_plan(B)["splits"] == plan["splits"], B
    finally:
        lay.set_batch_invariant(False)
    lay.check()
