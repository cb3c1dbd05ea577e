"""GPU parity of 5-8 bpw layers (glq 0.5.1 PyPI page, "Bit widths": a 16-bit
primary index plus 16-bit E8 and 8-bit residual stages) against the fp64
oracle, through the C ABI (glq_layer_create_stages):

* glq_dequant_reference bit-exact, every stage order and rounding included;
* the decode path (B <= 16) with the transforms fused and separate, and the
  tensor-core path (B > 16, W reconstructed in fp16 first), every token,
  fp32 output within 2e-3 (||y||_inf + 1), production dtype within that
  plus one output rounding;
* a mixed-precision step: layers of different bit widths back to back on
  one device.
(The full-size 24B-class layers at 5 and 6 bpw run in the workload sweep of
test_gpu_parity.py.)
"""
import numpy as np
import pytest

import glq_inputs as gi
from gpu_helpers import Device, production_tolerance, to_torch_x, tolerance
from oracle import glq_oracle as orc

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Device()


def oracle_y(L, xb, xdt):
    return orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out,
                      xb, xdt == "bf16", cb2=L.cb2_f16, threads=0)


SHAPES = [(272, 264), (1000, 968), (24, 56), (520, 1032)]


@pytest.mark.parametrize("bpw", [5, 6, 7, 8])
@pytest.mark.parametrize("m,n", SHAPES)
def test_dequant_bit_exact(dev, m, n, bpw):
    L = gi.make_layer(m + n + bpw, 8, m, n, bpw)
    lay = dev.layer(L)
    w = lay.dequant().cpu().numpy().astype(np.float64)
    ref = orc.decode_rows(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, cb2=L.cb2_f16)
    np.testing.assert_array_equal(w, ref)


CASES = [  # m, n, bpw, B, x dtype
    (272, 264, 5, 1, "bf16"), (1000, 968, 6, 3, "f16"), (24, 56, 7, 16, "bf16"), (520, 1032, 8, 9, "f16"),
    (2048, 2048, 5, 2, "bf16"), (960, 2560, 7, 8, "f16"), (4096, 5120, 6, 1, "bf16"), (2048, 11008, 8, 4, "bf16"),
    (272, 264, 5, 17, "bf16"), (1000, 968, 6, 300, "f16"), (136, 1024, 7, 600, "bf16"), (520, 1032, 8, 40, "f16"),
]


@pytest.mark.parametrize("m,n,bpw,B,xdt", CASES)
def test_linear_all_tokens(dev, m, n, bpw, B, xdt):
    L = gi.make_layer(3 * m + n, 9, m, n, bpw)
    xb = gi.make_x(3 * m + n, 9, B, n, xdt)
    lay = dev.layer(L)
    x = to_torch_x(xb, xdt)
    ref = oracle_y(L, xb, xdt)
    flags = (-1, 0) if B <= 16 else (-1,)
    for f in flags:  # default (fused where the library fuses) and separate transforms
        lay.set_fusion(f)
        y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
        err = np.max(np.abs(y - ref))
        print(f"\nSTAGES {m}x{n} bpw {bpw} B={B} fusion {f}: err {err:.3e} tol {tolerance(ref):.3e} "
              f"ratio {err / tolerance(ref):.3f}")
        assert err <= tolerance(ref), (f, err, tolerance(ref))
    lay.set_fusion(-1)
    yp = lay(x).float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(yp - ref) <= production_tolerance(ref, xdt))
    lay.check()


def test_decode_determinism_and_separate_kernels_batch_invariance(dev):
    """Run to run bitwise; per token across B <= 16 bitwise with the
    transforms as separate kernels (exact integer stage sums, a fixed
    8-bit-stage order per split plan)."""
    L = gi.make_layer(77, 3, 1024, 2048, 7)
    lay = dev.layer(L)
    xb = gi.make_x(77, 3, 16, 2048, "bf16")
    x = to_torch_x(xb, "bf16")
    lay.set_fusion(0)
    y16 = lay(x, out_dtype=torch.float32)
    assert torch.equal(y16, lay(x, out_dtype=torch.float32))
    for B in (9, 12):
        assert torch.equal(lay(x[:B].contiguous(), out_dtype=torch.float32), y16[:B]), B
    lay.set_fusion(-1)


def test_mixed_precision_step(dev):
    """The mixed-precision SmolLM3-3B-shaped set (q, o at 4 bpw; gate, up,
    down at 5 bpw) back to back on one stream, one token, every output."""
    wl = gi.WORKLOADS["smollm3-3b-mixed"]
    outs = []
    for li in range(len(wl.layers)):
        L = gi.workload_layer(wl, li)
        assert L.bpw == wl.layer_bpw[li]
        xb = gi.workload_x(wl, li, 1)
        lay = dev.layer(L)
        outs.append((L, xb, lay(to_torch_x(xb, "bf16"), out_dtype=torch.float32)))
    torch.cuda.synchronize()
    for L, xb, y in outs:
        ref = oracle_y(L, xb, "bf16")
        assert np.max(np.abs(y.cpu().numpy().astype(np.float64) - ref)) <= tolerance(ref), L.bpw
