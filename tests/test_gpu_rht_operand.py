"""GPU checks of the tensor-core path's input stage through the C ABI
(glq_rht_input_operand): the fp16 operand xh = xr 2^e and 2^-e per row,
with xr = H_n (S_in x), against the fp64 oracle's block-diagonal Hadamard.

Bounds (per element, ref = the oracle's xr):
* butterfly kernel: fp32 butterflies, then one rounding to fp16:
  2^-11 |ref| + 2^-18 max |ref|;
* tensor-core kernel: three roundings to fp16 (after its first and second
  16 x 16 products, and at the end).  The last is within 2^-11 |ref|.  Each
  intermediate one perturbs the values of that stage by at most 2^-11 of
  themselves; the remaining orthogonal stages spread those perturbations
  over every output as a sum of many independent terms, of standard
  deviation below 2^-11 rms(ref) / sqrt(3) per rounding.  The bound
  2^-11 |ref| + 2^-8 rms(ref) leaves more than ten standard deviations for
  the two of them.

Rows: seeded normal activations (with 1 % outlier columns x20 for bf16),
plus a zero row, a single spike near the dtype's largest values and a row of
values near its smallest normals.  Row lengths: every row size 2^9 .. 2^14
that the tensor-core kernel takes, with one to five Hadamard blocks; lengths
that are not a multiple of 256 (butterfly kernel) and one longer than 16384
(clustered kernel) through the automatic choice.
"""
import numpy as np
import pytest

import glq_inputs as gi
from gpu_helpers import Device, to_torch_x
from oracle import glq_oracle as orc

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Device()


TENSOR_N = [512, 768, 1024, 1280, 2048, 2304, 3840, 4096, 4352, 6144, 7936, 8192, 12288, 14336, 16128, 16384]
OTHER_N = [264, 968, 5000, 20480]


def x_to_f64(xbits, xdt):
    if xdt == "f16":
        return xbits.view(np.float16).astype(np.float64)
    return (xbits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rows(n, xdt, seed):
    """uint16 bit patterns [B][n]: normal rows, then zero, spike and tiny rows."""
    xb = gi.make_x(seed, 0, 4, n, xdt, outliers=(xdt == "bf16"))
    big = 6.0e4 if xdt == "f16" else 1.0e38
    tiny = 1.0e-4 if xdt == "f16" else 1.0e-36
    extra = np.zeros((3, n))
    extra[1, n // 3] = big
    rng = np.random.default_rng(seed)
    extra[2] = tiny * (1.0 + rng.random(n)) * rng.choice([-1.0, 1.0], size=n)
    if xdt == "f16":
        eb = extra.astype(np.float16).view(np.uint16)
    else:
        eb = gi.f64_to_bf16_bits(extra)
    return np.concatenate([xb, eb], axis=0)


def check_operand(xh, inv, ref, kind):
    got = xh.float().cpu().numpy().astype(np.float64)[:, : ref.shape[1]] * inv.cpu().numpy()[:, None]
    assert np.all(xh.float().cpu().numpy()[:, ref.shape[1]:] == 0.0), "padding columns"
    worst = 0.0
    for b in range(ref.shape[0]):
        r = ref[b]
        if kind == "butterfly":
            bound = 2.0 ** -11 * np.abs(r) + 2.0 ** -18 * np.abs(r).max()
        else:
            bound = 2.0 ** -11 * np.abs(r) + 2.0 ** -8 * np.sqrt(np.mean(r * r))
        err = np.abs(got[b] - r)
        assert np.all(np.isfinite(got[b])), (kind, b)
        assert np.all(err <= bound), (kind, b, float(np.max(err - bound)))
        if np.any(r):
            worst = max(worst, float(np.max(err / np.maximum(bound, 1e-300))))
    return worst


@pytest.mark.parametrize("xdt", ["bf16", "f16"])
@pytest.mark.parametrize("n", TENSOR_N)
def test_tensor_core_input_transform(dev, n, xdt):
    L = gi.make_layer(n, 0, 8, n, 2)
    lay = dev.layer(L)
    xb = rows(n, xdt, n + 7)
    x = to_torch_x(xb, xdt)
    ref = np.stack([orc.hadamard_apply(v) for v in x_to_f64(xb, xdt) * L.s_in])
    xh_t, inv_t = lay.rht_input_operand(x, kernel=lay.RHT_TENSOR)
    xh_b, inv_b = lay.rht_input_operand(x, kernel=lay.RHT_BUTTERFLY)
    xh_a, inv_a = lay.rht_input_operand(x, kernel=lay.RHT_AUTO)
    torch.cuda.synchronize()
    wt = check_operand(xh_t, inv_t, ref, "tensor")
    wb = check_operand(xh_b, inv_b, ref, "butterfly")
    print(f"\nRHT operand n={n} {xdt}: tensor {wt:.3f} of bound, butterfly {wb:.3f}")
    assert torch.equal(xh_a, xh_t) and torch.equal(inv_a, inv_t), "the automatic choice is the tensor-core kernel"
    assert torch.all(xh_t[4] == 0) and float(inv_t[4]) == 1.0, "zero row"


@pytest.mark.parametrize("xdt", ["bf16", "f16"])
@pytest.mark.parametrize("n", OTHER_N)
def test_other_lengths_take_another_kernel(dev, n, xdt):
    L = gi.make_layer(n, 0, 8, n, 2)
    lay = dev.layer(L)
    xb = rows(n, xdt, n + 11)
    x = to_torch_x(xb, xdt)
    ref = np.stack([orc.hadamard_apply(v) for v in x_to_f64(xb, xdt) * L.s_in])
    xh, inv = lay.rht_input_operand(x)
    check_operand(xh, inv, ref, "butterfly")
    import e8_lattice_codebook_b200 as glq
    with pytest.raises(glq.GlqError) as ei:
        lay.rht_input_operand(x, kernel=lay.RHT_TENSOR)
    assert ei.value.status == 2  # GLQ_ERR_SHAPE


def test_tensor_core_transform_determinism_and_row_independence(dev):
    """Bit-identical on a rerun, and each row's operand the same whatever the
    batch (rows land on different CTAs and staging slots)."""
    n = 14336
    L = gi.make_layer(3, 3, 8, n, 2)
    lay = dev.layer(L)
    xb = gi.make_x(3, 3, 700, n, "bf16", outliers=True)
    x = to_torch_x(xb, "bf16")
    xh1, inv1 = lay.rht_input_operand(x, kernel=lay.RHT_TENSOR)
    xh2, inv2 = lay.rht_input_operand(x, kernel=lay.RHT_TENSOR)
    assert torch.equal(xh1, xh2) and torch.equal(inv1, inv2)
    for B in (1, 17, 149, 300):
        xs = x[B - 1:].contiguous()
        xh3, inv3 = lay.rht_input_operand(xs[:B].contiguous(), kernel=lay.RHT_TENSOR)
        assert torch.equal(xh3, xh1[B - 1:2 * B - 1]) and torch.equal(inv3, inv1[B - 1:2 * B - 1]), B


@pytest.mark.parametrize("xdt", ["bf16", "f16"])
@pytest.mark.parametrize("B", [1, 4, 20])
def test_extreme_rows_through_the_layer(dev, B, xdt):
    """Rows of values near the dtype's smallest normals, a single spike near
    its largest, and a zero row, through glq_linear on the decode (B <= 16)
    and tensor-core paths: finite, and within the parity bound of the fp64
    oracle.  (The per-row power-of-two scale of the operand is kept finite
    for the tiniest rows.)"""
    m, n, bpw = 64, 4096, 4
    L = gi.make_layer(31, 1, m, n, bpw)
    lay = dev.layer(L)
    xb = rows(n, xdt, 5)[4:]  # zero, spike, tiny
    xb = np.concatenate([xb] * ((B + 2) // 3), axis=0)[:B]
    x = to_torch_x(xb, xdt)
    y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    ref = orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb,
                     xdt == "bf16")
    assert np.all(np.isfinite(y))
    for b in range(B):
        tol = 2e-3 * (np.abs(ref[b]).max() + 1.0)
        assert np.max(np.abs(y[b] - ref[b])) <= tol, b
