"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

* glq_dequant_reference: bit-exact against the oracle's explicit decode;
* glq_rht_input / glq_rht_output: against the oracle's dense Hadamard;
* glq_linear (fp32 output): max |y - y_oracle| <= 2e-3 (||y_oracle||_inf + 1),
  on small shapes spanning several tiles with ragged tails, and on every
  layer of every synthetic workload at full size and at every batch it names
  (every token of the decode batches, sampled tokens of the prefill batches;
  all outputs);
* production dtype output: the same bound plus one output unit roundoff;
* run-to-run bitwise determinism and per-token batch invariance.
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


def oracle_y(L, xbits, xdt):
    return orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in,
                      L.s_out, xbits, xdt == "bf16", cb2=L.cb2_f16)


def x_to_f64(xbits, xdt):
    if xdt == "f16":
        return xbits.view(np.float16).astype(np.float64)
    return (xbits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


SMALL = [  # m, n, bpw, B, x dtype -- several tiles, ragged row / column tails
    (16, 128, 2, 1, "f16"), (40, 200, 2, 3, "f16"), (272, 264, 4, 5, "bf16"),
    (64, 1024, 3, 8, "f16"), (1000, 968, 4, 9, "bf16"), (24, 56, 3, 16, "bf16"),
    (520, 136, 2, 16, "f16"), (8, 8, 4, 2, "f16"), (264, 520, 3, 13, "bf16"),
]


@pytest.mark.parametrize("m,n,bpw,B,xdt", SMALL)
def test_dequant_bit_exact_small(dev, m, n, bpw, B, xdt):
    L = gi.make_layer(m + n, 3, m, n, bpw)
    lay = dev.layer(L)
    w = lay.dequant().cpu().numpy().astype(np.float64)
    ref = orc.decode_rows(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, cb2=L.cb2_f16)
    np.testing.assert_array_equal(w, ref)


@pytest.mark.parametrize("m,n,bpw,B,xdt", SMALL)
def test_linear_small(dev, m, n, bpw, B, xdt):
    L = gi.make_layer(m * 7 + n, 1, m, n, bpw)
    xb = gi.make_x(m * 7 + n, 1, B, n, xdt)
    lay = dev.layer(L)
    x = to_torch_x(xb, xdt)
    y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    ref = oracle_y(L, xb, xdt)
    err = np.max(np.abs(y - ref))
    assert err <= tolerance(ref), (err, tolerance(ref))
    # production dtype
    yp = lay(x).float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(yp - ref) <= production_tolerance(ref, xdt))


@pytest.mark.parametrize("n", [8, 24, 56, 64, 200, 960, 1024, 2560, 5120, 11008, 14336, 32768])
def test_rht_input_matches_dense_hadamard(dev, n):
    m = 8
    L = gi.make_layer(n, 0, m, n, 2)
    xb = gi.make_x(n, 0, 3, n, "bf16")
    lay = dev.layer(L)
    xr = lay.rht_input(to_torch_x(xb, "bf16")).cpu().numpy().astype(np.float64)
    xf = x_to_f64(xb, "bf16") * L.s_in
    for b in range(3):
        ref = orc.hadamard_apply(xf[b])
        np.testing.assert_allclose(xr[b], ref, rtol=0, atol=1e-5 * (np.abs(ref).max() + 1))


@pytest.mark.parametrize("B", [2, 5])
@pytest.mark.parametrize("m", [8, 24, 56, 64, 200, 960, 2048, 4096, 5120, 11008, 14336, 32768])
def test_rht_output_matches_dense_hadamard(dev, m, B):
    """The output stage as glq_linear runs it at this batch (the row kernel
    for rows up to 16384, except one or two rows longer than 8192): fp32
    output within 1e-5 of the dense fp64 transform, 16-bit outputs within one
    rounding of that."""
    n = 8
    L = gi.make_layer(m, 0, m, n, 2)
    rng = np.random.default_rng(m + B)
    z = rng.standard_normal((B, m)).astype(np.float32)
    lay = dev.layer(L)
    zc = torch.from_numpy(z).cuda()
    y = lay.rht_output(zc).cpu().numpy().astype(np.float64)
    refs = [orc.hadamard_apply(z[b].astype(np.float64)) * L.s_out for b in range(B)]
    for b in range(B):
        np.testing.assert_allclose(y[b], refs[b], rtol=0, atol=1e-5 * (np.abs(refs[b]).max() + 1))
    for dt, u in ((torch.bfloat16, 2.0 ** -8), (torch.float16, 2.0 ** -11)):
        yh = lay.rht_output(zc, out_dtype=dt).float().cpu().numpy().astype(np.float64)
        for b in range(B):
            bound = u * np.abs(refs[b]) + 2e-5 * (np.abs(refs[b]).max() + 1)
            assert np.all(np.abs(yh[b] - refs[b]) <= bound), (dt, b)


def _workload_cases():
    cases = []
    for key, wl in gi.WORKLOADS.items():
        for li, spec in enumerate(wl.layers):
            for B in wl.batches:
                cases.append((key, li, B))
    return cases


_LAYERS = {}


def _workload_layer(dev, key, li):
    """Host inputs and device layer of one workload layer, built once (the
    layers of the previous workload are released first)."""
    if any(k != key for k, _ in _LAYERS):
        _LAYERS.clear()
    if (key, li) not in _LAYERS:
        L = gi.workload_layer(gi.WORKLOADS[key], li)
        _LAYERS[(key, li)] = (L, dev.layer(L))
    return _LAYERS[(key, li)]


@pytest.mark.parametrize("key,li,B", _workload_cases())
def test_linear_workloads_full_size(dev, key, li, B):
    """Every layer of every workload at full size and at every batch the
    workload names, on the workload's own seeded inputs (the ones the
    benchmark times).  Decode batches (B <= 16): every token and every
    output against the oracle.  Prefill batches: a seeded sample of tokens
    that includes the first, the last and both sides of the first 512-token
    tile boundary, all m outputs each.  fp32 output within
    2e-3 (||y||_inf + 1); the production dtype within that bound plus one
    output rounding.  The first batch of each layer also checks sampled rows
    of the dequantised W^ bit-exactly."""
    wl = gi.WORKLOADS[key]
    L, lay = _workload_layer(dev, key, li)
    xb = gi.workload_x(wl, li, B)
    x = to_torch_x(xb, wl.x_dtype)
    y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    yp = lay(x).float().cpu().numpy().astype(np.float64)
    if B <= 16:
        sample = list(range(B))
    else:
        rng = np.random.default_rng(1000 * li + B)
        sample = sorted(set([t for t in (0, 511, 512) if t < B] + [B - 1] +
                            [int(t) for t in rng.choice(B, size=3, replace=False)]))
    ref = orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out,
                     xb[sample], wl.x_dtype == "bf16", cb2=L.cb2_f16, threads=0)
    err = np.max(np.abs(y[sample] - ref))
    print(f"\nPARITY {key} layer {li} ({L.m}x{L.n}) B={B} tokens {len(sample)}: max err {err:.3e} "
          f"tol {tolerance(ref):.3e} ratio {err / tolerance(ref):.3f}")
    assert err <= tolerance(ref), (err, tolerance(ref))
    assert np.all(np.abs(yp[sample] - ref) <= production_tolerance(ref, wl.x_dtype))
    if B == wl.batches[0]:
        rng = np.random.default_rng(li)
        w = lay.dequant()
        rows = sorted(set([0, L.m - 1] + [int(r) for r in rng.choice(L.m, size=8, replace=False)]))
        wr = w[rows].cpu().numpy().astype(np.float64)
        del w
        for i, r in enumerate(rows):
            ref_w = orc.decode_rows(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale,
                                    r, r + 1, cb2=L.cb2_f16)
            np.testing.assert_array_equal(wr[i], ref_w[0])


def test_determinism_and_batch_invariance(dev):
    """Run to run: bitwise on both decode paths.  Per token across batch
    sizes: bitwise for every B <= 16 with the transforms as separate kernels;
    with fusion on, within B <= 8 (fused here: 8 x 4096 values) and within
    9 <= B <= 16 (separate kernels here)."""
    wl = gi.WORKLOADS["24b-decode-4bpw"]
    L = gi.workload_layer(wl, 0)
    lay = dev.layer(L)
    xb = gi.workload_x(wl, 0, 16)
    x = to_torch_x(xb, "bf16")
    y16 = lay(x, out_dtype=torch.float32)
    assert torch.equal(y16, lay(x, out_dtype=torch.float32))
    y8 = lay(x[:8].contiguous(), out_dtype=torch.float32)
    assert torch.equal(y8, lay(x[:8].contiguous(), out_dtype=torch.float32))
    for B in (1, 2, 4):
        assert torch.equal(lay(x[:B].contiguous(), out_dtype=torch.float32), y8[:B]), B
    for B in (9, 12):
        assert torch.equal(lay(x[:B].contiguous(), out_dtype=torch.float32), y16[:B]), B
    lay.set_fusion(0)
    try:
        s16 = lay(x, out_dtype=torch.float32)
        assert torch.equal(s16, y16)  # B = 16 took the separate kernels before too
        for B in (1, 2, 4, 8):
            assert torch.equal(lay(x[:B].contiguous(), out_dtype=torch.float32), s16[:B]), B
    finally:
        lay.set_fusion(-1)


FUSION_CASES = [  # m, n, bpw, B, x dtype: fused input and output transforms when aligned
    (2048, 2048, 4, 1, "bf16"), (11008, 2048, 4, 1, "bf16"), (2048, 11008, 4, 1, "bf16"),
    (960, 2560, 3, 2, "f16"), (2560, 960, 3, 8, "f16"), (1024, 1024, 2, 16, "f16"),
    (4096, 5120, 4, 4, "bf16"), (5120, 32768, 2, 1, "bf16"), (32768, 1024, 2, 1, "f16"),
    (136, 8200, 4, 3, "bf16"),
]


@pytest.mark.parametrize("m,n,bpw,B,xdt", FUSION_CASES)
def test_fused_and_separate_transforms(dev, m, n, bpw, B, xdt):
    """The same layer with the transforms fused into the GEMV launch and as
    separate kernels, and each one alone (glq_layer_set_fusion): all within
    the bound of the oracle, every token and output."""
    L = gi.make_layer(m + 3 * n, 2, m, n, bpw)
    xb = gi.make_x(m + 3 * n, 2, B, n, xdt)
    lay = dev.layer(L)
    ref = oracle_y(L, xb, xdt)
    x = to_torch_x(xb, xdt)
    errs = []
    for flags in (3, 1, 2, 0):  # both fused, input only, output only, neither
        lay.set_fusion(flags)
        y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
        errs.append(np.max(np.abs(y - ref)))
        assert errs[-1] <= tolerance(ref), (flags, errs[-1], tolerance(ref))
    lay.set_fusion(-1)
    print(f"\nFUSION {m}x{n} bpw {bpw} B={B}: ratios to tol (both, in, out, none) "
          + " ".join(f"{e / tolerance(ref):.3f}" for e in errs))


CLUSTER_CASES = [  # m, n, bpw, B, x dtype
    (2048, 2048, 4, 1, "bf16"), (11008, 2048, 4, 1, "bf16"), (2048, 11008, 4, 1, "bf16"),
    (4096, 5120, 4, 1, "bf16"), (32768, 5120, 4, 1, "bf16"), (960, 2560, 3, 2, "f16"),
    (2560, 960, 3, 8, "f16"), (1024, 1024, 2, 16, "f16"), (1000, 968, 4, 9, "bf16"),
    (5120, 4096, 4, 16, "bf16"),
]


@pytest.mark.parametrize("m,n,bpw,B,xdt", CLUSTER_CASES)
def test_cluster_splitk_matches_global_reduction(dev, m, n, bpw, B, xdt):
    """Split-K partial sums added through a thread-block cluster's distributed
    shared memory (GLQ_SPLITK_CLUSTER) give the same bits as the global
    workspace and last-arriving CTA (the summation order is the same), with
    the input transform fused and as its own kernel; the result is within the
    oracle bound."""
    L = gi.make_layer(7 * m + n, 3, m, n, bpw)
    xb = gi.make_x(7 * m + n, 3, B, n, xdt)
    lay = dev.layer(L)
    x = to_torch_x(xb, xdt)
    plans = []
    for fin in (1, 0):
        lay.set_fusion(fin | 4)
        plans.append(lay.decode_plan(B))
        yc = lay(x, out_dtype=torch.float32)
        lay.set_fusion(fin)
        assert lay.decode_plan(B)["cluster"] == 0
        yg = lay(x, out_dtype=torch.float32)
        assert torch.equal(yc, yg), (fin, plans[-1])
    lay.set_fusion(-1)
    y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    ref = oracle_y(L, xb, xdt)
    assert np.max(np.abs(y - ref)) <= tolerance(ref)
    print(f"\nCLUSTER {m}x{n} bpw {bpw} B={B}: plans (fused, separate) {plans}, default {lay.decode_plan(B)}")


def test_decode_plans_of_the_workloads(dev):
    """The decode plans of the SmolLM3-3B-shaped and 24B-class layers at 1 and
    16 tokens are consistent (a cluster, when used, holds a band's splits),
    the cluster reduction is in use on some of them, and at one token the
    3B-shaped layers fuse the input transform exactly when the row is
    longer than 8192.  At 16 tokens the
    32768-row gate / up layers (128 bands of 16-warp CTAs on 148 SMs) take one
    split: charged too little for the global reduction of two token tiles,
    the planner chose 8 splits over 7 waves there, 1.6x slower per step."""
    clustered = 0
    for key in ("smollm3-3b-4bpw", "24b-decode-4bpw"):
        wl = gi.WORKLOADS[key]
        for li in range(len(wl.layers)):
            L = gi.workload_layer(wl, li)
            lay = dev.layer(L)
            for B in (1, 16):
                plan = lay.decode_plan(B)
                assert plan["cluster"] in (0, plan["splits"]) and plan["cluster"] != 1, (key, li, B, plan)
                clustered += plan["cluster"] > 0
                if B == 16 and L.m == 32768 and torch.cuda.get_device_properties(0).multi_processor_count == 148:
                    assert plan["splits"] == 1, (key, li, plan)
                if B == 1 and key == "smollm3-3b-4bpw":
                    # the input transform is fused only for rows longer than
                    # 8192 (down: 11008 columns); shorter rows run it as its
                    # own kernel, launched early behind the previous one
                    assert plan["fused_input"] == (1 if L.n > 8192 else 0), (key, li, plan)
                print(f"\nPLAN {key} layer {li} B={B}: {plan}")
    assert clustered > 0


def test_empty_batch_and_errors(dev):
    import e8_lattice_codebook_b200 as glq
    L = gi.make_layer(0, 0, 64, 64, 2)
    lay = dev.layer(L)
    x = torch.zeros((0, 64), dtype=torch.float16, device="cuda")
    y = lay(x)
    assert y.shape == (0, 64)
    xx = torch.zeros((2, 64), dtype=torch.float16, device="cuda")
    yy = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(glq.GlqError) as e:
        glq.glq_linear(lay.handle, xx.data_ptr(), glq.GLQ_F16, yy.data_ptr(), glq.GLQ_BF16, 2,
                       torch.cuda.current_stream().cuda_stream)
    # a pointer that is not 16-byte aligned is rejected before any launch
    yh = torch.zeros((2, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(glq.GlqError) as e2:
        glq.glq_linear(lay.handle, xx.data_ptr() + 2, glq.GLQ_F16, yh.data_ptr(), glq.GLQ_F16, 1,
                       torch.cuda.current_stream().cuda_stream)
    assert e2.value.status == 1  # INVALID_ARG
    assert e.value.status == 3  # DTYPE
    lay.check()
