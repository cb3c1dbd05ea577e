"""GPU parity of the tensor-core (prefill, B > 16 tokens) path of glq_linear
against the fp64 oracle, through the C ABI.

The path rounds the rotated activations and the reconstructed codewords
(cb1 + rs cb2) to fp16 once each and accumulates in fp32 on the tensor
cores, so it keeps the same bound as the decode path:
max |y - y_oracle| <= 2e-3 (||y_oracle||_inf + 1).

* small shapes: every token of batches that span one and several 512-token
  tiles, with ragged row, column and token tails, all three bit rates, rows
  longer than the one-CTA-per-row transforms take (16384), and input rows of
  every size the tensor-core transform takes (2^10 .. 2^14 positions, one
  to five Hadamard blocks);
* full-size prefill workload at its largest batch: sampled tokens, the last
  (ragged) token tile included;
* run-to-run determinism, and per-token independence of the batch size
  within the tensor-core path.
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


PREFILL_SMALL = [  # m, n, bpw, B, x dtype
    (16, 128, 2, 17, "f16"),        # one row tile, one column chunk, smallest prefill batch
    (272, 264, 4, 40, "bf16"),      # ragged rows (3 row tiles) and columns
    (1000, 968, 3, 33, "f16"),      # 8 row tiles, 3 bpw residual table
    (136, 1024, 2, 600, "bf16"),    # second token tile has one live accumulator
    (264, 520, 4, 777, "f16"),      # second token tile: one full and one ragged accumulator
    (200, 2560, 3, 300, "bf16"),    # long K (40 steps), ragged accumulator
    (8, 8, 4, 20, "f16"),           # tiny layer, most of the tile is padding
    (1024, 1024, 2, 1100, "bf16"),  # three token tiles
    (64, 20480, 2, 33, "f16"),      # input rows above 16384: clustered transform kernel
    (20480, 64, 3, 20, "bf16"),     # output rows above 16384: clustered transform kernel
    # input rows a multiple of 256: the tensor-core transform kernel
    (48, 768, 2, 40, "bf16"),       # 2^10 positions, two Hadamard blocks
    (40, 3840, 4, 33, "f16"),       # 2^12, four blocks
    (24, 7936, 3, 50, "bf16"),      # 2^13 (one cross-tile bit), five blocks
    (16, 12288, 2, 20, "f16"),      # 2^14 (two cross-tile bits), two blocks
    (16, 16384, 4, 19, "bf16"),     # 2^14, one block
    # 75 row tiles: one more than a wave of the 74 CTA pairs, so the last
    # tile runs as two half tiles (256 tokens each; the second one ragged)
    (19200, 128, 4, 300, "bf16"),
]


MODES = {"fused": 1 << 40, "reconstructed": 17}  # glq_layer_set_prefill_reconstruct bound


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("m,n,bpw,B,xdt", PREFILL_SMALL)
def test_prefill_small_all_tokens(dev, m, n, bpw, B, xdt, mode):
    """Both ways of feeding W: rebuilt per tile in shared memory (fused) and
    reconstructed once into an fp16 matrix (reconstructed)."""
    L = gi.make_layer(m * 11 + n, 7, m, n, bpw)
    xb = gi.make_x(m * 11 + n, 7, B, n, xdt)
    lay = dev.layer(L)
    lay.set_prefill_reconstruct(MODES[mode])
    x = to_torch_x(xb, xdt)
    y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    ref = oracle_y(L, xb, xdt)
    err = np.max(np.abs(y - ref))
    print(f"\nPREFILL {mode} {m}x{n} bpw {bpw} B={B}: max err {err:.3e} tol {tolerance(ref):.3e} "
          f"ratio {err / tolerance(ref):.3f}")
    assert err <= tolerance(ref), (err, tolerance(ref))
    yp = lay(x).float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(yp - ref) <= production_tolerance(ref, xdt))
    lay.check()  # no bounded device wait gave up


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("li", [0, 1])
def test_prefill_workload_largest_batch(dev, li, mode):
    wl = gi.WORKLOADS["prefill-8b-mlp-4bpw"]
    L = gi.workload_layer(wl, li)
    lay = dev.layer(L)
    lay.set_prefill_reconstruct(MODES[mode])
    B = max(wl.batches)
    xb = gi.workload_x(wl, li, B)
    x = to_torch_x(xb, wl.x_dtype)
    y = lay(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(100 + li)
    sample = sorted(set([0, 511, 512, B - 1] + list(rng.choice(B, size=3, replace=False))))
    ref = oracle_y(L, xb[sample], wl.x_dtype)
    err = np.max(np.abs(y[sample] - ref))
    print(f"\nPARITY prefill {mode} layer {li} ({L.m}x{L.n}) B={B}: max err {err:.3e} "
          f"tol {tolerance(ref):.3e} ratio {err / tolerance(ref):.3f}")
    assert err <= tolerance(ref), (err, tolerance(ref))
    assert np.all(np.isfinite(y))
    lay.check()


@pytest.mark.parametrize("mode", sorted(MODES))
def test_prefill_determinism_and_batch_independence(dev, mode):
    m, n, bpw = 520, 1032, 4
    L = gi.make_layer(5, 5, m, n, bpw)
    lay = dev.layer(L)
    lay.set_prefill_reconstruct(MODES[mode])
    xb = gi.make_x(5, 5, 700, n, "bf16")
    x = to_torch_x(xb, "bf16")
    y1 = lay(x, out_dtype=torch.float32)
    y2 = lay(x, out_dtype=torch.float32)
    assert torch.equal(y1, y2)
    for B in (17, 300, 512, 513):
        yb = lay(x[:B].contiguous(), out_dtype=torch.float32)
        assert torch.equal(yb, y1[:B]), B
    lay.check()


def test_producer_back_to_back_calls_do_not_stall(dev):
    """The dequantising-producer variant at small batches, six calls back to
    back on one stream: each must run to completion (no bounded device wait
    giving up).  Launched with programmatic dependent launch behind the
    previous call's kernels, such calls stalled for seconds until a wait's
    limit released them (GLQ_ERR_TIMEOUT); the variant now starts after its
    predecessor completes."""
    import time
    wl = gi.WORKLOADS["prefill-8b-mlp-4bpw"]
    L = gi.workload_layer(wl, 0)
    lay = dev.layer(L)
    lay.set_prefill_reconstruct(1 << 40)  # the producer for every batch
    for B in (17, 64):
        xb = gi.workload_x(wl, 0, B)
        x = to_torch_x(xb, wl.x_dtype)
        y = torch.empty((B, L.m), dtype=torch.float32, device="cuda")
        lay(x, out=y)
        torch.cuda.synchronize()
        t0 = time.time()
        for _ in range(6):
            lay(x, out=y)
        lay.check()  # raises GlqError(GLQ_ERR_TIMEOUT) if a wait gave up
        assert time.time() - t0 < 1.0, B
        ref = oracle_y(L, xb[[0, B - 1]], wl.x_dtype)
        assert np.max(np.abs(y.cpu().numpy().astype(np.float64)[[0, B - 1]] - ref)) <= tolerance(ref)
    lay.set_prefill_reconstruct(-1)


def test_half_tiles_keep_results_bitwise(dev):
    """A last partial wave of whole tiles runs as half tiles (one accumulator
    of 256 tokens each): the same K order, so a token's result does not
    depend on whether its tile was halved.  19200 rows are 75 row tiles:
    at 512 tokens the 75th tile is the partial wave and runs halved; at 600
    tokens (150 tiles, a ragged second token tile of 88 tokens) nothing is
    halved."""
    m, n, bpw = 19200, 256, 2
    L = gi.make_layer(41, 2, m, n, bpw)
    lay = dev.layer(L)
    xb = gi.make_x(41, 2, 600, n, "bf16")
    x = to_torch_x(xb, "bf16")
    for mode in sorted(MODES):
        lay.set_prefill_reconstruct(MODES[mode])
        y600 = lay(x, out_dtype=torch.float32)
        y512 = lay(x[:512].contiguous(), out_dtype=torch.float32)
        assert torch.equal(y512, y600[:512]), mode
        sample = [0, 255, 256, 511]
        ref = oracle_y(L, xb[sample], "bf16")
        err = np.max(np.abs(y512.cpu().numpy().astype(np.float64)[sample] - ref))
        assert err <= tolerance(ref), (mode, err)
        lay.check()
    lay.set_prefill_reconstruct(-1)


def test_single_accumulator_items_alternate_bitwise(dev):
    """Items with one live accumulator (a batch of at most 256 tokens, or the
    ragged 88 tokens of a second token tile) take a CTA pair's two TMEM
    accumulators in turn, so that one drains while the next item computes.
    19200 rows are 75 row tiles for 74 CTA pairs: at 200 tokens every item
    has one accumulator and the first pair takes two of them (accumulators 0
    then 1); at 600 tokens (150 items) whole tiles, which use both, and
    single ones (the ragged second token tile) mix, two or three items per
    pair.  A token's result does not depend on which accumulator held it."""
    m, n, bpw = 19200, 256, 2
    L = gi.make_layer(43, 2, m, n, bpw)
    lay = dev.layer(L)
    xb = gi.make_x(43, 2, 600, n, "f16")
    x = to_torch_x(xb, "f16")
    for mode in sorted(MODES):
        lay.set_prefill_reconstruct(MODES[mode])
        y600 = lay(x, out_dtype=torch.float32)
        y200 = lay(x[:200].contiguous(), out_dtype=torch.float32)
        assert torch.equal(y200, y600[:200]), mode
        sample = [0, 199, 511, 512, 599]
        ref = oracle_y(L, xb[sample], "f16")
        err = np.max(np.abs(y600.cpu().numpy().astype(np.float64)[sample] - ref))
        assert err <= tolerance(ref), (mode, err)
        lay.check()
    lay.set_prefill_reconstruct(-1)
