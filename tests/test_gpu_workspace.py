"""The device's shared workspace and graph capture, through the C ABI.

* glq_layer_reserve covers decode (B <= 16) and tensor-core (B > 16) calls:
  after it, a decode call and a prefill call (W reconstructed in fp16) are
  captured together in one CUDA graph and replayed, and both outputs match
  the fp64 oracle; the workspace does not grow while capturing or replaying;
* a call that would need a larger workspace while its stream is being
  captured returns GLQ_ERR_CAPTURE and launches nothing (the capture stays
  valid);
* a layer's own device memory stays within 1.1x its index bytes after a
  prefill call: the reconstructed W and every other transient buffer live in
  the one shared workspace of the device, whose size glq_workspace_info
  reports (one W of the largest layer, not one per layer).
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


def _oracle(L, xb, xdt):
    return orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out,
                      xb, xdt == "bf16", cb2=L.cb2_f16, threads=0)


def _index_bytes(L):
    return L.m * L.n * L.bpw // 8


def test_decode_and_prefill_captured_in_one_graph(dev):
    import e8_lattice_codebook_b200 as glq
    glq.glq_workspace_release(torch.cuda.current_device())
    Ld = gi.make_layer(31, 0, 2048, 2048, 4)      # decode layer, 4 bpw
    Lp = gi.make_layer(31, 1, 3072, 1536, 3)      # prefill layer, 3 bpw (256-entry residual)
    dl, pl = dev.layer(Ld), dev.layer(Lp)
    Bd, Bp = 4, 600                               # 600 >= 256: W reconstructed once per call
    dl.reserve(Bd)
    pl.reserve(Bp)
    ws0 = glq.glq_workspace_info(torch.cuda.current_device())
    assert ws0 >= Lp.m * Lp.n * 2  # the reconstructed fp16 W of the prefill layer is in it
    xbd = gi.make_x(31, 0, Bd, Ld.n, "bf16")
    xbp = gi.make_x(31, 1, Bp, Lp.n, "f16")
    xd, xp = to_torch_x(xbd, "bf16"), to_torch_x(xbp, "f16")
    yd = torch.empty((Bd, Ld.m), dtype=torch.float32, device="cuda")
    yp = torch.empty((Bp, Lp.m), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm the launch paths outside capture
        dl(xd, out=yd)
        pl(xp, out=yp)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dl(xd, out=yd)
        pl(xp, out=yp)
    yd.fill_(float("nan"))
    yp.fill_(float("nan"))
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    dl.check()
    pl.check()
    assert glq.glq_workspace_info(torch.cuda.current_device()) == ws0
    refd, refp = _oracle(Ld, xbd, "bf16"), _oracle(Lp, xbp, "f16")
    ed = np.max(np.abs(yd.cpu().numpy().astype(np.float64) - refd))
    ep = np.max(np.abs(yp.cpu().numpy().astype(np.float64) - refp))
    print(f"\nGRAPH decode err {ed:.3e} tol {tolerance(refd):.3e}; prefill err {ep:.3e} tol {tolerance(refp):.3e}")
    assert ed <= tolerance(refd)
    assert ep <= tolerance(refp)
    # the layers hold their indices and little else, the W of the prefill included
    for L, lay in ((Ld, dl), (Lp, pl)):
        _, _, _, nbytes = glq.glq_layer_info(lay.handle)
        assert nbytes <= 1.1 * _index_bytes(L), (nbytes, _index_bytes(L))
    del g


def test_growth_during_capture_is_refused(dev):
    import e8_lattice_codebook_b200 as glq
    glq.glq_workspace_release(torch.cuda.current_device())
    L = gi.make_layer(32, 0, 1024, 1024, 2)
    lay = dev.layer(L)
    lay.reserve(2)
    x = to_torch_x(gi.make_x(32, 0, 400, L.n, "f16"), "f16")
    y = torch.empty((400, L.m), dtype=torch.float16, device="cuda")
    lay(x[:2], out=y[:2])  # warm
    torch.cuda.synchronize()
    ws0 = glq.glq_workspace_info(torch.cuda.current_device())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lay(x[:2], out=y[:2])
        with pytest.raises(glq.GlqError) as e:
            lay(x, out=y)  # 400 tokens were never reserved
    assert e.value.status == 11  # GLQ_ERR_CAPTURE
    g.replay()
    torch.cuda.synchronize()
    assert glq.glq_workspace_info(torch.cuda.current_device()) == ws0
    ref = _oracle(L, gi.make_x(32, 0, 400, L.n, "f16")[:2], "f16")
    assert np.max(np.abs(y[:2].float().cpu().numpy() - ref)) <= tolerance(ref) + 2 ** -11 * np.abs(ref).max()
    lay(x, out=y)  # outside capture the workspace grows
    torch.cuda.synchronize()
    assert glq.glq_workspace_info(torch.cuda.current_device()) > ws0
    del g


def test_many_layers_share_one_workspace(dev):
    """Ten prefill layers reconstructing W: the workspace holds one W (of
    the largest), not ten."""
    import e8_lattice_codebook_b200 as glq
    glq.glq_workspace_release(torch.cuda.current_device())
    layers = []
    for i in range(10):
        L = gi.make_layer(40 + i, 0, 1024 + 128 * i, 1024, 4)
        layers.append((L, dev.layer(L)))
    for i, (L, lay) in enumerate(layers):
        x = to_torch_x(gi.make_x(40 + i, 0, 300, L.n, "bf16"), "bf16")
        lay(x)
    torch.cuda.synchronize()
    ws = glq.glq_workspace_info(torch.cuda.current_device())
    biggest_w = max(L.m for L, _ in layers) * 1024 * 2
    assert ws < 3 * biggest_w, (ws, biggest_w)
    assert ws < sum(L.m * L.n * 2 for L, _ in layers) / 3
