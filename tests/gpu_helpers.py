"""Shared helpers of the GPU parity tests: build device layers from the
seeded host inputs, and the tolerance of the layer output."""
import numpy as np

import glq_inputs as gi


def tolerance(y_ref: np.ndarray) -> float:
    """max |y_gpu - y_oracle| <= 2e-3 (||y_oracle||_inf + 1)  (fp32 output)."""
    return 2e-3 * (float(np.max(np.abs(y_ref))) + 1.0) if y_ref.size else 0.0


def production_tolerance(y_ref: np.ndarray, dtype: str) -> np.ndarray:
    """The fp32 bound plus one unit roundoff of the output dtype per element."""
    u = 2.0 ** -11 if dtype == "f16" else 2.0 ** -8
    return tolerance(y_ref) + u * np.abs(y_ref)


class Device:
    """Codebooks shared by the layers of one test module."""

    def __init__(self):
        import e8_lattice_codebook_b200 as glq
        self.glq = glq
        self.e8 = glq.Codebook.e8()

    def layer(self, L: gi.LayerInputs):
        glq = self.glq
        res = None
        if L.bpw % 2:
            res = glq.Codebook(L.cb2_f16.reshape(256, 8))
        elif L.bpw == 4:
            res = self.e8
        return glq.GlqLinear(L.m, L.n, L.bpw, L.idx1, L.idx2, self.e8, res,
                             L.weight_scale, L.resid_scale, L.s_in, L.s_out)


def to_torch_x(xbits: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(xbits).view(np.int16).copy()).cuda()
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16)
