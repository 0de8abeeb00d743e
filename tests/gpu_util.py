"""Helpers for the GPU parity tests: move synth inputs to the device, run the
CUDA library through its C ABI, and compare with the oracle.

Tolerances (fp32 accumulation on the GPU, the oracle in double): the maximum
absolute error over a tensor must not exceed 1e-5 * max|reference| for fp32
storage and 1e-2 * max|reference| for bf16 storage.
"""
import numpy as np

import linear_spatial_propagation_b200 as lsp
import synth

TOL = {"f32": 1e-5, "bf16": 1e-2}


def torch():
    import torch as t
    return t


def to_dev(a: np.ndarray, dtype: str, device="cuda"):
    t = torch()
    if dtype == "bf16":
        return t.from_numpy(np.ascontiguousarray(a, dtype=np.uint16)).view(t.bfloat16).to(device)
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def from_dev(x) -> np.ndarray:
    t = torch()
    if x.dtype == t.bfloat16:
        return synth.bf16_bits_to_f32(x.view(t.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return x.float().cpu().numpy().astype(np.float64)


def dev_inputs(w, inp):
    return {k: to_dev(v, w.dtype) for k, v in inp.items()}


def run_fwd(w, dinp, out=None, ws=None):
    return lsp.forward(dinp["x"], dinp["logits"], dinp["lam"], dir_mask=w.dir_mask, groups=w.groups,
                       shared=w.shared, out=out, ws=ws)


def run_bwd(w, dinp):
    return lsp.backward(dinp["x"], dinp["logits"], dinp["lam"], dinp["dout"], dir_mask=w.dir_mask,
                        groups=w.groups, shared=w.shared)


def max_err(got: np.ndarray, want: np.ndarray):
    err = float(np.max(np.abs(got - want))) if got.size else 0.0
    ref = float(np.max(np.abs(want))) if want.size else 0.0
    return err, ref


def assert_close(got, want, dtype, what=""):
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err, ref = max_err(got, want)
    assert err <= TOL[dtype] * ref + 1e-30, f"{what}: max-abs err {err:.3e} > {TOL[dtype]:g} * {ref:.3e}"
    return err / ref if ref else 0.0
