"""Tolerance checks of GPU results against the fp64 oracle.

fp32 path: max|err| <= 1e-4 * max|ref|.
bf16 path (fp32 accumulation and state): max|err| <= 2e-2 * max|ref| and
||err||_2 / ||ref||_2 <= 5e-3.  Each bound applies to O, to Y (pre-norm test
path) and to the final state separately.
"""
import numpy as np
import torch

TOL = {"f32": dict(max_rel=1e-4, l2_rel=None), "bf16": dict(max_rel=2e-2, l2_rel=5e-3)}


def f64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def errors(got, ref):
    got, ref = f64(got), f64(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite GPU output"
    err = got - ref
    mx = float(np.max(np.abs(ref))) if ref.size else 0.0
    max_rel = float(np.max(np.abs(err))) / mx if mx > 0 else float(np.max(np.abs(err)))
    nr = float(np.linalg.norm(ref.ravel()))
    l2_rel = float(np.linalg.norm(err.ravel())) / nr if nr > 0 else float(np.linalg.norm(err.ravel()))
    return max_rel, l2_rel


def assert_close(got, ref, io, what=""):
    max_rel, l2_rel = errors(got, ref)
    tol = TOL[io]
    assert max_rel <= tol["max_rel"], f"{what}: max|err|/max|ref| = {max_rel:.3e} > {tol['max_rel']}"
    if tol["l2_rel"] is not None:
        assert l2_rel <= tol["l2_rel"], f"{what}: L2 rel err = {l2_rel:.3e} > {tol['l2_rel']}"
    return max_rel, l2_rel
