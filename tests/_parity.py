"""Comparison rules between the CUDA path and the float64 oracle.

Output O: |gpu - oracle| <= tol elementwise (2e-3 fp16, 1.5e-2 bf16), or, where
that tolerance is tighter than the 16-bit format can represent at |oracle|,
|gpu - oracle| < 1 ulp of the format at |oracle| (a faithful rounding).
LSE: |gpu - oracle| <= 1e-4 where finite; -inf exactly where the oracle has it.
Gradients: relative Frobenius error <= 1e-2.
"""

import math

import numpy as np
import torch

O_TOL = {torch.float16: 2e-3, torch.bfloat16: 1.5e-2}
MANT = {torch.float16: 10, torch.bfloat16: 7}
LSE_TOL = 1e-4
GRAD_TOL = 1e-2


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def ulp(x, dtype):
    ax = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(ax)) - MANT[dtype])


def check_out(gpu, ref, dtype, what="O"):
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    err = np.abs(g - ref)
    tol = O_TOL[dtype]
    ok = (err <= tol) | (err < ulp(ref, dtype))
    n_bad = int((~ok).sum())
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    assert n_bad == 0, (f"{what}: {n_bad}/{ok.size} elements outside tolerance; max err {err.max():.3e} "
                        f"(tol {tol})")
    return dict(max_err=float(err.max()), n_faithful_only=int(((err > tol) & ok).sum()))


def check_lse(gpu, ref):
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    ninf_r = np.isneginf(ref)
    assert (np.isneginf(g) == ninf_r).all(), "LSE: -inf pattern differs"
    fin = ~ninf_r
    if fin.any():
        err = np.abs(g[fin] - ref[fin]).max()
        assert err <= LSE_TOL, f"LSE max err {err:.3e}"
        return float(err)
    return 0.0


def rel_fro(gpu, ref):
    """||gpu - ref|| / max(||ref||, 1e-3 * sqrt(n)).

    The floor (an RMS of 1e-3) only matters when the exact gradient is
    (nearly) zero, e.g. dQ and dK with a single key, where P = 1 and
    dS = P (dP - Delta) = 0 exactly; a relative error is undefined there.
    """
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    den = max(np.linalg.norm(ref), 1e-3 * math.sqrt(max(ref.size, 1)))
    return float(np.linalg.norm(g - ref) / den)


def check_grad(gpu, ref, what):
    e = rel_fro(gpu, ref)
    assert e <= GRAD_TOL, f"{what}: relative Frobenius error {e:.3e}"
    return e
