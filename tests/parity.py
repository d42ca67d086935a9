"""Shared parity helpers for the GPU tests.

Tolerances (per element, GPU vs the fp64 oracle on identical seeded inputs):
  * bf16 tensors, fp32 accumulation: max-abs <= 3e-2 and mean-abs <= 3e-3;
  * fp32 tensors: max-abs <= 1e-4 and mean-abs <= 1e-4.
Index work (key sets, cache layout) is compared bit-exactly.
"""
import numpy as np
import torch

TOL = {"bf16": (3e-2, 3e-3), "f32": (1e-4, 1e-4)}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(gpu, ref, dtype, what=""):
    g = to64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), "%s: non-finite GPU output" % what
    err = np.abs(g - r)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    tmax, tmean = TOL[dtype]
    assert mx <= tmax and mean <= tmean, "%s: max-abs %.3g (<= %.1g), mean-abs %.3g (<= %.1g)" % (
        what, mx, tmax, mean, tmean)
    return mx, mean


def bits_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    a = a.contiguous().cpu()
    b = b.contiguous().cpu()
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)
