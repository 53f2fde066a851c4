"""Helpers shared by the GPU parity tests: error metric and tolerances.

Tolerances (relative L2 error over a whole output tensor, ||x - ref|| / ||ref||):
  fp32 inputs            1e-5   (CUDA-core FFMA path)
  bf16 inputs, fp32 acc  2e-2
The oracle reads exactly the values the kernel reads (bf16 inputs widened to
fp64), so the error measured is the kernel's arithmetic only.
"""
import numpy as np
import torch

TOL_F32 = 1e-5
TOL_BF16 = 2e-2


def tol_for(dtype) -> float:
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def rel_l2(x, ref) -> float:
    x = x.detach().to("cpu", torch.float64).numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def assert_close(x, ref, dtype, what=""):
    err = rel_l2(x, ref)
    tol = tol_for(dtype)
    assert np.all(np.isfinite(x.detach().float().cpu().numpy() if hasattr(x, "detach") else x)), f"{what}: non-finite"
    assert err <= tol, f"{what}: rel-L2 {err:.3e} > {tol:.0e}"
    return err
