"""Helpers shared by the GPU parity tests: moving seeded inputs to the device, reading results back
in the oracle's formats, and the tolerance check for GEMM outputs.

Tolerances:
  * layouts, AllGather, fp32 and bf16 ring reductions: bit-exact (the oracle emulates the same
    binary32 adds in the same order and the same single rounding to bf16);
  * GEMM-derived outputs (bf16 inputs, fp32 accumulation): max|gpu - oracle_fp64| <= 2e-2 * max|oracle|,
    the tolerance the workload specification states. For fp32-output GEMMs an additional bound
    derived from the arithmetic is checked: accumulating K exactly-representable products in binary32
    errs by at most about K * 2^-24 * sum|a||b|; tests use 1e-3 * max|oracle|, far above that for the
    K used and far below any indexing mistake.
"""
from __future__ import annotations

import numpy as np
import torch

import synthetic as S

GEMM_TOL = 2e-2
FP32_GEMM_TOL = 1e-3


def cuda(x: torch.Tensor) -> torch.Tensor:
    return x.to("cuda", non_blocking=False).contiguous()


def host_bits(x: torch.Tensor) -> np.ndarray:
    """Oracle format of a device tensor: float32 array, or uint16 bits for bf16."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return S.bf16_bits(x)
    return x.numpy().copy()


def f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().to(torch.float64).numpy()


def max_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref))) / (scale if scale > 0 else 1.0)


def assert_close(got, ref, tol=GEMM_TOL, what=""):
    err = max_rel_err(got, ref)
    assert err <= tol, f"{what}: max|err|/max|ref| = {err:.3e} > {tol:.1e}"
    return err


def same_bits(a: np.ndarray, b: np.ndarray) -> bool:
    a, b = np.ascontiguousarray(a), np.ascontiguousarray(b)
    if a.shape != b.shape or a.dtype.itemsize != b.dtype.itemsize:
        return False
    view = np.uint32 if a.dtype.itemsize == 4 else np.uint16
    return bool(np.array_equal(a.view(view), b.view(view)))
