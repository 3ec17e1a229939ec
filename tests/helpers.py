"""Helpers shared by the GPU parity tests (no method arithmetic here).

Tolerance for Y (bf16) against the oracle's binary64 matmul Y64:
  max bar        max|Y − Y64| ≤ 4e-3 · max|Y64|            (Y64 as computed, unrounded)
  Frobenius bar  ‖Y − bf16(Y64)‖_F ≤ 1e-3 · ‖bf16(Y64)‖_F   (Y64 rounded to Y's format)
Rounding any result to bf16 costs about 1.7e-3 relative Frobenius against the
unrounded sum, so the Frobenius bar is taken against the sum rounded to bf16;
against that rounded sum, though, a single correct-but-opposite rounding of a
near-tie output in the top binade moves the max error by one bf16 ulp
(2^-8..2^-7 of max|Y|), so the max bar is taken against the unrounded sum,
where any output rounded from an accurate fp32 sum stays within 2^-8.
"""
import numpy as np
import torch

import oracle
import workloads

MAX_REL = 4e-3
FRO_REL = 1e-3


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(
        np.float32).astype(np.float64)


def y_errors(Y_gpu_bits: np.ndarray, Y64: np.ndarray):
    """(max error / max|Y64|, Frobenius error vs bf16(Y64) / ‖bf16(Y64)‖)."""
    y = bits_to_f64(Y_gpu_bits).ravel()
    r64 = np.asarray(Y64, dtype=np.float64).ravel()
    rb = bits_to_f64(oracle.bf16_from_f64(r64))
    assert np.all(np.isfinite(y)), "non-finite output"
    amax = np.max(np.abs(r64))
    fro = np.linalg.norm(rb)
    emax = np.max(np.abs(y - r64))
    efro = np.linalg.norm(y - rb)
    return (emax / amax if amax > 0 else emax, efro / fro if fro > 0 else efro)


def assert_y_close(Y_gpu_bits, Y64, what=""):
    emax, efro = y_errors(Y_gpu_bits, Y64)
    assert emax <= MAX_REL and efro <= FRO_REL, f"{what}: max rel {emax:.3e}, fro rel {efro:.3e}"
    return emax, efro
