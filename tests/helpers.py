"""Shared helpers for the parity tests (no method arithmetic here)."""

import numpy as np
import torch


def f32(t: torch.Tensor) -> np.ndarray:
    """bf16/float tensor (any device) -> float32 numpy array (exact for bf16)."""
    return t.detach().float().cpu().numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.uint8)


def rms(a: np.ndarray) -> float:
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


# Tolerance on every floating-point output of the linear layer: the maximum
# absolute error may not exceed 2e-2 times the RMS of the float64 oracle.
REL_RMS_TOL = 2e-2


def assert_close_rms(got, ref, name: str, tol: float = REL_RMS_TOL) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    scale = rms(ref)
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    bound = tol * scale
    assert err <= bound, f"{name}: max abs err {err:.3e} > {tol} * rms {scale:.3e}"
    return err / scale if scale > 0 else 0.0
