"""Helpers shared by the GPU parity tests: host<->device bf16 transfers and
the comparison metrics against the fp64 oracle."""
import numpy as np
import torch

import synth

# Tolerances for bf16 output with fp32 accumulation against the fp64 oracle.
MAX_ABS_TOL = 2e-2
MEAN_ABS_TOL = 2e-3


def bits_to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 CUDA tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev_to_f64(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> exact fp64 numpy values."""
    bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return synth.bf16_bits_to_f64(bits)


def compare(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Assert the max-abs and mean-abs bars; returns (max_abs, mean_abs, argmax index)."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "%s: non-finite output" % what
    err = np.abs(got - ref)
    mx = float(err.max())
    mean = float(err.mean())
    where = np.unravel_index(int(err.argmax()), err.shape)
    assert mx <= MAX_ABS_TOL, "%s: max abs err %.3e at %s (tol %.1e)" % (what, mx, where, MAX_ABS_TOL)
    assert mean <= MEAN_ABS_TOL, "%s: mean abs err %.3e (tol %.1e)" % (what, mean, MEAN_ABS_TOL)
    return mx, mean, where
