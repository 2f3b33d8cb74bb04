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


# Bound for stress inputs whose softmax is nearly one-hot, so the output is
# close to a single V row of magnitude up to ~5. Rounding each probability to
# bf16 (8 significant bits) moves the weighted sum by up to 2^-9 * sum p|v|/l,
# at most ~1e-2 for |v| <= 5, covered by the 2e-2 absolute term; rounding the
# output itself costs up to 2^-8 |out| on top.
STRESS_ATOL = 2e-2
STRESS_RTOL = 2.0 ** -8


def compare_rel(got: np.ndarray, ref: np.ndarray, what: str = "", atol: float = STRESS_ATOL,
                rtol: float = STRESS_RTOL):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "%s: non-finite output" % what
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    worst = np.unravel_index(int(np.argmax(err - bound)), err.shape)
    assert np.all(err <= bound), "%s: err %.3e > bound %.3e at %s (ref %.4f)" % (
        what, err[worst], bound[worst], worst, ref[worst])
    return float(err.max())
