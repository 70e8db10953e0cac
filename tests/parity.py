"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerances (stated for this path; both sides get the same bf16-rounded inputs):
  * row norm: relative error <= 2e-3 for bf16 inputs, <= 1e-4 for fp32 inputs;
  * compose forward / backward outputs: |gpu - ref| <= 1e-2 |ref| + 1e-3;
  * near-unity forward (g - 1 ~ 1e-4): the same bound on y - base, with the
    bf16 output rounding taken into account (see ``near_unity_check``).
"""

from __future__ import annotations

import numpy as np
import torch

NORM_RTOL_BF16 = 2e-3
NORM_RTOL_F32 = 1e-4
ACT_RTOL = 1e-2
ACT_ATOL = 1e-3


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def bf16_round(x64: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even to bf16, returned as fp64."""
    return torch.from_numpy(np.ascontiguousarray(x64)).to(torch.bfloat16).to(torch.float64).numpy()


def norm_rel_err(got, ref) -> float:
    got, ref = f64(got), f64(ref)
    if got.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref) / np.abs(ref)))


def assert_norm_close(got, ref, dtype):
    tol = NORM_RTOL_F32 if dtype == torch.float32 else NORM_RTOL_BF16
    err = norm_rel_err(got, ref)
    assert np.all(np.isfinite(f64(got))), "non-finite norm"
    assert err <= tol, f"norm relative error {err:.3e} > {tol:.1e}"
    return err


def assert_act_close(got, ref, what="output"):
    got, ref = f64(got), f64(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    bound = ACT_RTOL * np.abs(ref) + ACT_ATOL
    bad = np.abs(got - ref) > bound
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside 1e-2|ref|+1e-3; "
            f"first at {tuple(idx)}: gpu {got[tuple(idx)]!r} ref {ref[tuple(idx)]!r}"
        )


def _bf16_bits(x64: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().astype(np.int32)


def near_unity_check(y_gpu, y_exact, base, max_midpoint_fraction=1e-3):
    """y - base within 1e-2|ref - base| + 1e-3, rounding-aware.

    ref = the exact (fp64) y rounded to bf16, as the kernel writes bf16.  An
    element also passes when the GPU value is the adjacent bf16 value of ref
    (same sign, bit patterns one apart) and the exact y lies within 1e-6 |y|
    of the midpoint between the two (the kernel's fp32 arithmetic may land on
    either side of such a near-tie).  Returns the fraction of elements that
    needed that second clause.
    """
    y_gpu, y_exact, base = f64(y_gpu), f64(y_exact), f64(base)
    ref = bf16_round(y_exact)
    d_gpu = y_gpu - base
    d_ref = ref - base
    ok = np.abs(d_gpu - d_ref) <= ACT_RTOL * np.abs(d_ref) + ACT_ATOL
    rescued = np.zeros_like(ok)
    other = ~ok
    if other.any():
        yg, yr, ye = y_gpu[other], ref[other], y_exact[other]
        adjacent = (np.sign(yg) == np.sign(yr)) & (np.abs(_bf16_bits(yg) - _bf16_bits(yr)) == 1)
        near_tie = np.abs(ye - 0.5 * (yg + yr)) <= 1e-6 * np.abs(ye)
        rescued[other] = adjacent & near_tie
    ok = ok | rescued
    assert ok.all(), f"near-unity check failed on {int((~ok).sum())} of {ok.size} elements"
    frac = float(rescued.sum()) / max(1, y_gpu.size)
    assert frac <= max_midpoint_fraction, f"midpoint clause used on {frac:.2e} of elements"
    return frac
