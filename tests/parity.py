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


# ---------------------------------------------------- norm-gradient bounds
# The attached-norm backward computes dB = s c (W A^T + B (sG)^T) and
# dA = (s c B)^T W + (s^2 H) A with c = d_n / n, G = A A^T, H = (c B)^T B; it
# rounds (s c B), sG and s^2 H to bf16 and accumulates every product in fp32.
# Rounding x to bf16 moves it by at most u |x| (u = 2^-8, eight significant
# bits); an fp32 sum of K terms is off by at most K 2^-24 times the sum of
# the terms' magnitudes; each rounded intermediate's error is carried through
# the product that uses it by the magnitudes of the other factor.
U_BF16 = 2.0 ** -8   # unit roundoff of bf16 (8 significant bits)
E_F32 = 2.0 ** -24   # unit roundoff of fp32


def grad_bounds(W, A, B, s, n, d_n, rows=None, cols=None):
    """First-order bounds (fp64 arrays) on |gpu - exact| for dA [r, d_in] and
    dB [d_out, r] (only dA's `cols` and dB's `rows` when given), from the
    arithmetic described above."""
    W, A, B = (np.asarray(x, dtype=np.float64) for x in (W, A, B))
    n, d_n = np.asarray(n, dtype=np.float64), np.asarray(d_n, dtype=np.float64)
    d_out, d_in = W.shape
    r = A.shape[0]
    u, e = U_BF16, E_F32
    c = d_n / n
    aA, aB = np.abs(A), np.abs(B)
    # ---- dB rows: s c_i (sum_k W_ik A_jk + sum_l B_il (sG)_lj), one fp32 sum over d_in + r
    Wr = W if rows is None else W[rows]
    Br, cr = (B, c) if rows is None else (B[rows], c[rows])
    sG = s * (A @ A.T)
    sG_err = u * np.abs(sG) + d_in * e * abs(s) * (aA @ aA.T)  # its fp32 sum, then bf16
    termW = np.abs(Wr) @ aA.T
    termG = np.abs(Br) @ np.abs(sG)
    eB = np.abs(s * cr)[:, None] * ((d_in + r) * e * (termW + termG) + np.abs(Br) @ sG_err + e * (termW + termG))
    # ---- dA columns: sum_i (s c_i B_ij) W_ik + sum_l (s^2 H)_jl A_lk, one fp32 sum over d_out + r
    Wc, Ac = (W, A) if cols is None else (W[:, cols], A[:, cols])
    scB = (s * c)[:, None] * B
    s2H = s * (scB.T @ B)
    s2H_err = u * np.abs(s2H) + (u + d_out * e) * abs(s) * (np.abs(scB).T @ aB)  # (s c B) in bf16, fp32 sum, bf16
    termB = np.abs(scB).T @ np.abs(Wc)
    termH = np.abs(s2H) @ np.abs(Ac)
    eA = u * termB + s2H_err @ np.abs(Ac) + (d_out + r) * e * (termB + termH)
    return eA, eB
