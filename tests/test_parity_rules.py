"""The comparison rules themselves, on CPU: the near-unity check accepts a
correctly rounded stable compose and rejects the unstable one that rounds
g = m / n to bf16 first (the cancellation the Scaling DoRA abstract warns
about for the near-unity regime)."""

import numpy as np
import pytest
import torch

import oracle
from tests import parity as P


def _case(seed=0, T=64, d=512):
    rng = np.random.default_rng(seed)
    base = P.bf16_round(rng.normal(0, 1.36, (T, d)))
    lora = P.bf16_round(rng.normal(0, 0.023, (T, d)))
    m = rng.uniform(0.5, 2.0, d).astype(np.float32).astype(np.float64)
    g = 1 + rng.normal(0, 1e-4, d)
    n = (m / g).astype(np.float32).astype(np.float64)
    return base, lora, m, n


def test_correctly_rounded_compose_passes():
    base, lora, m, n = _case()
    y_exact = oracle.compose_forward(base, lora, m, n, 0.5)
    frac = P.near_unity_check(P.bf16_round(y_exact), y_exact, base)
    assert frac == 0.0


def test_stable_fp32_form_passes():
    base, lora, m, n = _case(1)
    b32, l32 = base.astype(np.float32), lora.astype(np.float32)
    m32, n32 = m.astype(np.float32), n.astype(np.float32)
    delta = (m32 - n32) / n32
    gs = (m32 / n32) * np.float32(0.5)
    y32 = b32 + (delta[None, :] * b32 + gs[None, :] * l32)
    y_exact = oracle.compose_forward(base, lora, m, n, 0.5)
    P.near_unity_check(P.bf16_round(y32.astype(np.float64)), y_exact, base)


def test_g_rounded_to_bf16_is_rejected():
    base, lora, m, n = _case(2)
    g_bf16 = P.bf16_round(m / n)  # bf16 cannot hold 1 + 1e-4: g collapses to 1
    y_bad = P.bf16_round(g_bf16[None, :] * (base + 0.5 * lora))
    y_exact = oracle.compose_forward(base, lora, m, n, 0.5)
    try:
        P.near_unity_check(y_bad, y_exact, base)
    except AssertionError:
        return
    raise AssertionError("rounding g to bf16 should have been caught")


def test_act_close_bounds():
    ref = np.array([1.0, -2.0, 0.0])
    P.assert_act_close(ref + np.array([9e-3, -1e-2, 9e-4]), ref)
    for bad in (np.array([1.02, -2.0, 0.0]), np.array([1.0, -2.0, 2e-3])):
        try:
            P.assert_act_close(bad, ref)
        except AssertionError:
            continue
        raise AssertionError("bound not enforced")


def test_norm_tolerances():
    ref = np.array([1.0, 2.0])
    P.assert_norm_close(ref * (1 + 1.9e-3), ref, torch.bfloat16)
    P.assert_norm_close(ref * (1 + 0.9e-4), ref, torch.float32)
    for got, dt in ((ref * (1 + 2.1e-3), torch.bfloat16), (ref * (1 + 1.1e-4), torch.float32)):
        try:
            P.assert_norm_close(got, ref, dt)
        except AssertionError:
            continue
        raise AssertionError("norm tolerance not enforced")


# ------------------------------------------- the norm-gradient error model
def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def _emulated_norm_bwd(W, A, B, s, n, d_n, plant=None):
    """The backward's arithmetic on the CPU: (s c B), sG and s^2 H rounded to
    bf16, every product summed in fp32 (float32 matmuls), outputs fp32."""
    f32 = np.float32
    c = (d_n.astype(f32) / n.astype(f32)).astype(np.float64)
    sG = _bf16((s * (A.astype(f32) @ A.astype(f32).T)).astype(np.float64))
    scB = _bf16((s * c)[:, None] * B)
    s2H = _bf16((s * (scB.astype(f32).T @ B.astype(f32))).astype(np.float64))
    if plant == "drop_gram":
        sG = np.zeros_like(sG)
    if plant == "H_scale":
        s2H = s2H / s
    K1 = np.concatenate([W, B], axis=1).astype(f32)
    N1 = np.concatenate([A, sG], axis=1).astype(f32)
    dB = (s * c)[:, None] * (K1 @ N1.T).astype(np.float64)
    dA = (scB.astype(f32).T @ W.astype(f32)).astype(np.float64) + (s2H.astype(f32) @ A.astype(f32)).astype(np.float64)
    if plant == "transpose_B":
        dB = dB[:, ::-1].copy()
    return dA.astype(np.float32).astype(np.float64), dB.astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("shape,s", [((96, 160, 32), 0.5), ((64, 512, 48), -2.0), ((200, 96, 16), 1.25)])
def test_grad_bound_covers_the_kernels_arithmetic(shape, s):
    """An fp32/bf16 emulation of the backward's arithmetic stays within twice
    the per-element bound of the exact (oracle) gradients."""
    d_out, d_in, r = shape
    rng = np.random.default_rng(7)
    W = _bf16(rng.standard_normal((d_out, d_in)) * 0.02)
    A = _bf16(rng.uniform(-1, 1, (r, d_in)) / np.sqrt(d_in))
    B = _bf16(rng.standard_normal((d_out, r)) * 0.01)
    n = np.linalg.norm(W + s * (B @ A), axis=1).astype(np.float32).astype(np.float64)
    d_n = rng.standard_normal(d_out)
    rA, rB = oracle.norm_backward(W, A, B, s, n, d_n)
    gA, gB = _emulated_norm_bwd(W, A, B, s, n, d_n)
    eA, eB = P.grad_bounds(W, A, B, s, n, d_n)
    assert (np.abs(gA - rA) <= 2 * eA + 1e-30).all()
    assert (np.abs(gB - rB) <= 2 * eB + 1e-30).all()
    # the bound stays a small fraction of the gradients themselves (dA's sums
    # over d_out cancel, so its worst-case bound is the looser one): not vacuous
    assert np.median(eA / np.maximum(np.abs(rA), 1e-300)) < 0.1
    assert np.median(eB / np.maximum(np.abs(rB), 1e-300)) < 0.02


@pytest.mark.parametrize("plant", ["drop_gram", "H_scale", "transpose_B"])
def test_grad_bound_rejects_a_planted_mistake(plant):
    """A dropped Gram term, a wrong power of s on H or permuted dB columns
    leave the bound somewhere."""
    d_out, d_in, r, s = 128, 96, 32, 0.5
    rng = np.random.default_rng(11)
    W = _bf16(rng.standard_normal((d_out, d_in)) * 0.02)
    A = _bf16(rng.uniform(-1, 1, (r, d_in)) / np.sqrt(d_in))
    B = _bf16(rng.standard_normal((d_out, r)) * 0.05)
    n = np.linalg.norm(W + s * (B @ A), axis=1).astype(np.float32).astype(np.float64)
    d_n = rng.standard_normal(d_out)
    rA, rB = oracle.norm_backward(W, A, B, s, n, d_n)
    gA, gB = _emulated_norm_bwd(W, A, B, s, n, d_n, plant=plant)
    eA, eB = P.grad_bounds(W, A, B, s, n, d_n)
    outside = (np.abs(gA - rA) > 2 * eA).any() or (np.abs(gB - rB) > 2 * eB).any()
    assert outside, plant
