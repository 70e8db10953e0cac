"""The comparison rules themselves, on CPU: the near-unity check accepts a
correctly rounded stable compose and rejects the unstable one that rounds
g = m / n to bf16 first (the cancellation the Scaling DoRA abstract warns
about for the near-unity regime)."""

import numpy as np
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
