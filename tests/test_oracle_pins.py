"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""

import functools

import numpy as np
import pytest
import torch

import oracle
from factored_weight_norm_b200 import workloads as wlmod
from tests import pins


def test_bruteforce_norm():
    pins.pin_bruteforce_norm(oracle.row_norm)


def test_bruteforce_compose():
    pins.pin_bruteforce_compose(oracle.compose_forward, oracle.compose_backward)


def test_closed_forms():
    pins.pin_closed_forms(oracle.row_norm)


def test_compose_invariants():
    pins.pin_compose_invariants(oracle.compose_forward, oracle.compose_backward)


def test_finite_differences():
    pins.pin_finite_differences(oracle.compose_forward, oracle.compose_backward)


def test_norm_backward():
    pins.pin_norm_backward(oracle.norm_backward)


def _nb_no_s(W, A, B, s, n, d_n):
    return oracle.norm_backward(W, A, B, 1.0, n, d_n)


def _nb_dB_sign(W, A, B, s, n, d_n):
    dA, dB = oracle.norm_backward(W, A, B, s, n, d_n)
    return dA, -dB


def _nb_no_div(W, A, B, s, n, d_n):
    return oracle.norm_backward(W, A, B, s, np.ones(len(n)), d_n)


def _nb_s_once(W, A, B, s, n, d_n):
    # forgets that V itself carries s B A (uses W only inside dV)
    W64, A64, B64 = (np.asarray(v, float) for v in (W, A, B))
    dV = (np.asarray(d_n, float) / np.asarray(n, float))[:, None] * W64
    return s * (B64.T @ dV), s * (dV @ A64.T)


@pytest.mark.parametrize("mutant", [_nb_no_s, _nb_dB_sign, _nb_no_div, _nb_s_once], ids=lambda f: f.__name__)
def test_norm_backward_mutant_is_caught(mutant):
    with pytest.raises((AssertionError, ValueError)):
        pins.pin_norm_backward(mutant)


def test_layer():
    pins.pin_layer(oracle.linear_forward, oracle.compose_forward)


def _l_g_on_rows(x, W, A, B, m, n, s, bias=None, cols=None):
    y = oracle.linear_forward(x, W, A, B, np.ones(len(m)), np.ones(len(n)), s, bias=bias, cols=cols)
    b = 0.0 if bias is None else np.asarray(bias, float)[None, :]
    if cols is not None:
        b = b if bias is None else np.asarray(bias, float)[cols][None, :]
    g = np.asarray(m, float) / np.asarray(n, float)
    T = y.shape[0]
    return b + g[:T, None] * (y - b) if T <= len(g) else y


def _l_no_s(x, W, A, B, m, n, s, bias=None, cols=None):
    return oracle.linear_forward(x, W, A, B, m, n, 1.0, bias=bias, cols=cols)


def _l_transposed_A(x, W, A, B, m, n, s, bias=None, cols=None):
    A = np.asarray(A, float)
    return oracle.linear_forward(x, W, A[::-1], B, m, n, s, bias=bias, cols=cols)


def _l_bias_scaled(x, W, A, B, m, n, s, bias=None, cols=None):
    y = oracle.linear_forward(x, W, A, B, m, n, s, cols=cols)
    if bias is None:
        return y
    b = np.asarray(bias, float)
    b = b if cols is None else b[cols]
    g = np.asarray(m, float) / np.asarray(n, float)
    g = g if cols is None else g[cols]
    return y + (g * b)[None, :]


@pytest.mark.parametrize("mutant", [_l_g_on_rows, _l_no_s, _l_transposed_A, _l_bias_scaled], ids=lambda f: f.__name__)
def test_layer_mutant_is_caught(mutant):
    with pytest.raises((AssertionError, ValueError)):
        pins.pin_layer(mutant, oracle.compose_forward)


def test_bias_layer():
    pins.pin_bias_layer(oracle.compose_forward, oracle.compose_backward)


def test_autograd():
    pins.pin_autograd(oracle.compose_backward)


def test_hand_cases():
    pins.pin_hand_cases(oracle.row_norm, oracle.compose_forward, oracle.compose_backward)


def test_identity_random():
    rng = np.random.default_rng(7)
    for d_out, d_in, r in ((4, 4, 1), (33, 70, 5), (128, 200, 48)):
        W, A, B = pins.tiny_case(rng, d_out, d_in, r)
        for s in (0.0, 0.5, -2.0):
            pins.pin_identity(oracle.row_norm, W, A, B, s)


def _rows_of(wl, nrows=256, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [v for v in (0, 1, 127, 128, wl.d_out - 1) if v < wl.d_out]
    return np.unique(np.concatenate([fixed, rng.integers(0, wl.d_out, nrows)]))


@pytest.mark.parametrize("name", ["tiny_f32", "bf16_4096_r64", "bf16_8192_r384", "bf16_mlp_up_5120x27648_r384"])
def test_identity_on_workloads(name):
    """Factored (base + cross + Gram) == dense, on the bf16-rounded workload inputs."""
    wl = wlmod.WORKLOADS[name]
    W, A, B, _ = wlmod.make_weights(wl)
    rows = _rows_of(wl)
    W64, A64, B64 = (t.double().numpy() for t in (W, A, B))
    got = oracle.row_norm_rows(W64, A64, B64, wl.s, rows)
    ref = np.sqrt(pins.factored_row_norm_sq(W64[rows], A64, B64[rows], wl.s))
    assert pins.rel_err(got, ref) < 1e-11
    # the sampled-row entry point agrees with the whole-matrix one where both run
    if wl.d_out * wl.d_in <= 4096 * 4096:
        full = oracle.row_norm(W64, A64, B64, wl.s)
        assert pins.rel_err(got, full[rows]) < 1e-14


def test_rank_sweep_identity_small_rows():
    for wl in wlmod.RANK_SWEEP[::3]:
        W, A, B, _ = wlmod.make_weights(wl.with_(d_out=256))
        W64, A64, B64 = (t.double().numpy() for t in (W, A, B))
        pins.pin_identity(oracle.row_norm, W64, A64, B64, wl.s)


def test_backward_columns_matches_full():
    rng = np.random.default_rng(11)
    T, d = 17, 13
    dy, base, lora = (rng.standard_normal((T, d)) for _ in range(3))
    n = rng.uniform(0.5, 2, d)
    m = n * 1.001
    cols = np.array([0, 5, 12])
    _, _, d_m = oracle.compose_backward(dy, base, lora, m, n, 0.5)
    got = oracle.compose_backward_columns(dy, base, lora, m, n, 0.5, cols)
    assert np.max(np.abs(got - d_m[cols])) <= 1e-14 * (1 + np.max(np.abs(d_m)))


def test_zero_norm_is_ieee():
    W = np.array([[1.0, 2.0, 2.0]])
    A = np.array([[0.5, 1.0, 1.0]])
    B = np.array([[2.0]])
    n = oracle.row_norm(W, A, B, -1.0)
    assert n[0] == 0.0
    y = oracle.compose_forward(np.ones((1, 1)), np.zeros((1, 1)), np.ones(1), n, -1.0)
    assert np.isinf(y[0, 0])


def test_empty_tokens():
    base = np.zeros((0, 4))
    y = oracle.compose_forward(base, base, np.ones(4), np.ones(4), 0.5)
    assert y.shape == (0, 4)
    d_base, d_lora, d_m = oracle.compose_backward(base, base, base, np.ones(4), np.ones(4), 0.5)
    assert d_base.shape == (0, 4) and np.array_equal(d_m, np.zeros(4))


# ---------------------------------------------------------------- mutants
def _m_drop_s(W, A, B, s):
    Wp = np.asarray(W, float) + np.asarray(B, float) @ np.asarray(A, float)
    return np.sqrt(np.sum(Wp * Wp, axis=1))


def _m_sign(W, A, B, s):
    Wp = np.asarray(W, float) - s * (np.asarray(B, float) @ np.asarray(A, float))
    return np.sqrt(np.sum(Wp * Wp, axis=1))


def _m_s_squared(W, A, B, s):
    Wp = np.asarray(W, float) + s * s * (np.asarray(B, float) @ np.asarray(A, float))
    return np.sqrt(np.sum(Wp * Wp, axis=1))


def _m_column_norm(W, A, B, s):
    Wp = np.asarray(W, float) + s * (np.asarray(B, float) @ np.asarray(A, float))
    return np.sqrt(np.sum(Wp * Wp, axis=0))


def _m_no_sqrt(W, A, B, s):
    Wp = np.asarray(W, float) + s * (np.asarray(B, float) @ np.asarray(A, float))
    return np.sum(Wp * Wp, axis=1)


def _m_index(W, A, B, s):
    A = np.asarray(A, float)[::-1]
    Wp = np.asarray(W, float) + s * (np.asarray(B, float) @ A)
    return np.sqrt(np.sum(Wp * Wp, axis=1))


def _m_drop_col(W, A, B, s):
    Wp = np.asarray(W, float) + s * (np.asarray(B, float) @ np.asarray(A, float))
    return np.sqrt(np.sum(Wp[:, :-1] ** 2, axis=1)) if Wp.shape[1] > 1 else np.zeros(Wp.shape[0])


def _with_bias(f):
    # a forward mutant that handles the bias correctly, so that its own
    # defect is the one a pin has to catch
    @functools.wraps(f)
    def g(base, lora, m, n, s, bias=None):
        if bias is None:
            return f(base, lora, m, n, s)
        b = np.asarray(bias, float)[None, :]
        return b + f(np.asarray(base, float) - b, lora, m, n, s)

    return g


def _f_bias_not_removed(base, lora, m, n, s, bias=None):
    return (np.asarray(m, float) / np.asarray(n, float))[None, :] * (np.asarray(base, float) + s * np.asarray(lora))


def _f_bias_not_restored(base, lora, m, n, s, bias=None):
    b = 0.0 if bias is None else np.asarray(bias, float)[None, :]
    return (np.asarray(m, float) / np.asarray(n, float))[None, :] * (np.asarray(base, float) - b + s * np.asarray(lora))


def _f_inverted(base, lora, m, n, s):
    return (np.asarray(n, float) / np.asarray(m, float))[None, :] * (base + s * np.asarray(lora))


def _f_no_s(base, lora, m, n, s):
    return (np.asarray(m, float) / np.asarray(n, float))[None, :] * (base + np.asarray(lora))


def _f_g_on_base_only(base, lora, m, n, s):
    return (np.asarray(m, float) / np.asarray(n, float))[None, :] * base + s * np.asarray(lora)


def _f_axis(base, lora, m, n, s):
    return (np.asarray(m, float) / np.asarray(n, float))[:, None] * (base + s * np.asarray(lora))


def _bwd(variant):
    def f(dy, base, lora, m, n, s, bias=None):
        dy, base, lora, m, n = (np.asarray(v, float) for v in (dy, base, lora, m, n))
        if bias is not None and variant != "dm_bias_kept":
            base = base - np.asarray(bias, float)[None, :]
        g = m / n
        d_base = g[None, :] * dy
        d_lora = s * g[None, :] * dy
        d_m = np.sum(dy * (base + s * lora), axis=0) / n
        if variant == "dm_no_div":
            d_m = np.sum(dy * (base + s * lora), axis=0)
        elif variant == "dm_no_lora":
            d_m = np.sum(dy * base, axis=0) / n
        elif variant == "dlora_no_s":
            d_lora = g[None, :] * dy
        elif variant == "dbase_no_g":
            d_base = dy.copy()
        elif variant == "dm_div_m":
            d_m = np.sum(dy * (base + s * lora), axis=0) / m
        elif variant == "dm_axis":
            d_m = np.sum(dy * (base + s * lora), axis=1)
        return d_base, d_lora, d_m

    return f


def _run_all_pins(row_norm, fwd, bwd):
    pins.pin_bruteforce_norm(row_norm)
    pins.pin_closed_forms(row_norm)
    rng = np.random.default_rng(9)
    W, A, B = pins.tiny_case(rng, 6, 10, 3)
    pins.pin_identity(row_norm, W, A, B, 0.7)
    pins.pin_bruteforce_compose(fwd, bwd)
    pins.pin_compose_invariants(fwd, bwd)
    pins.pin_finite_differences(fwd, bwd)
    pins.pin_autograd(bwd)
    pins.pin_hand_cases(row_norm, fwd, bwd)
    pins.pin_bias_layer(fwd, bwd)


def test_pins_pass_on_oracle():
    _run_all_pins(oracle.row_norm, oracle.compose_forward, oracle.compose_backward)


NORM_MUTANTS = [_m_drop_s, _m_sign, _m_s_squared, _m_column_norm, _m_no_sqrt, _m_index, _m_drop_col]
FWD_MUTANTS = [_with_bias(f) for f in (_f_inverted, _f_no_s, _f_g_on_base_only, _f_axis)] + [
    _f_bias_not_removed,
    _f_bias_not_restored,
]
BWD_MUTANTS = [
    _bwd(v) for v in ("dm_no_div", "dm_no_lora", "dlora_no_s", "dbase_no_g", "dm_div_m", "dm_axis", "dm_bias_kept")
]


@pytest.mark.parametrize("mutant", NORM_MUTANTS, ids=lambda f: f.__name__)
def test_norm_mutant_is_caught(mutant):
    with pytest.raises((AssertionError, ValueError)):
        _run_all_pins(mutant, oracle.compose_forward, oracle.compose_backward)


@pytest.mark.parametrize("mutant", FWD_MUTANTS, ids=lambda f: f.__name__)
def test_forward_mutant_is_caught(mutant):
    with pytest.raises((AssertionError, ValueError)):
        _run_all_pins(oracle.row_norm, mutant, oracle.compose_backward)


@pytest.mark.parametrize("idx", range(len(BWD_MUTANTS)))
def test_backward_mutant_is_caught(idx):
    with pytest.raises((AssertionError, ValueError)):
        _run_all_pins(oracle.row_norm, oracle.compose_forward, BWD_MUTANTS[idx])


def test_workload_generators_are_deterministic():
    wl = wlmod.TINY_F32
    a = wlmod.make_weights(wl)
    b = wlmod.make_weights(wl)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    W, A, B, m = a
    assert W.shape == (64, 128) and A.shape == (8, 128) and B.shape == (64, 8) and m.dtype == torch.float32
    assert W.dtype == torch.float32
    x, base, lora = wlmod.make_activations(wl, W, A, B)
    assert base.shape == (32, 64) and lora.shape == (32, 64)
    assert wlmod.make_grad(wl).shape == (32, 64)
    assert float(B.abs().max()) > 0  # B nonzero: the cross and Gram terms are exercised
