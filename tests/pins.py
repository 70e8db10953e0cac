"""Pins for the CPU oracle: checks that do not trust the oracle's own code.

Each pin takes the oracle functions as arguments, so the same pin can be run
against the real oracle (it must pass) and against a deliberately broken copy
(``test_oracle_mutants`` shows that at least one pin then fails).

What pins what (definitions from "Scaling DoRA: High-Rank Adaptation via
Factored Norms and Fused Kernels", Abstract, and the DoRA summary page,
Method):

* brute force      - pure-Python loops over BA, W + sBA, row norms, compose
                     forward and backward on tiny shapes;
* identity         - the factored evaluation ||W_i||^2 + 2s<B_i, W_i A^T>
                     + s^2 B_i (A A^T) B_i^T of the Scaling DoRA abstract
                     ("base, cross, and Gram terms"), written here
                     independently, equals the oracle's dense norm;
* closed forms     - B = 0 or s = 0 gives the plain row norm (numpy.linalg);
                     orthonormal A rows scaled by c with W orthogonal to A's
                     row space gives Pythagoras; r = 1 gives a scalar formula;
* invariants       - m = n gives y = base + s*lora; lora = 0 gives y = g*base;
                     dy = 1 gives column sums; d_lora = s * d_base;
* derivatives      - central finite differences and fp64 torch.autograd of
                     the forward definition with n held constant;
* hand-worked      - small integer cases with exact answers worked by hand,
                     stored in tests/golden/hand_cases.json;
* norm backward    - the gradients of the row norms into A and B equal
                     central finite differences of an independent
                     pure-Python row norm, and fp64 torch.autograd of
                     ||W + sBA||_row (numpy-free);
* layer            - the adapted layer (dense W' = W + sBA applied to x,
                     rescaled per output channel, plus b) equals pure-Python
                     loops on tiny shapes and the separately pinned compose
                     form fed base = x W^T + b and lora = (x A^T) B^T;
* bias             - the compose form with a bias (base = x W^T + b) equals
                     the adapted layer itself, x (diag(m / n) (W + sBA))^T + b
                     with n from numpy.linalg.norm, and its d_m equals
                     torch.autograd of that layer in m (n constant).
"""

from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers
def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.maximum(np.abs(b), 1e-300)
    return float(np.max(np.abs(a - b) / den)) if a.size else 0.0


def tiny_case(rng, d_out=5, d_in=7, r=3):
    W = rng.standard_normal((d_out, d_in))
    A = rng.standard_normal((r, d_in))
    B = rng.standard_normal((d_out, r))
    return W, A, B


# ------------------------------------------------------------ brute force
def brute_row_norm(W, A, B, s):
    d_out, d_in = len(W), len(W[0])
    r = len(A)
    out = []
    for i in range(d_out):
        acc = 0.0
        for k in range(d_in):
            ba = 0.0
            for j in range(r):
                ba += B[i][j] * A[j][k]
            w = W[i][k] + s * ba
            acc += w * w
        out.append(math.sqrt(acc))
    return out


def brute_compose(base, lora, m, n, s, dy):
    T, d = len(base), len(base[0])
    y = [[0.0] * d for _ in range(T)]
    d_base = [[0.0] * d for _ in range(T)]
    d_lora = [[0.0] * d for _ in range(T)]
    d_m = [0.0] * d
    for i in range(d):
        g = m[i] / n[i]
        acc = 0.0
        for t in range(T):
            v = base[t][i] + s * lora[t][i]
            y[t][i] = g * v
            d_base[t][i] = g * dy[t][i]
            d_lora[t][i] = s * g * dy[t][i]
            acc += dy[t][i] * v
        d_m[i] = acc / n[i]
    return y, d_base, d_lora, d_m


def pin_bruteforce_norm(row_norm, seed=0):
    rng = np.random.default_rng(seed)
    for d_out, d_in, r in ((1, 1, 1), (3, 5, 2), (8, 16, 4), (6, 9, 4)):
        W, A, B = tiny_case(rng, d_out, d_in, r)
        for s in (0.0, 0.5, -1.25, 2.0):
            ref = brute_row_norm(W.tolist(), A.tolist(), B.tolist(), s)
            got = row_norm(W, A, B, s)
            assert np.shape(got) == (d_out,)
            assert rel_err(got, ref) < 1e-12, (d_out, d_in, r, s)


def pin_bruteforce_compose(compose_forward, compose_backward, seed=1):
    rng = np.random.default_rng(seed)
    for T, d in ((1, 1), (3, 4), (8, 6)):
        base = rng.standard_normal((T, d))
        lora = rng.standard_normal((T, d))
        dy = rng.standard_normal((T, d))
        n = rng.uniform(0.5, 2.0, d)
        m = n * rng.uniform(0.8, 1.2, d)
        for s in (0.0, 0.5, 2.0, -0.75):
            y, db, dl, dm = brute_compose(base.tolist(), lora.tolist(), m.tolist(), n.tolist(), s, dy.tolist())
            y2 = compose_forward(base, lora, m, n, s)
            db2, dl2, dm2 = compose_backward(dy, base, lora, m, n, s)
            assert np.shape(y2) == (T, d) and np.shape(dm2) == (d,)
            assert np.max(np.abs(y2 - np.array(y))) <= 1e-12 * (1 + np.max(np.abs(y)))
            assert np.max(np.abs(db2 - np.array(db))) <= 1e-12 * (1 + np.max(np.abs(db)))
            assert np.max(np.abs(dl2 - np.array(dl))) <= 1e-12 * (1 + np.max(np.abs(dl)))
            assert np.max(np.abs(dm2 - np.array(dm))) <= 1e-12 * (1 + np.max(np.abs(dm)))


# --------------------------------------------------------------- identity
def factored_row_norm_sq(W, A, B, s):
    """Base + cross + Gram terms, evaluated without forming BA."""
    W, A, B = (np.asarray(v, dtype=np.float64) for v in (W, A, B))
    base = np.einsum("ik,ik->i", W, W)
    U = W @ A.T  # [d_out, r]
    cross = np.einsum("ij,ij->i", B, U)
    G = A @ A.T  # [r, r]
    gram = np.einsum("ij,ij->i", B @ G, B)
    return base + 2.0 * s * cross + s * s * gram


def pin_identity(row_norm, W, A, B, s, tol=1e-11):
    got = row_norm(W, A, B, s)
    ref = np.sqrt(np.maximum(factored_row_norm_sq(W, A, B, s), 0.0))
    assert rel_err(got, ref) < tol


# ----------------------------------------------------------- closed forms
def pin_closed_forms(row_norm, seed=2):
    rng = np.random.default_rng(seed)
    W, A, B = tiny_case(rng, 6, 12, 3)
    plain = np.linalg.norm(W, axis=1)
    # B = 0 and s = 0: the adapter vanishes
    assert rel_err(row_norm(W, A, np.zeros_like(B), 1.7), plain) < 1e-14
    assert rel_err(row_norm(W, A, B, 0.0), plain) < 1e-14
    # A = c * (orthonormal rows); W rows orthogonal to A's row space:
    # ||W_i + s B_i A||^2 = ||W_i||^2 + s^2 c^2 ||B_i||^2 (Pythagoras)
    d_in, r, c, s = 12, 3, 0.37, 1.9
    Q, _ = np.linalg.qr(rng.standard_normal((d_in, d_in)))
    A_o = c * Q[:, :r].T
    W_o = rng.standard_normal((6, d_in - r)) @ Q[:, r:].T
    B_o = rng.standard_normal((6, r))
    ref = np.sqrt(np.linalg.norm(W_o, axis=1) ** 2 + (s * c) ** 2 * np.linalg.norm(B_o, axis=1) ** 2)
    assert rel_err(row_norm(W_o, A_o, B_o, s), ref) < 1e-12
    # r = 1: n_i^2 = ||W_i||^2 + 2 s b_i (a . W_i) + s^2 b_i^2 ||a||^2
    a = rng.standard_normal((1, 12))
    b = rng.standard_normal((6, 1))
    s = -0.6
    ref = np.sqrt(
        np.linalg.norm(W, axis=1) ** 2 + 2 * s * b[:, 0] * (W @ a[0]) + s * s * b[:, 0] ** 2 * np.dot(a[0], a[0])
    )
    assert rel_err(row_norm(W, a, b, s), ref) < 1e-12
    # scaling: n(cW, A, cB) = |c| n(W, A, B)
    assert rel_err(row_norm(3.0 * W, A, 3.0 * B, 0.8), 3.0 * row_norm(W, A, B, 0.8)) < 1e-13
    # orientation: a non-square case where a column norm cannot even be formed row-wise
    W2, A2, B2 = tiny_case(rng, 3, 8, 2)
    assert np.shape(row_norm(W2, A2, B2, 1.0)) == (3,)


# ------------------------------------------------------------- invariants
def pin_compose_invariants(compose_forward, compose_backward, seed=3):
    rng = np.random.default_rng(seed)
    T, d = 9, 11
    base = rng.standard_normal((T, d))
    lora = rng.standard_normal((T, d))
    n = rng.uniform(0.5, 2.0, d)
    m = n * rng.uniform(0.9, 1.1, d)
    s = 0.625
    # m = n  =>  g = 1  =>  y = base + s*lora (exactly: g is 1.0 in fp64)
    y = compose_forward(base, lora, n, n, s)
    assert np.array_equal(y, base + s * lora)
    # lora = 0  =>  y = g * base
    y = compose_forward(base, np.zeros_like(lora), m, n, s)
    assert np.max(np.abs(y - (m / n)[None, :] * base)) < 1e-14
    # dy = 1  =>  d_m = column sums of (base + s lora) / n
    d_base, d_lora, d_m = compose_backward(np.ones((T, d)), base, lora, m, n, s)
    ref = np.array([sum(base[t, i] + s * lora[t, i] for t in range(T)) for i in range(d)]) / n
    assert np.max(np.abs(d_m - ref)) < 1e-12
    # d_lora = s * d_base, bitwise for a power-of-two s
    dy = rng.standard_normal((T, d))
    d_base, d_lora, _ = compose_backward(dy, base, lora, m, n, 0.5)
    assert np.array_equal(d_lora, 0.5 * d_base)
    # d_base = g * dy
    assert np.max(np.abs(d_base - (m / n)[None, :] * dy)) < 1e-15


# ------------------------------------------------------------ derivatives
def pin_finite_differences(compose_forward, compose_backward, seed=4):
    rng = np.random.default_rng(seed)
    T, d = 4, 5
    base = rng.standard_normal((T, d))
    lora = rng.standard_normal((T, d))
    dy = rng.standard_normal((T, d))
    n = rng.uniform(0.5, 2.0, d)
    m = n * rng.uniform(0.9, 1.1, d)
    s = 1.3

    def loss(b, l, mm):
        return float(np.sum(dy * compose_forward(b, l, mm, n, s)))

    d_base, d_lora, d_m = compose_backward(dy, base, lora, m, n, s)
    h = 1e-6
    for t in range(T):
        for i in range(d):
            e = np.zeros((T, d))
            e[t, i] = h
            fd_b = (loss(base + e, lora, m) - loss(base - e, lora, m)) / (2 * h)
            fd_l = (loss(base, lora + e, m) - loss(base, lora - e, m)) / (2 * h)
            assert abs(fd_b - d_base[t, i]) < 1e-7 * (1 + abs(fd_b))
            assert abs(fd_l - d_lora[t, i]) < 1e-7 * (1 + abs(fd_l))
    for i in range(d):
        e = np.zeros(d)
        e[i] = h
        fd_m = (loss(base, lora, m + e) - loss(base, lora, m - e)) / (2 * h)
        assert abs(fd_m - d_m[i]) < 1e-7 * (1 + abs(fd_m))


def pin_autograd(compose_backward, seed=5):
    import torch

    rng = np.random.default_rng(seed)
    T, d = 6, 7
    base = torch.tensor(rng.standard_normal((T, d)), dtype=torch.float64, requires_grad=True)
    lora = torch.tensor(rng.standard_normal((T, d)), dtype=torch.float64, requires_grad=True)
    n_np = rng.uniform(0.5, 2.0, d)
    m = torch.tensor(n_np * rng.uniform(0.9, 1.1, d), dtype=torch.float64, requires_grad=True)
    n = torch.tensor(n_np, dtype=torch.float64)  # constant: no grad
    dy = torch.tensor(rng.standard_normal((T, d)), dtype=torch.float64)
    s = 0.75
    y = (m / n)[None, :] * (base + s * lora)
    y.backward(dy)
    d_base, d_lora, d_m = compose_backward(
        dy.numpy(), base.detach().numpy(), lora.detach().numpy(), m.detach().numpy(), n_np, s
    )
    assert np.max(np.abs(d_base - base.grad.numpy())) < 1e-14
    assert np.max(np.abs(d_lora - lora.grad.numpy())) < 1e-14
    assert np.max(np.abs(d_m - m.grad.numpy())) < 1e-12


# ------------------------------------------------------------------ bias
def pin_bias_layer(compose_forward, compose_backward, seed=6):
    """DoRA summary page, Method: the adapted weight is m * V / ||V|| per output
    channel, V = W + sBA; a bias b is added after the product and is not
    rescaled.  A framework's base layer returns x W^T + b."""
    import torch

    rng = np.random.default_rng(seed)
    T, d_in, d_out, r = 5, 7, 6, 3
    x = rng.standard_normal((T, d_in))
    W, A, B = tiny_case(rng, d_out, d_in, r)
    b = rng.standard_normal(d_out)
    dy = rng.standard_normal((T, d_out))
    for s in (0.5, -1.5):
        V = W + s * (B @ A)
        n = np.linalg.norm(V, axis=1)
        m = n * rng.uniform(0.8, 1.2, d_out)
        y_layer = x @ ((m / n)[:, None] * V).T + b[None, :]
        base = x @ W.T + b[None, :]
        lora = (x @ A.T) @ B.T
        y = compose_forward(base, lora, m, n, s, bias=b)
        assert np.max(np.abs(y - y_layer)) < 1e-12 * (1 + np.max(np.abs(y_layer)))
        # no bias and a zero bias are the same thing
        z = np.zeros(d_out)
        assert np.array_equal(compose_forward(base, lora, m, n, s), compose_forward(base, lora, m, n, s, bias=z))

        mt = torch.tensor(m, dtype=torch.float64, requires_grad=True)
        yt = torch.tensor(x) @ ((mt / torch.tensor(n))[:, None] * torch.tensor(V)).T + torch.tensor(b)[None, :]
        yt.backward(torch.tensor(dy))
        d_base, d_lora, d_m = compose_backward(dy, base, lora, m, n, s, bias=b)
        assert np.max(np.abs(d_m - mt.grad.numpy())) < 1e-11 * (1 + np.max(np.abs(d_m)))
        # the bias does not change the activation gradients
        d_base0, d_lora0, _ = compose_backward(dy, base, lora, m, n, s)
        assert np.array_equal(d_base, d_base0) and np.array_equal(d_lora, d_lora0)
        assert np.max(np.abs(d_base - (m / n)[None, :] * dy)) < 1e-15 * (1 + np.max(np.abs(d_base)))


# --------------------------------------------------------- norm backward
def pin_norm_backward(norm_backward, seed=8):
    import torch

    pin_hand_norm_backward(norm_backward)

    rng = np.random.default_rng(seed)
    for d_out, d_in, r in ((3, 4, 2), (5, 7, 3), (4, 9, 5)):
        W, A, B = tiny_case(rng, d_out, d_in, r)
        d_n = rng.standard_normal(d_out)
        for s in (0.7, -1.3):
            n = np.array(brute_row_norm(W.tolist(), A.tolist(), B.tolist(), s))
            dA, dB = norm_backward(W, A, B, s, n, d_n)
            assert np.shape(dA) == (r, d_in) and np.shape(dB) == (d_out, r)

            def loss(A_, B_):
                return float(np.dot(d_n, brute_row_norm(W.tolist(), A_.tolist(), B_.tolist(), s)))

            h = 1e-6
            for (i, j) in ((0, 0), (r - 1, d_in - 1), (r // 2, d_in // 2)):
                e = np.zeros_like(A)
                e[i, j] = h
                fd = (loss(A + e, B) - loss(A - e, B)) / (2 * h)
                assert abs(fd - dA[i, j]) < 1e-6 * (1 + abs(fd)), ("dA", i, j)
            for (i, j) in ((0, 0), (d_out - 1, r - 1), (d_out // 2, r // 2)):
                e = np.zeros_like(B)
                e[i, j] = h
                fd = (loss(A, B + e) - loss(A, B - e)) / (2 * h)
                assert abs(fd - dB[i, j]) < 1e-6 * (1 + abs(fd)), ("dB", i, j)

            At = torch.tensor(A, requires_grad=True)
            Bt = torch.tensor(B, requires_grad=True)
            nt = torch.linalg.vector_norm(torch.tensor(W) + s * (Bt @ At), dim=1)
            (nt * torch.tensor(d_n)).sum().backward()
            assert np.max(np.abs(dA - At.grad.numpy())) < 1e-12 * (1 + np.max(np.abs(dA)))
            assert np.max(np.abs(dB - Bt.grad.numpy())) < 1e-12 * (1 + np.max(np.abs(dB)))


# ----------------------------------------------------------------- layer
def brute_layer(x, W, A, B, m, n, s, b):
    T, d_in, d_out, r = len(x), len(W[0]), len(W), len(A)
    y = [[0.0] * d_out for _ in range(T)]
    for i in range(d_out):
        row = [W[i][k] + s * sum(B[i][j] * A[j][k] for j in range(r)) for k in range(d_in)]
        for t in range(T):
            y[t][i] = b[i] + (m[i] / n[i]) * sum(x[t][k] * row[k] for k in range(d_in))
    return y


def pin_layer(linear_forward, compose_forward, seed=7):
    pin_hand_layer(linear_forward)
    rng = np.random.default_rng(seed)
    for T, d_in, d_out, r in ((1, 1, 1, 1), (3, 5, 4, 2), (6, 9, 7, 3)):
        x = rng.standard_normal((T, d_in))
        W, A, B = tiny_case(rng, d_out, d_in, r)
        b = rng.standard_normal(d_out)
        n = rng.uniform(0.5, 2.0, d_out)
        m = n * rng.uniform(0.8, 1.2, d_out)
        for s in (0.0, 0.75, -1.5):
            ref = np.array(brute_layer(x.tolist(), W.tolist(), A.tolist(), B.tolist(), m.tolist(), n.tolist(), s,
                                       b.tolist()))
            y = linear_forward(x, W, A, B, m, n, s, bias=b)
            assert np.shape(y) == (T, d_out)
            assert np.max(np.abs(y - ref)) <= 1e-12 * (1 + np.max(np.abs(ref)))
            y2 = compose_forward(x @ W.T + b[None, :], (x @ A.T) @ B.T, m, n, s, bias=b)
            assert np.max(np.abs(y - y2)) <= 1e-12 * (1 + np.max(np.abs(ref)))
            cols = [d_out - 1, 0]
            assert np.max(np.abs(linear_forward(x, W, A, B, m, n, s, bias=b, cols=cols) - ref[:, cols])) <= 1e-12 * (
                1 + np.max(np.abs(ref)))
            y0 = linear_forward(x, W, A, B, m, n, s)
            assert np.max(np.abs(y0 - (ref - b[None, :]))) <= 1e-12 * (1 + np.max(np.abs(ref)))


# ------------------------------------------------------------ hand-worked
def load_hand_cases():
    with open(os.path.join(GOLDEN, "hand_cases.json")) as f:
        return json.load(f)["cases"]


def pin_hand_layer(linear_forward):
    """The adapted layer on the hand-worked case (exact in binary)."""
    for case in load_hand_cases():
        if "x" not in case:
            continue
        W, A, B, m, n, x, b = (np.array(case[k], dtype=np.float64) for k in ("W", "A", "B", "m", "n", "x", "bias"))
        y = linear_forward(x, W, A, B, m, n, float(case["s"]), bias=b)
        assert np.array_equal(np.asarray(y, float), np.array(case["y_layer"], dtype=np.float64)), case["name"]


def pin_hand_norm_backward(norm_backward):
    """Gradients of n w.r.t. A and B on the hand-worked case (exact in binary)."""
    for case in load_hand_cases():
        if "d_n" not in case:
            continue
        W, A, B, n, d_n = (np.array(case[k], dtype=np.float64) for k in ("W", "A", "B", "n", "d_n"))
        dA, dB = norm_backward(W, A, B, float(case["s"]), n, d_n)
        assert np.array_equal(np.asarray(dA, float), np.array(case["dA"], dtype=np.float64)), case["name"]
        assert np.array_equal(np.asarray(dB, float), np.array(case["dB"], dtype=np.float64)), case["name"]


def pin_hand_cases(row_norm, compose_forward, compose_backward):
    for case in load_hand_cases():
        W, A, B, s = (np.array(case[k], dtype=np.float64) for k in ("W", "A", "B", "s"))
        s = float(s)
        got = row_norm(W, A, B, s)
        assert rel_err(got, np.array(case["n"], dtype=np.float64)) < 1e-15, case["name"]
        if "base" in case:
            base, lora, m, n, dy = (np.array(case[k], dtype=np.float64) for k in ("base", "lora", "m", "n", "dy"))
            y = compose_forward(base, lora, m, n, s)
            d_base, d_lora, d_m = compose_backward(dy, base, lora, m, n, s)
            assert np.array_equal(y, np.array(case["y"], dtype=np.float64)), case["name"]
            assert np.array_equal(d_base, np.array(case["d_base"], dtype=np.float64)), case["name"]
            assert np.array_equal(d_lora, np.array(case["d_lora"], dtype=np.float64)), case["name"]
            assert np.array_equal(d_m, np.array(case["d_m"], dtype=np.float64)), case["name"]
