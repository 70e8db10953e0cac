"""dora_factored_norm_bwd (gradients of the row norms into A and B) vs the oracle.

The oracle differentiates ||W + sBA||_row on the dense definition in fp64.
The GPU computes dB = s c (W A^T + B (sG)^T) and dA = (s c B)^T W + (s^2 H) A
with c = d_n / n, G = A A^T and H = (c B)^T B; it rounds (s c B), sG and s^2 H
to bf16 and accumulates every product in fp32.  The bar is a per-element
first-order error bound of exactly that arithmetic (grad_bounds below):
rounding a value x to bf16 moves it by at most u |x| (u = 2^-8, eight
significant bits), and an fp32 sum of K terms is off by at most K 2^-24 times
the sum of the terms' magnitudes; each rounded intermediate's error is carried
through the product that uses it by the magnitudes of the other factor.  A
result passes if it is within twice that bound (second-order terms and the
reference's own rounding).  The 8192 x 8192, r = 384 shape is checked on
sampled rows of dB and columns of dA (dB's rows depend only on the same rows
of W and B; dA's columns only on the same columns of W and A, so the oracle
and the bound are evaluated on those slices).
"""

import numpy as np
import pytest
import torch

import oracle
from factored_weight_norm_b200 import dora as D
from factored_weight_norm_b200 import workloads as wlmod
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"
def assert_grad_close(got, ref, bound, what):
    got, ref = P.f64(got), np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape == bound.shape, (got.shape, ref.shape, bound.shape)
    bad = np.abs(got - ref) > 2.0 * bound + 1e-30
    if bad.any():
        idx = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside twice the error bound; first at {idx}: "
                             f"gpu {got[idx]!r} ref {ref[idx]!r} bound {bound[idx]!r}")


def _case(d_out, d_in, r, s, seed=13):
    wl = wlmod.Workload(f"nb_{d_out}x{d_in}_r{r}", d_out, d_in, r, s, 64, "bf16", 0.02, 0.01, 1e-3, seed)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = torch.linalg.vector_norm(W.float() + s * (B.float() @ A.float()), dim=1).contiguous()
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    d_n = torch.randn(d_out, generator=g).to(DEV)
    return W, A, B, n, d_n


SMALL = [(128, 64, 16), (256, 512, 64), (296, 520, 48), (1000, 1000, 128), (512, 1024, 384), (264, 4104, 512),
         (200, 328, 272)]


@pytest.mark.parametrize("shape", SMALL, ids=lambda t: "x".join(map(str, t)))
@pytest.mark.parametrize("s", [0.5, -2.0])
def test_norm_bwd_small(shape, s):
    d_out, d_in, r = shape
    W, A, B, n, d_n = _case(d_out, d_in, r, s)
    dA, dB = D.dora_factored_norm_bwd(W, A, B, s, n, d_n)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    rA, rB = oracle.norm_backward(P.f64(W), P.f64(A), P.f64(B), s, P.f64(n), P.f64(d_n))
    eA, eB = P.grad_bounds(P.f64(W), P.f64(A), P.f64(B), s, P.f64(n), P.f64(d_n))
    assert_grad_close(dA, rA, eA, "dA")
    assert_grad_close(dB, rB, eB, "dB")


def test_norm_bwd_matches_torch_autograd_of_the_dense_norm():
    # an independent GPU check: fp32 autograd through ||W + sBA||_row
    d_out, d_in, r, s = 512, 768, 128, 0.75
    W, A, B, _, d_n = _case(d_out, d_in, r, s, seed=21)
    A32 = A.float().requires_grad_()
    B32 = B.float().requires_grad_()
    nt = torch.linalg.vector_norm(W.float() + s * (B32 @ A32), dim=1)
    (nt * d_n).sum().backward()
    dA, dB = D.dora_factored_norm_bwd(W, A, B, s, nt.detach().contiguous(), d_n)
    torch.cuda.synchronize()
    # fp32 autograd has its own rounding: every fp32 sum is off by at most K 2^-24 of its magnitudes,
    # which the bound's fp32 terms cover once more when doubled
    eA, eB = P.grad_bounds(P.f64(W), P.f64(A), P.f64(B), s, P.f64(nt.detach()), P.f64(d_n))
    assert_grad_close(dA, P.f64(A32.grad), eA, "dA vs autograd")
    assert_grad_close(dB, P.f64(B32.grad), eB, "dB vs autograd")


def test_norm_bwd_headline_sampled():
    wl = wlmod.HEADLINE
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    g = torch.Generator(device=DEV).manual_seed(3)
    d_n = torch.randn(wl.d_out, generator=g, device=DEV)
    dA, dB = D.dora_factored_norm_bwd(W, A, B, wl.s, n, d_n)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    W64, A64, B64, n64, dn64 = P.f64(W), P.f64(A), P.f64(B), P.f64(n), P.f64(d_n)
    rows = np.array([0, 1, 127, 128, 4095, 8191])
    cols = np.array([0, 63, 64, 255, 256, 5000, 8191])
    eA, eB = P.grad_bounds(W64, A64, B64, wl.s, n64, dn64, rows=rows, cols=cols)
    _, rB = oracle.norm_backward(W64[rows], A64, B64[rows], wl.s, n64[rows], dn64[rows])
    assert_grad_close(P.f64(dB)[rows], rB, eB, "dB rows")
    rA, _ = oracle.norm_backward(W64[:, cols], A64[:, cols], B64, wl.s, n64, dn64)
    assert_grad_close(P.f64(dA)[:, cols], rA, eA, "dA columns")


def test_norm_bwd_degenerate_sizes_and_determinism():
    W, A, B, n, d_n = _case(256, 512, 64, 0.5)
    a1, b1 = D.dora_factored_norm_bwd(W, A, B, 0.5, n, d_n)
    a2, b2 = D.dora_factored_norm_bwd(W, A, B, 0.5, n, d_n)
    torch.cuda.synchronize()
    assert torch.equal(a1, a2) and torch.equal(b1, b2)  # fixed summation order
    # d_n = 0: both gradients vanish exactly
    z = torch.zeros_like(d_n)
    a0, b0 = D.dora_factored_norm_bwd(W, A, B, 0.5, n, z)
    torch.cuda.synchronize()
    assert not a0.any() and not b0.any()
    # no output rows: dA = 0 (written, not left as it was)
    dA = torch.full((64, 512), 7.0, device=DEV)
    D.dora_factored_norm_bwd(W[:0], A, B[:0], 0.5, n[:0], d_n[:0], dA=dA)
    torch.cuda.synchronize()
    assert not dA.any()


def test_norm_bwd_mlp_up_shape_sampled():
    # the largest configured projection: 27648 x 5120, r = 384
    wl = wlmod.MLP_UP_32B
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    n = D.dora_factored_norm(W, A, B, wl.s)
    g = torch.Generator(device=DEV).manual_seed(4)
    d_n = torch.randn(wl.d_out, generator=g, device=DEV)
    dA, dB = D.dora_factored_norm_bwd(W, A, B, wl.s, n, d_n)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    W64, A64, B64, n64, dn64 = P.f64(W), P.f64(A), P.f64(B), P.f64(n), P.f64(d_n)
    rows = np.array([0, 255, 13824, 27647])
    cols = np.array([0, 255, 256, 5119])
    eA, eB = P.grad_bounds(W64, A64, B64, wl.s, n64, dn64, rows=rows, cols=cols)
    _, rB = oracle.norm_backward(W64[rows], A64, B64[rows], wl.s, n64[rows], dn64[rows])
    assert_grad_close(P.f64(dB)[rows], rB, eB, "dB rows")
    rA, _ = oracle.norm_backward(W64[:, cols], A64[:, cols], B64, wl.s, n64, dn64)
    assert_grad_close(P.f64(dA)[:, cols], rA, eA, "dA columns")


def test_norm_bwd_no_input_columns_zeroes_dB():
    # d_in = 0: V = W + sBA is empty per row, n = 0 would be the forward, and
    # the gradient into B is exactly zero (written, not left as it was)
    W, A, B, n, d_n = _case(256, 512, 64, 0.5)
    dB = torch.full((256, 64), 7.0, device=DEV)
    D.dora_factored_norm_bwd(W[:, :0].contiguous(), A[:, :0].contiguous(), B, 0.5, n, d_n, dB=dB)
    torch.cuda.synchronize()
    assert not dB.any()


@pytest.mark.parametrize("r", [1024])
def test_norm_bwd_large_rank(r):
    W, A, B, n, d_n = _case(512, 1024, r, 0.5)
    dA, dB = D.dora_factored_norm_bwd(W, A, B, 0.5, n, d_n)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    rA, rB = oracle.norm_backward(P.f64(W), P.f64(A), P.f64(B), 0.5, P.f64(n), P.f64(d_n))
    eA, eB = P.grad_bounds(P.f64(W), P.f64(A), P.f64(B), 0.5, P.f64(n), P.f64(d_n))
    assert_grad_close(dA, rA, eA, "dA")
    assert_grad_close(dB, rB, eB, "dB")


def test_norm_bwd_allocates_nothing_and_has_no_dense_term():
    # the dense B A of this shape would be 8 MB of bf16; the call allocates nothing
    W, A, B, n, d_n = _case(2048, 2048, 384, 0.5)
    dA = torch.empty(384, 2048, device=DEV)
    dB = torch.empty(2048, 384, device=DEV)
    ws = torch.empty(D.dora_factored_norm_bwd_workspace_size(2048, 2048, 384), dtype=torch.uint8, device=DEV)
    D.dora_factored_norm_bwd(W, A, B, 0.5, n, d_n, dA=dA, dB=dB, workspace=ws)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        D.dora_factored_norm_bwd(W, A, B, 0.5, n, d_n, dA=dA, dB=dB, workspace=ws)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
