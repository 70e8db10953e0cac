"""Compose forward / backward with a base-layer bias, CUDA path vs the oracle.

The base output includes the bias b (x W^T + b); the rescaling acts on the
weight's product only: y = b + g * ((base - b) + s * lora), and d_m sums
dy * ((base - b) + s * lora).  No bias must be bit-identical to a zero bias.
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


def _inputs(T, d_out, dtype, seed=23, bias_std=0.5):
    wl = wlmod.Workload(f"bias_{T}x{d_out}", d_out, 64, 16, 0.5, T, dtype, 0.02, 0.01, 1e-3, seed)
    W, A, B, m = wlmod.make_weights(wl, DEV)
    _, base, lora = wlmod.make_activations(wl, W, A, B, DEV)
    dy = wlmod.make_grad(wl, DEV)
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    bias = (bias_std * torch.randn(d_out, generator=g)).to(base.dtype).to(DEV)
    base = (base.float() + bias.float()[None, :]).to(base.dtype).contiguous()  # the base layer adds its bias
    n = (torch.linalg.vector_norm(W.float(), dim=1) * (1 + 1e-3 * torch.randn(d_out, generator=g).to(DEV))).contiguous()
    return base, lora, bias, m.float().contiguous(), n.float().contiguous(), dy, wl.s


CASES = [(37, 264, "bf16"), (300, 1000, "bf16"), (129, 2056, "bf16"), (33, 130, "f32"), (16, 4, "f32"), (64, 4096, "f32")]


@pytest.mark.parametrize("T,d_out,dtype", CASES)
def test_compose_with_bias_matches_oracle(T, d_out, dtype):
    base, lora, bias, m, n, dy, s = _inputs(T, d_out, dtype)
    y = D.dora_compose_fwd(base, lora, m, n, s, bias=bias)
    d_base, d_lora, d_m = D.dora_compose_bwd(dy, base, lora, m, n, s, bias=bias)
    torch.cuda.synchronize()
    args = [P.f64(t) for t in (base, lora, m, n)]
    b64 = P.f64(bias)
    P.assert_act_close(y, oracle.compose_forward(*args, s, bias=b64), "y")
    rb, rl, rm = oracle.compose_backward(P.f64(dy), *args, s, bias=b64)
    P.assert_act_close(d_base, rb, "d_base")
    P.assert_act_close(d_lora, rl, "d_lora")
    P.assert_act_close(d_m, rm, "d_m")
    # the bias changes d_m (against the no-bias oracle) on these inputs
    _, _, rm0 = oracle.compose_backward(P.f64(dy), *args, s)
    assert np.max(np.abs(rm - rm0)) > 10 * (1e-2 * np.max(np.abs(rm)) + 1e-3)


def test_bias_near_unity_is_stable():
    # m = n (1 + 1e-4): y - base = delta (base - b) + g s lora is tiny next to
    # base; the stable form keeps it to the rounding of y
    base, lora, bias, m, n, dy, s = _inputs(512, 2048, "bf16", seed=41)
    m = (n * (1 + 1e-4)).contiguous()
    y = D.dora_compose_fwd(base, lora, m, n, s, bias=bias)
    torch.cuda.synchronize()
    y_exact = oracle.compose_forward(P.f64(base), P.f64(lora), P.f64(m), P.f64(n), s, bias=P.f64(bias))
    frac = P.near_unity_check(y, y_exact, base)
    assert frac < 1e-3


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_no_bias_is_a_zero_bias_bitwise(dtype):
    base, lora, _, m, n, dy, s = _inputs(65, 1024, dtype, seed=5)
    zero = torch.zeros(base.shape[1], dtype=base.dtype, device=DEV)
    y0 = D.dora_compose_fwd(base, lora, m, n, s)
    y1 = D.dora_compose_fwd(base, lora, m, n, s, bias=zero)
    g0 = D.dora_compose_bwd(dy, base, lora, m, n, s)
    g1 = D.dora_compose_bwd(dy, base, lora, m, n, s, bias=zero)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    for a, b in zip(g0, g1):
        assert torch.equal(a, b)


def test_noalloc_with_bias_matches_workspace_version():
    base, lora, bias, m, n, dy, s = _inputs(777, 8192, "bf16", seed=9)
    ref = D.dora_compose_bwd(dy, base, lora, m, n, s, bias=bias)
    outs = (torch.empty_like(base), torch.empty_like(base), torch.empty(base.shape[1], device=DEV))
    got = D.dora_compose_bwd_noalloc(dy, base, lora, m, n, s, *outs, bias=bias)
    torch.cuda.synchronize()
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    P.assert_act_close(got[2], P.f64(ref[2]), "d_m")
    assert D.dora_device_status() == D.DORA_OK


def test_bias_argument_checks():
    base, lora, bias, m, n, dy, s = _inputs(8, 64, "bf16")
    with pytest.raises(ValueError):
        D.dora_compose_fwd(base, lora, m, n, s, bias=bias[:32])
    with pytest.raises(TypeError):
        D.dora_compose_fwd(base, lora, m, n, s, bias=bias.float())
