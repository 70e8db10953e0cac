"""dora_fused_linear_fwd (compose fused into the producing GEMMs) vs the oracle.

The oracle is the adapted layer itself: b + (m / n) * x (W + sBA)^T in fp64.
The GPU rounds P = s x A^T to bf16 once (as a framework's LoRA path rounds
x A^T) and y once; both sit well inside the activation tolerance
1e-2 |ref| + 1e-3.  Small cases span several 128-row and 256-column tiles with
ragged M, N and K tails and ranks that are not multiples of 64; the headline
shape is checked on sampled rows and columns.
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


def _case(T, d_in, d_out, r, s=0.5, bias=True, seed=3):
    wl = wlmod.Workload(f"lin_{T}x{d_in}x{d_out}_r{r}", d_out, d_in, r, s, T, "bf16", 0.02, 0.01, 1e-3, seed)
    W, A, B, m = wlmod.make_weights(wl, DEV)
    x, _, _ = wlmod.make_activations(wl, W, A, B, DEV)
    g = torch.Generator(device="cpu").manual_seed(seed + 7)
    b = (0.3 * torch.randn(d_out, generator=g)).to(torch.bfloat16).to(DEV) if bias else None
    # n is an input here (any positive vector would do): the row norm of W + sBA
    n = torch.linalg.vector_norm(W.float() + s * (B.float() @ A.float()), dim=1).contiguous()
    return x.contiguous(), W, A, B, b, m.float().contiguous(), n, s


def _ref(x, W, A, B, b, m, n, s, rows=None, cols=None):
    xr = P.f64(x) if rows is None else P.f64(x)[rows]
    return oracle.linear_forward(xr, P.f64(W), P.f64(A), P.f64(B), P.f64(m), P.f64(n), s,
                                 bias=None if b is None else P.f64(b), cols=cols)


SMALL = [
    (128, 64, 256, 16),     # one tile each way
    (300, 520, 1000, 48),   # ragged M, K and N tails
    (257, 1024, 512, 384),  # rank over several K blocks, M tail of 1
    (64, 4104, 264, 512),   # K tail of 8, N tail of 8
    (1, 64, 8, 8),          # one token, smallest N and r
    (130, 136, 2056, 40),   # r not a multiple of 64
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("bias", [True, False])
def test_fused_linear_small(shape, bias):
    T, d_in, d_out, r = shape
    x, W, A, B, b, m, n, s = _case(T, d_in, d_out, r, bias=bias)
    y = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    P.assert_act_close(y, _ref(x, W, A, B, b, m, n, s), "y")


@pytest.mark.parametrize("s", [-2.0, 0.0])
def test_fused_linear_negative_and_zero_scale(s):
    x, W, A, B, b, m, n, _ = _case(200, 256, 512, 64, s=s)
    y = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b)
    torch.cuda.synchronize()
    P.assert_act_close(y, _ref(x, W, A, B, b, m, n, s), "y")


def test_fused_linear_rank_zero():
    x, W, A, B, b, m, n, s = _case(96, 128, 264, 0)
    y = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b)
    torch.cuda.synchronize()
    P.assert_act_close(y, _ref(x, W, A, B, b, m, n, s), "y")


def test_fused_linear_zero_tokens():
    x, W, A, B, b, m, n, s = _case(0, 64, 256, 16)
    y = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b)
    assert y.shape == (0, 256)


def test_fused_linear_matches_unfused_path_and_is_deterministic():
    # same inputs through base = x W^T + b, lora = (x A^T) B^T and the compose
    x, W, A, B, b, m, n, s = _case(384, 1024, 2048, 128)
    y1 = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b)
    y2 = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b)
    base = (x.float() @ W.float().t() + b.float()).to(torch.bfloat16)
    lora = ((x.float() @ A.float().t()) @ B.float().t()).to(torch.bfloat16)
    yc = D.dora_compose_fwd(base, lora, m, n, s, bias=b)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    P.assert_act_close(y1, P.f64(yc), "fused vs unfused")


def test_fused_linear_headline_sampled():
    # 8192 tokens x (8192 -> 8192), r = 384: the bench's fused-linear workload
    wl = wlmod.HEADLINE
    W, A, B, m = wlmod.make_weights(wl, DEV)
    g = torch.Generator(device=DEV).manual_seed(5)
    x = torch.randn(wl.tokens, wl.d_in, generator=g, device=DEV).to(torch.bfloat16)
    n = D.dora_factored_norm(W, A, B, wl.s)
    b = (0.1 * torch.randn(wl.d_out, generator=g, device=DEV)).to(torch.bfloat16)
    y = D.dora_fused_linear_fwd(x, W, A, B, m.float().contiguous(), n, wl.s, bias=b)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    rows = np.array([0, 1, 127, 128, 4095, 4096, 8000, 8191])
    cols = np.array([0, 1, 255, 256, 3000, 8190, 8191])
    ref = _ref(x, W, A, B, b, m, n, wl.s, rows=rows, cols=cols)
    got = P.f64(y)[rows][:, cols]
    P.assert_act_close(got, ref, "y sampled")


def test_fused_linear_workspace_reuse_and_errors():
    x, W, A, B, b, m, n, s = _case(128, 256, 512, 64)
    ws = torch.empty(D.dora_fused_linear_fwd_workspace_size(128, 64), dtype=torch.uint8, device=DEV)
    y1 = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b, workspace=ws)
    y2 = D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=None, workspace=ws)
    torch.cuda.synchronize()
    P.assert_act_close(y1, _ref(x, W, A, B, b, m, n, s), "y with bias")
    P.assert_act_close(y2, _ref(x, W, A, B, None, m, n, s), "y without bias")
    with pytest.raises(RuntimeError):
        D.dora_fused_linear_fwd(x, W, A, B, m, n, s, workspace=ws[:100])
    with pytest.raises(TypeError):
        D.dora_fused_linear_fwd(x.float(), W, A, B, m, n, s)


def test_fused_linear_mlp_up_shape_sampled():
    # the largest configured projection: 16384 tokens x (5120 -> 27648), r = 384
    wl = wlmod.MLP_UP_32B
    W, A, B, m = wlmod.make_weights(wl, DEV)
    g = torch.Generator(device=DEV).manual_seed(9)
    x = torch.randn(wl.tokens, wl.d_in, generator=g, device=DEV).to(torch.bfloat16)
    n = D.dora_factored_norm(W, A, B, wl.s)
    y = D.dora_fused_linear_fwd(x, W, A, B, m.float().contiguous(), n, wl.s)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    rows = np.array([0, 255, 256, 9999, 16383])
    cols = np.array([0, 191, 192, 13824, 27647])
    ref = _ref(x, W, A, B, None, m, n, wl.s, rows=rows, cols=cols)
    P.assert_act_close(P.f64(y)[rows][:, cols], ref, "y sampled")


def test_fused_linear_no_output_channels():
    x, W, A, B, b, m, n, s = _case(64, 128, 256, 16)
    y = D.dora_fused_linear_fwd(x, W[:0].contiguous(), A, B[:0].contiguous(), m[:0], n[:0], s)
    assert y.shape == (64, 0)


def test_fused_linear_allocates_nothing():
    # with the caller's workspace and output, the call allocates no device memory
    x, W, A, B, b, m, n, s = _case(512, 2048, 1024, 384)
    y = torch.empty(512, 1024, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(D.dora_fused_linear_fwd_workspace_size(512, 384), dtype=torch.uint8, device=DEV)
    D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b, y=y, workspace=ws)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        D.dora_fused_linear_fwd(x, W, A, B, m, n, s, bias=b, y=y, workspace=ws)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
