"""The library's calls captured into CUDA graphs and replayed.

Every entry point takes its stream and all of its buffers from the caller and
launches a fixed sequence (programmatic dependent launches, clusters, no
memset nodes), so a step can be captured once and replayed with new input
values written into the same buffers.  Each replay must reproduce, bit for
bit, what eager calls on the same inputs give (every path sums in a fixed
order).
"""

import pytest
import torch

from factored_weight_norm_b200 import dora as D
from factored_weight_norm_b200 import workloads as wlmod

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fresh(wl, seed):
    W, A, B, m = wlmod.make_weights(wl.with_(seed=seed), DEV)
    _, base, lora = wlmod.make_activations(wl.with_(seed=seed), W, A, B, DEV)
    dy = wlmod.make_grad(wl.with_(seed=seed), DEV)
    return W, A, B, m.float().contiguous(), base, lora, dy


def test_step_graph_replays_match_eager():
    wl = wlmod.Workload("graph_step", 1024, 2048, 128, 0.5, 512, "bf16", 0.02, 0.01, 1e-3, 5)
    W, A, B, m, base, lora, dy = _fresh(wl, 5)
    n = torch.empty(wl.d_out, device=DEV)
    y = torch.empty_like(base)
    d_base, d_lora = torch.empty_like(base), torch.empty_like(base)
    d_m = torch.empty(wl.d_out, device=DEV)
    ws_n = torch.empty(D.dora_factored_norm_workspace_size(wl.d_out, wl.d_in, wl.r), dtype=torch.uint8, device=DEV)
    ws_b = torch.empty(D.dora_compose_bwd_workspace_size(wl.tokens, wl.d_out), dtype=torch.uint8, device=DEV)

    def step():
        D.dora_factored_norm(W, A, B, wl.s, n_out=n, workspace=ws_n)
        D.dora_compose_fwd(base, lora, m, n, wl.s, y=y)
        D.dora_compose_bwd(dy, base, lora, m, n, wl.s, d_base, d_lora, d_m, ws_b)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # first calls (device setup) outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for seed in (11, 12, 13):
        W2, A2, B2, m2, base2, lora2, dy2 = _fresh(wl, seed)
        for dst, src in ((W, W2), (A, A2), (B, B2), (m, m2), (base, base2), (lora, lora2), (dy, dy2)):
            dst.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (n, y, d_base, d_lora, d_m)]
        step()  # eager, same buffers and inputs
        torch.cuda.synchronize()
        for a, b, name in zip(got, (n, y, d_base, d_lora, d_m), ("n", "y", "d_base", "d_lora", "d_m")):
            assert torch.equal(a, b), f"{name}: graph replay differs from the eager call (seed {seed})"
    assert D.dora_device_status() == D.DORA_OK


def test_fused_linear_and_norm_backward_graph_replays_match_eager():
    wl = wlmod.Workload("graph_lin", 768, 1024, 64, 0.5, 640, "bf16", 0.02, 0.01, 1e-3, 6)
    W, A, B, m, _, _, _ = _fresh(wl, 6)
    x = torch.randn(wl.tokens, wl.d_in, device=DEV).to(torch.bfloat16)
    bias = (0.1 * torch.randn(wl.d_out, device=DEV)).to(torch.bfloat16)
    n = D.dora_factored_norm(W, A, B, wl.s)
    d_n = torch.randn(wl.d_out, device=DEV)
    y = torch.empty(wl.tokens, wl.d_out, dtype=torch.bfloat16, device=DEV)
    dA = torch.empty(wl.r, wl.d_in, device=DEV)
    dB = torch.empty(wl.d_out, wl.r, device=DEV)
    ws_l = torch.empty(D.dora_fused_linear_fwd_workspace_size(wl.tokens, wl.r), dtype=torch.uint8, device=DEV)
    ws_g = torch.empty(D.dora_factored_norm_bwd_workspace_size(wl.d_out, wl.d_in, wl.r), dtype=torch.uint8,
                       device=DEV)

    def calls():
        D.dora_fused_linear_fwd(x, W, A, B, m, n, wl.s, bias=bias, y=y, workspace=ws_l)
        D.dora_factored_norm_bwd(W, A, B, wl.s, n, d_n, dA=dA, dB=dB, workspace=ws_g)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        calls()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls()
    for seed in (21, 22):
        gen = torch.Generator(device=DEV).manual_seed(seed)
        x.copy_(torch.randn(x.shape, generator=gen, device=DEV).to(torch.bfloat16))
        d_n.copy_(torch.randn(d_n.shape, generator=gen, device=DEV))
        A.copy_((A.float() * (1 + 0.01 * torch.randn(A.shape, generator=gen, device=DEV))).to(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (y, dA, dB)]
        calls()
        torch.cuda.synchronize()
        for a, b, name in zip(got, (y, dA, dB), ("y", "dA", "dB")):
            assert torch.equal(a, b), f"{name}: graph replay differs from the eager call (seed {seed})"
    assert D.dora_device_status() == D.DORA_OK
