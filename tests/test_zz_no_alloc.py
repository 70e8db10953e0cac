"""dora_compose_bwd_noalloc: the compose backward for callers that cannot
allocate device memory when they call it (graph-captured code, runtimes whose
memory is fixed after start-up, callers holding only their tensors), checked
through the C ABI against dora_compose_bwd on the same inputs, two calls in a
row.  Collected last on purpose so that a run stopping at the first failure has
already run everything else."""

import ctypes

import pytest
import torch

from factored_weight_norm_b200 import dora as D
from factored_weight_norm_b200 import workloads as wlmod
from tests import parity as P
import oracle

pytestmark = pytest.mark.gpu
MAX_D_OUT = 32768  # DORA_NOALLOC_MAX_D_OUT in include/dora.h


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(T, d_out, dtype):
    wl = wlmod.Workload(f"noalloc_{T}x{d_out}", d_out, 64, 16, 0.5, T, dtype, 0.02, 0.01, 1e-3, 17)
    W, A, B, m = wlmod.make_weights(wl, "cuda")
    _, base, lora = wlmod.make_activations(wl, W, A, B, "cuda")
    dy = wlmod.make_grad(wl, "cuda")
    n = (torch.linalg.vector_norm(W.float(), dim=1) * 1.0007).contiguous()
    return dy, base, lora, m.contiguous(), n, wl.s


def _noalloc(dy, base, lora, m, n, s, d_base, d_lora, d_m, bias=None):
    T, d_out = base.shape
    d_base.fill_(float("nan"))
    d_lora.fill_(float("nan"))
    d_m.fill_(float("nan"))
    head = (_ptr(dy), _ptr(base), _ptr(lora))
    tail = (_ptr(m), _ptr(n), s, T, d_out, D.DORA_BF16 if base.dtype == torch.bfloat16 else D.DORA_F32,
            _ptr(d_base), _ptr(d_lora), _ptr(d_m), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if bias is None:
        st = D.lib().dora_compose_bwd_noalloc(*head, *tail)
    else:
        st = D.lib().dora_compose_bwd_noalloc_bias(*head, _ptr(bias), *tail)
    assert st == D.DORA_OK, D.status_string(st)
    return d_base, d_lora, d_m


@pytest.mark.parametrize("T,d_out,dtype", [(513, 8192, "bf16"), (64, 1000, "f32"), (4096, MAX_D_OUT, "bf16")])
def test_noalloc_matches_workspace_version_twice(T, d_out, dtype):
    dy, base, lora, m, n, s = _inputs(T, d_out, dtype)
    ref = D.dora_compose_bwd(dy, base, lora, m, n, s)
    outs = (torch.empty_like(base), torch.empty_like(base), torch.empty(base.shape[1], device="cuda"))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):  # the scratch keeps the previous call's contents
        got = _noalloc(dy, base, lora, m, n, s, *outs)
        torch.cuda.synchronize()
        for g, r, name in zip(got, ref, ("d_base", "d_lora", "d_m")):
            P.assert_act_close(g, P.f64(r), name)
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0  # nothing was allocated
    assert D.dora_device_status() == D.DORA_OK


def test_noalloc_rejects_d_out_above_its_maximum():
    fake = ctypes.c_void_p(0x10000)
    st = D.lib().dora_compose_bwd_noalloc(fake, fake, fake, fake, fake, 0.5, 4, MAX_D_OUT + 8, D.DORA_BF16,
                                          fake, fake, fake, None)
    assert st == D.DORA_ERR_UNSUPPORTED


def test_noalloc_f32_scalar_vectors_at_the_largest_width():
    # fp32 with d_out not a multiple of 4: one element per vector, the most
    # column strips (2048) and so the most arrival counters the scratch holds
    T, d_out = 40, MAX_D_OUT - 2
    dy, base, lora, m, n, s = _inputs(T, d_out, "f32")
    ref = D.dora_compose_bwd(dy, base, lora, m, n, s)
    outs = (torch.empty_like(base), torch.empty_like(base), torch.empty(base.shape[1], device="cuda"))
    got = _noalloc(dy, base, lora, m, n, s, *outs)
    torch.cuda.synchronize()
    for g, r, name in zip(got, ref, ("d_base", "d_lora", "d_m")):
        P.assert_act_close(g, P.f64(r), name)


@pytest.mark.parametrize("dtype,d_out,with_bias", [("bf16", 1024, False), ("f32", 998, True)])
def test_noalloc_against_the_oracle_twice(dtype, d_out, with_bias):
    # the fp64 oracle's compose backward directly, so that a fault shared by
    # both CUDA entry points cannot pass; fp32 with d_out not a multiple of 4
    # runs one element per vector, with a bias
    T = 96
    dy, base, lora, m, n, s = _inputs(T, d_out, dtype)
    bias = None
    b64 = None
    if with_bias:
        g = torch.Generator(device="cpu").manual_seed(5)
        bias = (0.5 * torch.randn(d_out, generator=g)).to(base.dtype).cuda()
        base = (base + bias).contiguous()
        b64 = P.f64(bias)
    ref = oracle.compose_backward(P.f64(dy), P.f64(base), P.f64(lora), P.f64(m), P.f64(n), s, bias=b64)
    outs = (torch.empty_like(base), torch.empty_like(base), torch.empty(d_out, device="cuda"))
    for _ in range(2):
        got = _noalloc(dy, base, lora, m, n, s, *outs, bias=bias)
        torch.cuda.synchronize()
        for gt, rf, name in zip(got, ref, ("d_base", "d_lora", "d_m")):
            if name != "d_m" and base.dtype == torch.bfloat16:
                rf = P.bf16_round(rf)
            P.assert_act_close(gt, rf, name)
