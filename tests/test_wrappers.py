"""The Python binding refuses mismatched tensors before it launches anything.

Each kernel takes its element type from one tensor (W for the norm, base_out
for the compose) and trusts the caller's buffers to match; a bf16 output where
fp32 is expected, a short d_m or a tensor on another device would otherwise be
written or read past its end.  These checks run on the host only: shape and
dtype mismatches are reported for CPU tensors too, and consistent CPU tensors
are refused as not living on a CUDA device.  No test here needs a GPU."""

import pytest
import torch

from factored_weight_norm_b200 import dora as D

T, N = 8, 16


def acts(dtype=torch.bfloat16, shape=(T, N)):
    return torch.zeros(shape, dtype=dtype)


def vec(dtype=torch.float32, n=N):
    return torch.ones(n, dtype=dtype)


def compose_fwd_args(**over):
    a = dict(base_out=acts(), lora_out=acts(), m=vec(), n=vec(), s=0.5, y=None, bias=None)
    a.update(over)
    return a


def compose_bwd_args(**over):
    a = dict(dy=acts(), base_out=acts(), lora_out=acts(), m=vec(), n=vec(), s=0.5, d_base=None, d_lora=None,
             d_m=None, bias=None)
    a.update(over)
    return a


@pytest.mark.parametrize(
    "over, exc",
    [
        (dict(lora_out=acts(torch.float32)), TypeError),
        (dict(lora_out=acts(shape=(T, N + 8))), ValueError),
        (dict(y=acts(torch.float32)), TypeError),
        (dict(y=acts(shape=(T - 1, N))), ValueError),
        (dict(m=vec(torch.bfloat16)), TypeError),
        (dict(n=vec(n=N - 1)), ValueError),
        (dict(bias=vec(torch.float32)), TypeError),
        (dict(base_out=acts(torch.float32), lora_out=acts(torch.float32), y=acts()), TypeError),
    ],
)
def test_compose_fwd_mismatches_raise(over, exc):
    with pytest.raises(exc):
        D.dora_compose_fwd(**compose_fwd_args(**over))


@pytest.mark.parametrize(
    "over, exc",
    [
        (dict(dy=acts(torch.float32)), TypeError),
        (dict(dy=acts(shape=(T + 1, N))), ValueError),
        (dict(lora_out=acts(torch.float32)), TypeError),
        (dict(d_base=acts(torch.float32)), TypeError),
        (dict(d_lora=acts(shape=(T, N - 8))), ValueError),
        (dict(d_m=vec(n=N // 2)), ValueError),
        (dict(d_m=vec(torch.bfloat16)), TypeError),
        (dict(m=vec(torch.float64)), TypeError),
        (dict(base_out=acts(torch.float32), lora_out=acts(torch.float32), dy=acts(torch.float32),
              d_base=acts()), TypeError),
    ],
)
def test_compose_bwd_mismatches_raise(over, exc):
    with pytest.raises(exc):
        D.dora_compose_bwd(**compose_bwd_args(**over))


def test_compose_bwd_noalloc_requires_outputs_and_checks_them():
    a = compose_bwd_args(d_base=acts(), d_lora=acts(), d_m=vec())
    with pytest.raises(ValueError):
        D.dora_compose_bwd_noalloc(**{**a, "d_m": None})
    with pytest.raises(TypeError):
        D.dora_compose_bwd_noalloc(**{**a, "d_lora": acts(torch.float32)})
    with pytest.raises(ValueError):
        D.dora_compose_bwd_noalloc(**{**a, "d_m": vec(n=N + 1)})


def test_consistent_host_tensors_are_refused_as_not_on_cuda():
    with pytest.raises(ValueError, match="CUDA"):
        D.dora_compose_fwd(**compose_fwd_args())
    with pytest.raises(ValueError, match="CUDA"):
        D.dora_compose_bwd(**compose_bwd_args())


def test_norm_output_and_operand_checks():
    W, A, B = torch.zeros(N, 32, dtype=torch.bfloat16), torch.zeros(16, 32, dtype=torch.bfloat16), \
        torch.zeros(N, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        D.dora_factored_norm(W, A, B, 0.5, n_out=vec(n=N - 1))
    with pytest.raises(TypeError):
        D.dora_factored_norm(W, A, B, 0.5, n_out=vec(torch.bfloat16))
    with pytest.raises(TypeError):
        D.dora_factored_norm(W, A.float(), B, 0.5)
    with pytest.raises(ValueError, match="CUDA"):
        D.dora_factored_norm(W, A, B, 0.5)


def test_norm_bwd_and_fused_linear_output_checks():
    W, A, B = torch.zeros(N, 32, dtype=torch.bfloat16), torch.zeros(16, 32, dtype=torch.bfloat16), \
        torch.zeros(N, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        D.dora_factored_norm_bwd(W, A, B, 0.5, vec(), vec(), dA=torch.zeros(16, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        D.dora_factored_norm_bwd(W, A, B, 0.5, vec(), vec(), dB=torch.zeros(N, 8))
    x = torch.zeros(T, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        D.dora_fused_linear_fwd(x, W, A, B, vec(), vec(), 0.5, y=torch.zeros(T, N))
    with pytest.raises(TypeError):
        D.dora_fused_linear_fwd(x, W, A, B, vec(torch.bfloat16), vec(), 0.5)
