"""dora_factored_norm_batched vs the fp64 oracle and vs one-module calls.

A mixed batch covers the batched path (bf16, 16 <= r <= 512: ragged M tiles
and K blocks, one and two MMA pieces, r not a multiple of 64, negative and
zero s) next to modules that take the one-by-one path (r = 0, r > 512), in
one call.  A larger batch of many modules of one shape is checked on sampled
rows.
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


def _module(d_out, d_in, r, s, seed):
    wl = wlmod.Workload(f"m_{d_out}x{d_in}_r{r}", d_out, d_in, r, s, 64, "bf16", 0.02, 0.01, 1e-3, seed)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    return W, A, B, s


def _oracle(W, A, B, s, rows=None):
    W64, A64, B64 = P.f64(W), P.f64(A), P.f64(B)
    if rows is None:
        return oracle.row_norm(W64, A64, B64, s)
    return oracle.row_norm_rows(W64, A64, B64, s, rows)


MIXED = [
    (128, 64, 16, 0.5),
    (300, 520, 48, -2.0),     # ragged M tile and K block
    (1000, 1000, 128, 0.5),
    (512, 1024, 384, 0.5),    # two MMA pieces
    (200, 328, 272, 0.25),    # 256 + 16
    (264, 4104, 512, 0.5),    # largest batched rank, K tail of 8
    (384, 640, 256, 0.0),     # s = 0: the plain row norm of W
    (256, 512, 0, 0.5),       # r = 0: one-by-one path
    (384, 640, 768, 0.5),     # r > 512: one-by-one path
]


def test_mixed_batch_matches_oracle_and_single_calls():
    mods = [_module(d_out, d_in, r, s, seed=11 + i) for i, (d_out, d_in, r, s) in enumerate(MIXED)]
    ns = D.dora_factored_norm_batched(mods)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    for (W, A, B, s), n in zip(mods, ns):
        P.assert_norm_close(n, _oracle(W, A, B, s), torch.bfloat16)
        single = D.dora_factored_norm(W, A, B, s)
        torch.cuda.synchronize()
        P.assert_norm_close(n, P.f64(single), torch.bfloat16)


def test_batch_is_deterministic_and_order_free():
    mods = [_module(d_out, d_in, r, s, seed=31 + i) for i, (d_out, d_in, r, s) in enumerate(MIXED[:6])]
    a = [n.clone() for n in D.dora_factored_norm_batched(mods)]
    b = D.dora_factored_norm_batched(mods)
    c = D.dora_factored_norm_batched(mods[::-1])[::-1]
    torch.cuda.synchronize()
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y)  # fixed summation order
        assert torch.equal(x, z)  # a module's result does not depend on its neighbours


def test_many_modules_sampled_rows():
    # 48 modules of 1024 x 2048 at r = 384 (several waves of work items)
    mods = [_module(1024, 2048, 384, 0.5, seed=100 + i) for i in range(48)]
    ns = D.dora_factored_norm_batched(mods)
    torch.cuda.synchronize()
    assert D.dora_device_status() == D.DORA_OK
    rows = np.array([0, 1, 127, 128, 511, 640, 1023])
    for (W, A, B, s), n in zip(mods[::7], ns[::7]):
        P.assert_norm_close(n[torch.as_tensor(rows, device=n.device)], _oracle(W, A, B, s, rows), torch.bfloat16)


def test_batch_workspace_reused_across_calls():
    # the descriptor table in the workspace is rewritten by every call
    mods1 = [_module(256, 512, 64, 0.5, seed=200 + i) for i in range(3)]
    mods2 = [_module(384, 640, 128, -1.0, seed=300 + i) for i in range(5)]
    need = max(D.dora_factored_norm_batched_workspace_size(mods1), D.dora_factored_norm_batched_workspace_size(mods2))
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    n1 = D.dora_factored_norm_batched(mods1, workspace=ws)
    n2 = D.dora_factored_norm_batched(mods2, workspace=ws)
    torch.cuda.synchronize()
    for (W, A, B, s), n in zip(mods1 + mods2, n1 + n2):
        P.assert_norm_close(n, _oracle(W, A, B, s), torch.bfloat16)
