"""Squared-norm shares of d_in shards on the GPU, summed, then finished.

dora_factored_norm_sq on each shard of W and A (split along d_in) must give
the shard's squared norm; their sum, through dora_norm_finish, the whole
layer's norm (bf16, fp32, rank 0).
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


@pytest.mark.parametrize("dtype,shape,parts", [("bf16", (384, 1536, 128), 3), ("bf16", (1000, 2048, 384), 2),
                                               ("f32", (64, 96, 8), 2), ("bf16", (256, 1024, 0), 4)])
def test_shares_sum_to_the_whole_norm(dtype, shape, parts):
    d_out, d_in, r = shape
    wl = wlmod.Workload("shard", d_out, d_in, r, 0.5, 16, dtype, 0.02, 0.01, 1e-3, 31)
    W, A, B, _ = wlmod.make_weights(wl, DEV)
    edges = np.linspace(0, d_in, parts + 1).astype(int)
    total = torch.zeros(d_out, device=DEV)
    for i in range(parts):
        sl = slice(int(edges[i]), int(edges[i + 1]))
        Ws, As = W[:, sl].contiguous(), A[:, sl].contiguous()
        share = D.dora_factored_norm_sq(Ws, As, B, wl.s)
        torch.cuda.synchronize()
        ref_share = oracle.row_norm(P.f64(Ws), P.f64(As), P.f64(B), wl.s) ** 2
        tol = 2e-3 if dtype == "bf16" else 1e-4
        assert np.max(np.abs(P.f64(share) - ref_share) / np.maximum(ref_share, 1e-30)) < 2 * tol
        total += share
    n = D.dora_norm_finish(total)
    torch.cuda.synchronize()
    P.assert_norm_close(n, oracle.row_norm(P.f64(W), P.f64(A), P.f64(B), wl.s),
                        torch.bfloat16 if dtype == "bf16" else torch.float32)
