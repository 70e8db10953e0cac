"""The factored norm of a row-parallel layer: W and A split along d_in.

Every term of n_i^2 = ||W_i||^2 + 2s <B_i, W_i A^T> + s^2 B_i (A A^T) B_i^T is
a sum over d_in, so each rank's squared norm over its own columns
(``dora_factored_norm_sq``) is its share of the whole n^2.  One all-reduce of
d_out fp32 values sums the shares (NCCL over NVLink between GPUs: the only
exchange the norm has) and ``dora_norm_finish`` takes the square root.  B is
whole on every rank.  Scaling DoRA, Abstract: the norm from base, cross and
Gram terms without the dense product; the decomposition is the same one,
split along the contraction.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import dora as D


def sum_shares(n2: torch.Tensor, group=None) -> torch.Tensor:
    """Adds every rank's squared-norm shares in place (one all-reduce)."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(n2, op=dist.ReduceOp.SUM, group=group)
    return n2


def sharded_factored_norm(W_shard, A_shard, B, s: float, group=None, n_out=None, workspace=None, stream=None):
    """n = ||W + sBA||_row for W = [W_0 | W_1 | ...], A = [A_0 | A_1 | ...] split along
    d_in over the ranks of ``group`` (this rank holds W_shard, A_shard and all of B)."""
    n2 = D.dora_factored_norm_sq(W_shard, A_shard, B, s, n2_out=n_out, workspace=workspace, stream=stream)
    sum_shares(n2, group)
    return D.dora_norm_finish(n2, stream=stream)
