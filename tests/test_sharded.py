"""The norm of a row-parallel layer (W and A split along d_in), on CPU.

* the decomposition: the squared norm of the whole adapted weight equals the
  sum over d_in shards of each shard's squared norm (oracle only);
* the exchange: two gloo ranks each holding one shard's share (computed by the
  oracle) all-reduce them with ``sharded.sum_shares`` and recover the whole
  layer's norm.
The CUDA shares (``dora_factored_norm_sq``) and ``dora_norm_finish`` are
checked against the same oracle on the GPU in ``test_sharded_gpu.py``.
"""

import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from tests import pins


def _shards(d_in, parts):
    edges = np.linspace(0, d_in, parts + 1).astype(int)
    return [slice(edges[i], edges[i + 1]) for i in range(parts)]


@pytest.mark.parametrize("parts", [2, 3, 5])
def test_squared_norm_is_the_sum_of_shard_shares(parts):
    rng = np.random.default_rng(parts)
    W, A, B = pins.tiny_case(rng, 7, 23, 4)
    for s in (0.5, -1.25):
        full = oracle.row_norm(W, A, B, s) ** 2
        shares = sum(oracle.row_norm(W[:, sl], A[:, sl], B, s) ** 2 for sl in _shards(23, parts))
        assert np.max(np.abs(shares - full)) <= 1e-12 * np.max(full)


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from factored_weight_norm_b200 import sharded

        rng = np.random.default_rng(77)
        W, A, B = pins.tiny_case(rng, 9, 40, 5)
        sl = _shards(40, world)[rank]
        share = torch.tensor(oracle.row_norm(W[:, sl], A[:, sl], B, 0.75) ** 2)
        sharded.sum_shares(share)
        n = torch.sqrt(torch.clamp(share, min=0))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"n": n.tolist(), "ref": oracle.row_norm(W, A, B, 0.75).tolist()}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_recover_the_whole_norm(tmp_path):
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for rank in range(2):
        got = json.load(open(tmp_path / f"rank{rank}.json"))
        assert np.max(np.abs(np.array(got["n"]) - np.array(got["ref"])) / np.array(got["ref"])) < 1e-12
