"""bench.py's multi-rank host logic on CPU: two gloo ranks (no GPU).

One process per rank, as under torchrun.  Each rank reports different times;
both must see the element-wise maximum (the slowest rank decides every number),
rank 0 alone builds the JSON line, whose rates count the work of both replicas,
and the reference arm runs on rank 0 only.
"""

import importlib.util
import io
import json
import os
import socket
import contextlib

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        # rank k is slower on a different quantity than the other rank
        mine = [1.0 + rank, 0.5 + 0.25 * (1 - rank), 0.1 + 0.05 * rank, 0.2]
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        result = {"max": got}
        if rank == 0:
            wl = bench.WL.HEADLINE
            res = dict(t_total=got[0], t_norm=got[1], t_fwd=got[2], t_bwd=got[3], clocks=None, status=0, wl=wl,
                       e2e=dict(t_norm=2 * got[1], t_fwd=2 * got[2], t_bwd=2 * got[3], h2d=10, d2h=20, steps=5),
                       launches=28, flushed=False)

            class Args:
                steps, warmup = 7, 3

            peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
            line = bench.build_line(Args, res, world, peaks, "test", {}, None)
            result["line"] = json.loads(json.dumps(line))
        # the reference arm: rank 0 only (rank 1 returns at once, printing nothing)
        if rank == 1:
            buf = io.StringIO()

            class RefArgs:
                steps, warmup, gpus, workload = 1, 0, world, bench.WL.HEADLINE.name

            with contextlib.redirect_stdout(buf):
                rc = bench.run_reference(RefArgs, rank, world)
            result["ref_rc"] = rc
            result["ref_out"] = buf.getvalue()
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(result, f)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("ranks"))
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    return [json.load(open(os.path.join(out, f"rank{r}.json"))) for r in range(2)]


def test_every_rank_sees_the_max(two_ranks):
    expect = [2.0, 0.75, 0.15, 0.2]
    for r in two_ranks:
        assert r["max"] == pytest.approx(expect)


def test_line_counts_both_replicas(two_ranks):
    bench = _bench()
    line = two_ranks[0]["line"]
    wl = bench.WL.HEADLINE
    F = bench.norm_flops(wl.d_out, wl.d_in, wl.r)
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["config"]["parallelism"] == "replicas x2"
    assert line["value"] == pytest.approx(2 * F / 0.75 / 1e12)
    assert line["compose"]["fwd"]["value"] == pytest.approx(2 * bench.fwd_bytes(wl.tokens, wl.d_out) / 0.15 / 1e9)
    assert line["compose"]["bwd"]["value"] == pytest.approx(2 * bench.bwd_bytes(wl.tokens, wl.d_out) / 0.2 / 1e9)
    assert line["ms_per_step"] == pytest.approx(2.0 / 7 * 1e3)
    # roofline fractions are per replica (one GPU's kernel against one GPU's peak)
    assert line["norm"]["frac"] == pytest.approx(F / 0.75 / 1e12 / 1000.0)
    assert line["roofline"]["kernel"] == "norm" and line["roofline"]["traffic"] is None
    assert line["e2e"]["value"] == pytest.approx(2 * F / 1.5 / 1e12)
    assert line["gpu_launches"] == 28 and line["dtype"] == "bf16"
    assert line["config"]["l2"].startswith("no flush")


def _line_for(bench, wl, traffic, flushed=False):
    res = dict(t_total=1.0, t_norm=1e-4, t_fwd=1e-4, t_bwd=1e-4, clocks=None, status=0, wl=wl,
               e2e=dict(t_norm=2e-4, t_fwd=2e-4, t_bwd=2e-4, h2d=10, d2h=20, steps=5), launches=4, flushed=flushed)

    class Args:
        steps, warmup = 1, 3

    return bench.build_line(Args, res, 1, {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}, "test", traffic, None)


def test_traffic_is_taken_only_for_its_own_workload():
    """A traffic row counts only for the workload it was captured on: the
    headline's rows give nothing to the 4096 module, whose line says null."""
    bench = _bench()
    traffic = {("norm", "bf16_8192_r384"): 150e6, ("compose_fwd", "bf16_8192_r384_T8192"): 410e6,
               ("compose_bwd", "bf16_8192_r384_T8192"): 680e6}
    head = _line_for(bench, bench.WL.HEADLINE, traffic)
    assert [k["traffic"] for k in head["rooflines"]] == [150e6, 410e6, 680e6]
    other = _line_for(bench, bench.WL.SINGLE_4096, traffic)
    assert [k["traffic"] for k in other["rooflines"]] == [None, None, None]
    # a headline run with another token count has no compose row either
    t4096 = _line_for(bench, bench.WL.HEADLINE.with_(tokens=4096), traffic)
    assert [k["traffic"] for k in t4096["rooflines"]] == [150e6, None, None]


def test_line_carries_the_step_spread_and_the_unflushed_pass():
    bench = _bench()
    wl = bench.WL.HEADLINE
    res = dict(t_total=2.0, t_norm=1e-4, t_fwd=2e-4, t_bwd=3e-4, clocks=None, status=0, wl=wl,
               e2e=dict(t_norm=2e-4, t_fwd=2e-4, t_bwd=2e-4, h2d=10, d2h=20, steps=5), launches=4, flushed=True,
               unflushed=dict(t_total=2.2, t_norm=1.2e-4, t_fwd=2e-4, t_bwd=3e-4),
               spread={"norm": {"median_us": 99.0, "min_us": 98.0, "max_us": 120.0}})

    class Args:
        steps, warmup = 10, 3

    line = bench.build_line(Args, res, 1, {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}, "test", {}, None)
    assert line["step_time_spread"]["norm"]["max_us"] == 120.0
    F = bench.norm_flops(wl.d_out, wl.d_in, wl.r)
    u = line["steps_without_clean"]
    assert u["norm"]["time_us"] == pytest.approx(120.0)
    assert u["norm"]["tflops"] == pytest.approx(F / 1.2e-4 / 1e12)
    assert u["ms_per_step"] == pytest.approx(2.2 / 10 * 1e3)


def test_dtype_and_l2_follow_the_workload():
    bench = _bench()
    tiny = bench.WL.TINY_F32
    assert bench.step_bytes(tiny) < 2 * bench.L2_BYTES  # the tiny step is flushed before every step
    line = _line_for(bench, tiny, {}, flushed=True)
    assert line["dtype"] == "f32"
    assert line["config"]["l2"].startswith("L2 cleaned before every step")
    # fp32 moves four bytes an element
    assert line["norm"]["bytes"] == bench.norm_bytes(tiny.d_out, tiny.d_in, tiny.r, 4)


def test_reference_arm_runs_on_rank_zero_only(two_ranks):
    assert two_ranks[1]["ref_rc"] == 0
    assert two_ranks[1]["ref_out"] == ""
    assert "line" not in two_ranks[1]


def test_sweep_refuses_several_ranks():
    """The sweep times one GPU; under torchrun every rank would otherwise pick
    cuda:0, so a world size above one is refused before any device work."""
    import subprocess
    import sys

    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--sweep"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert p.returncode != 0
    assert "one GPU" in p.stderr


def test_line_has_every_contract_key(two_ranks):
    line = two_ranks[0]["line"]
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert k in line, k
    assert line["higher_is_better"] is True and line["steps"] == 7 and line["warmup"] == 3
    assert "workload" in line["config"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in line["roofline"], k
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in line["e2e"], k
    assert line["gpu_launches"] > 0
