"""Host-side logic of the multi-GPU benchmark, run as two gloo ranks on CPU.

The path shards by sequence (replicas, weak scaling): each rank draws its own
batch from its own seed, and the only collectives are a barrier and the max
over ranks of the timed interval.  These tests exercise exactly that plumbing
without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from long_context_compressed_06_b200 import workloads as W

    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_init(world, backend="gloo")
    cpu = torch.device("cpu")
    # each rank reports a different "step time"; every rank must see the max
    t_local = 0.25 + 0.5 * rank
    t_max = bench.max_over_ranks(t_local, world, cpu)
    bench.barrier(world)
    # per-rank batches are drawn from distinct seeds
    wl = W.TINY.scaled(seed=bench.rank_seed(0, rank))
    q = W.queries(wl, cpu)
    kI = W.index_keys(wl, cpu)
    torch.save({"t_max": t_max, "seed": wl.seed, "q": q, "kI": kI,
                "rate": bench.job_rate(wl.batch * wl.nq, 10, world, t_max)},
               os.path.join(out_dir, "rank%d.pt" % rank))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [torch.load(os.path.join(tmp_path, "rank%d.pt" % r)) for r in range(world)]
    # max over ranks: the slower rank's time, seen identically by both ranks
    assert res[0]["t_max"] == res[1]["t_max"] == 0.75
    # independent batches: different seeds, different data
    assert res[0]["seed"] != res[1]["seed"]
    assert not torch.equal(res[0]["q"], res[1]["q"])
    assert not torch.equal(res[0]["kI"], res[1]["kI"])
    # whole-job rate: all ranks' queries over the slowest rank's time
    assert res[0]["rate"] == pytest.approx(1 * 1 * 10 * 2 / 0.75)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(1.5, 1, torch.device("cpu")) == 1.5
    bench.barrier(1)
    bench.dist_init(1)  # no-op at world size 1
    assert bench.rank_seed(0, 0) == 0
    assert len({bench.rank_seed(0, r) for r in range(8)}) == 8


def _run_bench(env_extra, *args):
    import subprocess
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env, cwd=ROOT,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_line():
    """`bench.py --impl reference` times the oracle on host cores and prints the
    contract's line with the same metric and workload as the GPU arm."""
    import json
    import bench
    from long_context_compressed_06_b200 import workloads as W
    p = _run_bench({}, "--impl", "reference", "--steps", "1", "--warmup", "0")
    assert p.returncode == 0, p.stderr[-2000:]
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "queries/s" and line["higher_is_better"] is True
    assert line["config"] == bench.decode_config(W.CSA_DECODE, 1)
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "queries/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    p = _run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--impl", "reference", "--steps", "1")
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
