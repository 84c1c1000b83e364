"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The forward pass does not shard: with N GPUs, bench.py runs N independent replicas,
one per rank.  These tests check the host side of that path without a GPU: the
process group comes up over gloo, the timing reduction takes the slowest rank, the
ranks draw different seeded inputs of the same shapes, and the whole-job throughput
counts every rank's tokens.  The reference arm (the fp64 oracle) runs on rank 0 only;
the other ranks exit 0 without work.
"""
import json
import os
import socket
import subprocess
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
    sys.path.insert(0, ROOT)
    import bench
    from gtr_inputs import WORKLOADS

    w_, r_, l_ = bench.dist_env()
    dist = bench.init_dist(w_, l_)
    try:
        # every rank reports a different time; all of them must see the largest
        t_max = bench.max_over_ranks(dist, 10.0 + 5.0 * rank, torch.device("cpu"))
        bench.barrier(dist)
        sets = bench.make_sets(WORKLOADS["tiny"], 2, torch.device("cpu"), rank)
        torch.save({"rank": r_, "world": w_, "t_max": t_max,
                    "q0": sets[0][1], "dirs": [s[0] for s in sets]},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        if dist is not None:
            dist.destroy_process_group()


def test_two_gloo_ranks_reduce_the_slowest_time_and_draw_distinct_inputs(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r0 = torch.load(tmp_path / "rank0.pt")
    r1 = torch.load(tmp_path / "rank1.pt")
    assert (r0["rank"], r1["rank"]) == (0, 1) and r0["world"] == r1["world"] == 2
    assert r0["t_max"] == r1["t_max"] == 15.0
    assert r0["dirs"] == r1["dirs"]
    assert r0["q0"].shape == r1["q0"].shape
    assert not torch.equal(r0["q0"], r1["q0"]), "replicas must not time identical inputs"


def test_whole_job_throughput_counts_every_replica():
    import bench
    # two ranks of 10 steps of 1600 tokens; the slower rank took 4 ms
    assert bench.replica_tokens_per_s(2, 10, 1600, 4.0) == pytest.approx(2 * 10 * 1600 / 4e-3)
    assert bench.replica_tokens_per_s(1, 10, 1600, 4.0) == pytest.approx(10 * 1600 / 4e-3)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "3", "--gpus", "2"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    if rank != 0:
        assert lines == []
        return
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2
    assert d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
