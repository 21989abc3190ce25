"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Every (sequence, head) chain is independent, so N ranks each run their own
batch (weak scaling) and the only collectives are the barrier and the max
reduction of the timings.  These tests run that logic without a GPU.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        local = [10.0 + 5.0 * rank, 3.0 - rank]
        dist.barrier()
        got = bench.max_over_ranks(local, ws)
        # every rank draws a different batch of the same shape
        from chunkwise_recurrence_b200.inputs import WORKLOADS, generate
        w = WORKLOADS["gdn_b8_h16_t4096_d128_bf16"].with_(B=1, T=8, H=1)
        inp = generate(w, seed=bench.rank_seed(0, rank))
        gathered = [torch.zeros_like(inp.q.float()) for _ in range(ws)]
        dist.all_gather(gathered, inp.q.float())
        q.put((rank, got, [g.sum().item() for g in gathered]))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_sharding():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q))
             for r in range(ws)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, sums in res:
        assert got == [15.0, 3.0]           # max over ranks, element-wise
        assert sums[0] != sums[1]           # different batches per rank


def test_job_throughput_counts_all_ranks():
    # 32768 tokens per rank-step, 2 ranks, 10 steps in 20 ms (slowest rank)
    v = bench.job_throughput(32768, 2, 10, 20.0)
    assert v == pytest.approx(32768 * 2 * 10 / 0.020)
    assert bench.rank_seed(7, 0) != bench.rank_seed(7, 1)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    import json
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--workload", "gdn_b4_h8_t2048_d128_bf16",
                        "--ref-seqs", "1"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _bench(*args, env_extra=None):
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"),
                           *args], capture_output=True, text=True, env=env,
                          timeout=300)


def test_gpus_flag_launches_that_many_ranks():
    # run directly, --gpus 2 re-executes bench.py as two ranks (one per
    # GPU) under torch.distributed.run; the launch check does the rank
    # plumbing over gloo without a GPU and rank 0 alone prints
    r = _bench("--gpus", "2", "--launch-check")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["ranks_seen"] == [0, 1]


def test_gpus_flag_must_match_the_launchers_world_size():
    r = _bench("--gpus", "2", "--launch-check",
               env_extra={"WORLD_SIZE": "3", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode != 0
    assert "WORLD_SIZE=3" in (r.stderr + r.stdout)


def test_relaunch_command_is_one_node_on_loopback():
    cmd = bench.relaunch_command(["--gpus", "4", "--steps", "3"], 4, 29500)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-3:] == ["--gpus", "4", "--steps", "3"][-3:]
