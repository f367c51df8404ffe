"""The benchmark's multi-rank plumbing at world size 2 on CPU (gloo): the
process group comes up from the torchrun environment, the step time is the
max over ranks, whole-job throughput counts every rank's units, each rank
draws its own seeded batch, and only rank 0 prints (the reference arm runs on
rank 0 alone and the other ranks exit 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import synth
    r, w, local = bench.dist_init()
    assert (r, w, local) == (rank, world, rank)
    # a slower rank 1: the job's step time is its time on every rank
    local_ms = 10.0 + 5.0 * rank
    bench.barrier(w)
    ms_max = bench.max_over_ranks(local_ms, w)
    value = bench.job_rate(64, w, ms_max)
    # each rank's batch comes from its own seed
    s = bench.dataclass_seed(synth.FLASH_DECODE, rank)
    inp = synth.decode_inputs(s, device="cpu", batch=1)
    digest = float(inp["q"].float().sum())
    bench.barrier(w)
    bench.dist_done(w)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"ms_max": ms_max, "value": value, "seed": s.seed, "digest": digest}, f)


def test_two_ranks_max_time_and_job_rate(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    # max over ranks: both ranks report the slower rank's 15 ms
    assert res[0]["ms_max"] == res[1]["ms_max"] == 15.0
    # whole-job throughput: 2 ranks x 64 queries per 15 ms
    assert res[0]["value"] == res[1]["value"] == pytest.approx(2 * 64 / 0.015)
    # independent batches per rank (weak scaling over distinct problems)
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["digest"] != res[1]["digest"]


def test_job_rate_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_rate(64, 1, 0.25) == pytest.approx(256000.0)
    assert bench.job_rate(64, 4, 0.5) == pytest.approx(4 * 128000.0)


def test_reference_arm_under_torchrun_prints_once_on_rank0(tmp_path):
    """`bench.py --impl reference` launched like the multi-GPU bench: rank 0
    times the oracle and prints the one JSON line, rank 1 exits 0 silently."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "hca_decode"]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
