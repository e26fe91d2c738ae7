"""The multi-rank host path of bench.py on CPU with two gloo ranks: the job runs independent
replicas (each rank its own seeded batch, no data-path collective), the job time is the max over
ranks, the value counts every rank's work, and the reference arm prints on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        job_ms = bench.max_over_ranks(local_ms, world, "cpu")
        c = workloads.config(1)
        q, _, _ = workloads.make_inputs(c["b"], c["hq"], c["hk"], c["sq"], c["sk"], c["dqk"],
                                        c["dv"], bench.rank_seed(c["seed"], rank))
        digest = float(q.float().sum())
        all_digests = [None] * world
        dist.all_gather_object(all_digests, digest)
        out[rank] = {"job_ms": job_ms, "digests": all_digests}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_and_max_time():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    for r in range(world):
        assert out[r]["job_ms"] == 5.0  # the slowest rank sets the job's time
    d = out[0]["digests"]
    assert d[0] != d[1]  # each rank draws its own batch
    sys.path.insert(0, ROOT)
    import bench
    # the whole-job value counts both ranks' work over the slowest rank's time
    assert abs(bench.job_value(2, 1e12, 5.0) - 2 * 1e12 / 5e-3 / 1e12) < 1e-9


def test_reference_arm_prints_on_rank_zero_only():
    outs = []
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
        p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--config", "1", "--steps", "1", "--warmup", "0"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert p.returncode == 0, p.stderr[-2000:]
        outs.append(p.stdout.strip())
    assert outs[1] == ""
    line = json.loads(outs[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def test_reference_line_carries_the_contract_keys():
    """The reference arm's JSON line has every key of the benchmark contract, with its own
    cpu_baseline and an e2e that moves no bytes."""
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "1", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"),
                       capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    line = json.loads(p.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl", "gpu_launches"):
        assert key in line, key
    assert line["steps"] == 1 and line["warmup"] == 0 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "mha_b1_h2_s128_d64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
