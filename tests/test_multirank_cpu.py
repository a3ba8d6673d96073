"""The N > 1 host logic of bench.py, run as two gloo ranks on the CPU.

The benchmark shards by replica: every rank runs the whole hot path on its
own seeded inputs and the job's time is the slowest rank's.  These tests
exercise that plumbing (process-group setup, max over ranks, barriers,
per-rank inputs, whole-job aggregation) without a GPU, and check that the
reference arm does its work on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist
    import bench
    import seeded_inputs as si

    r, wsz, local = bench.init_dist("gloo")
    assert (r, wsz, local) == (rank, world, rank)
    # each rank "measures" a different time; every rank must see the largest
    my_ms = 2.0 + 3.0 * rank
    job_ms = bench.max_over_ranks(my_ms, wsz, "cpu")
    bench.barrier(wsz)
    w = bench.replica_workload(si.WORKLOADS["tiny"], rank)
    q, _, _ = si.qkv(w)
    digest = int(np.asarray(q).view(np.uint16).astype(np.uint64).sum())
    value = bench.job_tflops(bench.full_flops(w), wsz, job_ms)
    cfg = bench.job_config(w, wsz)
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump({"job_ms": job_ms, "seed": w.seed, "digest": digest, "value": value,
                   "global_batch": cfg["global_batch"]}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    # max over ranks, identical on every rank
    assert [r["job_ms"] for r in res] == [5.0, 5.0]
    # ranks attend over different sequences; rank 0 keeps the 1-GPU inputs
    import seeded_inputs as si
    assert res[0]["seed"] == si.WORKLOADS["tiny"].seed
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["digest"] != res[1]["digest"]
    # whole-job value: both ranks' FLOPs over the slowest rank's time
    import bench
    flops = bench.full_flops(si.WORKLOADS["tiny"])
    assert res[0]["value"] == pytest.approx(2 * flops / 5e-3 / 1e12)
    assert res[0]["value"] == res[1]["value"]
    assert res[0]["global_batch"] == 2 * si.WORKLOADS["tiny"].batch


def _run_reference(rank, world, tmp_path):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT="1")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny", "--steps", "2", "--warmup", "3",
                           "--gpus", str(world)],
                          env=env, capture_output=True, text=True, timeout=300, cwd=str(tmp_path))


def test_reference_arm_runs_on_rank_zero_only(tmp_path):
    other = _run_reference(1, 2, tmp_path)
    assert other.returncode == 0, other.stderr
    assert other.stdout.strip() == ""
    zero = _run_reference(0, 2, tmp_path)
    assert zero.returncode == 0, zero.stderr
    lines = [l for l in zero.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_e2e_loop_runs_as_many_steps_as_the_timed_loop(monkeypatch):
    # the pipelined end-to-end loop spreads its one unoverlapped upload and
    # download over its steps, so by default it runs --steps of them
    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "7"])
    assert bench.parse_args().e2e_steps == 7
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "7", "--e2e-steps", "3"])
    assert bench.parse_args().e2e_steps == 3
