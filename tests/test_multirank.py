"""The N>1 path of bench.py on the CPU: two ranks over the gloo backend.

Every rank runs its own replica of the workload (weak scaling, no collective
on the data path); the only cross-rank steps are the barriers around the
timed region and the max-over-ranks reduction of the measured times.  These
tests drive exactly those steps, the per-rank input draw, the whole-job
aggregate and the rank-0-only output, with world size 2 on 127.0.0.1.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth_inputs import WORKLOADS, draw_workload  # noqa: E402

WORLD = 2


def free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # times as the bench measures them, different on each rank
        step, fwd, bwd, mask = 1.0 + rank, 0.25 * (1 - rank) + 0.5, 0.7 + 0.1 * rank, 0.03 - 0.01 * rank
        dist.barrier()
        red = bench.max_over_ranks([step, fwd, bwd, mask], WORLD)
        e2e = bench.max_over_ranks([5.0 - rank], WORLD)[0]
        # each rank's inputs
        w, _ = bench.parse_workload("tiny:none")
        bits = draw_workload(bench.rank_workload(w, rank))
        digest = {n: int(np.bitwise_xor.reduce(bits[n].ravel().astype(np.uint64) * np.uint64(2654435761)
                                                  + np.arange(bits[n].size, dtype=np.uint64)))
                  for n in ("q", "k", "v", "dout")}
        shapes = {n: list(bits[n].shape) for n in ("q", "k", "v", "dout")}
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, {"digest": digest, "shapes": shapes})
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"red": red, "e2e": e2e, "gathered": gathered}, f)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_rank_results(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    mp.start_processes(_rank_main, args=(free_port(), str(out)), nprocs=WORLD, join=True, start_method="spawn")
    return [json.load(open(out / f"rank{r}.json")) for r in range(WORLD)]


def test_times_are_max_over_ranks(two_rank_results):
    expect = [2.0, 0.75, 0.8, 0.03]
    for r in two_rank_results:
        assert r["red"] == pytest.approx(expect)
        assert r["e2e"] == pytest.approx(5.0)


def test_every_rank_sees_the_same_reduction(two_rank_results):
    assert two_rank_results[0]["red"] == two_rank_results[1]["red"]
    assert two_rank_results[0]["e2e"] == two_rank_results[1]["e2e"]


def test_ranks_draw_independent_inputs_of_the_same_shape(two_rank_results):
    g = two_rank_results[0]["gathered"]
    assert g == two_rank_results[1]["gathered"]
    assert g[0]["shapes"] == g[1]["shapes"]
    for n in ("q", "k", "v", "dout"):
        assert g[0]["digest"][n] != g[1]["digest"][n]


def test_rank0_replica_is_the_single_gpu_workload():
    w = WORKLOADS["dense"]
    assert bench.rank_workload(w, 0) == w
    a = draw_workload(bench.rank_workload(WORKLOADS["tiny"], 0))
    b = draw_workload(WORKLOADS["tiny"])
    for n in ("q", "k", "v", "dout"):
        assert np.array_equal(a[n], b[n])


def test_single_rank_reduction_is_identity():
    assert bench.max_over_ranks([3.0, 1.0], 1) == [3.0, 1.0]


def test_job_throughput_scales_with_world():
    f = 4.4e12
    one = bench.job_throughput(f, 1, 2.0)
    assert one == pytest.approx(f / 2e-3 / 1e12)
    assert bench.job_throughput(f, 2, 2.0) == pytest.approx(2 * one)
    # a slower rank sets the job's time
    assert bench.job_throughput(f, 2, 4.0) == pytest.approx(one)


def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={WORLD}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", str(WORLD),
           "--workload", "tiny:none", "--steps", "1", "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=240)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == WORLD
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"
