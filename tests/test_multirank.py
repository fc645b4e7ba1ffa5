"""World-size-2 checks of the benchmark's multi-rank host logic on CPU (gloo).

The hot path has no exchange step: a run on N GPUs is N independent replicas,
joined only for the timing barrier and the max over ranks. These tests run
that plumbing as two gloo processes and check what rank 0 reports.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_RANK_SCRIPT = r"""
import json, os, sys
sys.path.insert(0, os.environ["ROOT"])
import bench
world, rank, local = bench.dist_setup(2, backend="gloo")
assert (world, rank, local) == (2, int(os.environ["RANK"]), int(os.environ["LOCAL_RANK"]))
bench.barrier(world)
# rank 1 is the slow one: the job's time is the larger of the two
mine = 10.0 if rank == 0 else 25.0
slowest = bench.max_over_ranks(mine, world)
us = bench.whole_job_us_per_layer(slowest, steps=5, world=world)
bench.barrier(world)
import torch.distributed as dist
dist.destroy_process_group()
print(json.dumps({"rank": rank, "slowest": slowest, "us": us}))
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(script: str, world: int, extra_env=None, timeout=120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, ROOT=ROOT, RANK=str(r), LOCAL_RANK=str(r),
                   WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                   CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    outs = []
    try:
        for p in procs:
            out, err = p.communicate(timeout=timeout)
            outs.append((p.returncode, out, err))
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    return outs


def test_two_rank_timing_is_max_over_ranks():
    import json
    outs = _launch(_RANK_SCRIPT, 2)
    for rc, out, err in outs:
        assert rc == 0, err
    lines = [json.loads(o.strip().splitlines()[-1]) for _, o, _ in outs]
    for ln in lines:
        assert ln["slowest"] == 25.0
        # 2 ranks x 5 steps = 10 layers in 25 ms -> 2500 us per layer
        assert ln["us"] == pytest.approx(2500.0)


def test_whole_job_value_scales_with_ranks():
    sys.path.insert(0, ROOT)
    import bench
    # same per-rank time on twice the ranks: twice the layers, half the us/layer
    assert bench.whole_job_us_per_layer(10.0, 4, 1) == pytest.approx(2500.0)
    assert bench.whole_job_us_per_layer(10.0, 4, 2) == pytest.approx(1250.0)


_REF_SCRIPT = r"""
import os, sys
sys.path.insert(0, os.environ["ROOT"])
import bench
sys.argv = ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
bench.main()
"""


def test_reference_arm_non_zero_rank_exits_without_work():
    # rank 1 of the reference arm does no work, prints nothing and joins no group
    outs = _launch(_REF_SCRIPT, 2, extra_env={"RANK": "1"}, timeout=60)
    for rc, out, err in outs:
        assert rc == 0, err
        assert out.strip() == ""
