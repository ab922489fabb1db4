"""The multi-rank host path of bench.py on CPU: two gloo ranks (world size 2, 127.0.0.1)
join the group, agree on the max-over-ranks device time, aggregate the whole-job value, and
only rank 0 runs the reference arm (no GPU is touched)."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["DLMH_ROOT"])
import bench
world, rank, local = bench.dist_setup(None, backend="gloo")
elapsed = 10.0 + 5.0 * rank            # rank 1 is the slow one
m = bench.max_over_ranks(elapsed, world)
bench.barrier(world)
v = bench.job_value(world, 4, 1e9, m)
print(json.dumps({"rank": rank, "world": world, "max": m, "value": v}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(code, world=2, extra_env=None, args=()):
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), DLMH_ROOT=ROOT, CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        cmd = [sys.executable, "-c", code] if code else [sys.executable, os.path.join(ROOT, "bench.py"), *args]
        procs.append(subprocess.Popen(cmd, env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    return outs


def test_two_gloo_ranks_agree_on_max_time_and_job_value():
    outs = _launch(CHILD)
    lines = [json.loads(o.strip().splitlines()[-1]) for o in outs]
    for d in lines:
        assert d["world"] == 2
        assert d["max"] == 15.0                       # the slowest rank's time, on every rank
        assert d["value"] == pytest.approx(2 * 4 * 1e9 / 15e-3 / 1e9)


def test_reference_arm_runs_on_rank_zero_only():
    outs = _launch(None, args=("--impl", "reference", "--steps", "1", "--warmup", "3"))
    printed = [o.strip() for o in outs]
    assert printed[1] == ""                           # rank 1 exits without work
    line = json.loads(printed[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
