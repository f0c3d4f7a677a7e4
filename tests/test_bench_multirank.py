"""The N > 1 path of bench.py on CPU: world size 2 over gloo.

Under torchrun every rank runs its own replica of the workload (the units are
independent; the only collectives are the timing barrier and one max
all-reduce of the device time). These tests run two real processes with a
gloo process group on 127.0.0.1 and check the whole-job aggregation, the
per-rank inputs and the reference arm's rank behaviour. No GPU is used.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_RANK = r"""
import datetime, json, sys
import torch, torch.distributed as dist
sys.path.insert(0, sys.argv[1])
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
total_ms = [10.0, 12.5][rank]           # this rank's timed device milliseconds
ms, value = bench.aggregate_over_ranks(total_ms, 5, 2.0e12, world, torch.device("cpu"))
print(json.dumps({"rank": rank, "ms_per_step": ms, "value": value,
                  "seed": bench.replica_seed(1, rank)}))
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(code_args, world=2, extra_env=None):
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen(code_args, cwd=ROOT, env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    return outs


def test_two_ranks_take_the_slowest_device_time():
    outs = _launch([sys.executable, "-c", _RANK, ROOT])
    res = sorted((json.loads(o) for o in outs), key=lambda r: r["rank"])
    for r in res:
        # both ranks see the max over ranks (12.5 ms over 5 steps) ...
        assert abs(r["ms_per_step"] - 2.5) < 1e-12
        # ... and the whole-job throughput counts the work of both replicas
        assert abs(r["value"] - 2 * 2.0e12 / 2.5e-3 / 1e12) < 1e-6
    assert res[0]["seed"] != res[1]["seed"]


def test_reference_arm_prints_on_rank_zero_only():
    """Under torchrun the reference arm runs on rank 0 alone; the other ranks
    exit 0 without work or output (checked for rank 1)."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.strip() == ""


def test_gpus_must_match_the_world_size():
    """--gpus N without N ranks (or N ranks with another --gpus) stops with an
    error before any work, instead of printing a line for the wrong N."""
    for gpus, env_world in ((2, None), (1, "2")):
        env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
        env.pop("WORLD_SIZE", None)
        if env_world:
            env.update(RANK="0", LOCAL_RANK="0", WORLD_SIZE=env_world)
        res = subprocess.run([sys.executable, "bench.py", "--gpus", str(gpus), "--steps", "1",
                              "--warmup", "3"], cwd=ROOT, env=env, capture_output=True,
                             text=True, timeout=300)
        assert res.returncode != 0, (gpus, env_world)
        assert res.stdout.strip() == ""
        assert "WORLD_SIZE" in res.stderr
