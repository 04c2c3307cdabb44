"""The multi-process plumbing of bench.py at world size 2, on CPU with gloo.

The decode path does not shard (one layer's step is a few microseconds of work), so
`bench.py --gpus N` runs N independent replicas: every rank decodes its own synthetic
sequence, the timed region is bracketed by barriers, the slowest rank's time counts, and
the value is the work of all ranks over that time. These tests check that plumbing without
a GPU: the rank helpers, per-rank inputs, and the reference arm under torchrun.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["QSA_ROOT"])
import numpy as np
import bench, synth
world, rank, local = bench.dist_setup(2)
bench.barrier(world)
slowest = bench.max_over_ranks(10.0 + rank, world)
wl = synth.workload("tiny")
packed, views = synth.device_steps(wl, 2, 3, device="cpu", rank=rank)
with open(os.path.join(os.environ["QSA_OUT"], f"rank{rank}.json"), "w") as f:
    json.dump({"rank": rank, "world": world, "max": slowest,
               "q0": views["q"][0, 0, :4].float().tolist(), "k_sum": float(views["k"].float().sum())}, f)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _torchrun(args, timeout=240, out_dir=""):
    env = dict(os.environ, QSA_ROOT=ROOT, QSA_OUT=str(out_dir), CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", *args]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def test_rank_helpers_and_per_rank_inputs(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(_WORKER)
    r = _torchrun([str(script)], out_dir=tmp_path)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [json.loads((tmp_path / f"rank{i}.json").read_text()) for i in range(2)]
    assert sorted(x["rank"] for x in lines) == [0, 1]
    assert all(x["world"] == 2 for x in lines)
    assert all(x["max"] == 11.0 for x in lines)          # the slowest rank's time, on every rank
    a, b = sorted(lines, key=lambda x: x["rank"])
    assert a["q0"] != b["q0"] and a["k_sum"] != b["k_sum"]  # each replica decodes its own sequence


@pytest.mark.slow
def test_reference_arm_prints_once_under_torchrun():
    r = _torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "2",
                   "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
