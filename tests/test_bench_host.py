"""bench.py host logic on CPU: the algorithmic work counts and the multi-rank
helpers (gloo, world size 2: max over ranks, barrier, rank-0-only reference arm)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from selective_state_space_22_b200 import inputs  # noqa: E402


def test_algorithmic_counts_mamba2_layer():
    # x and y bf16 (2 x 33.55 MB), dt 1.05 MB, B and C bf16 2.10 MB, final state 4.19 MB
    assert bench.algorithmic_bytes(inputs.MAMBA2_1B) == 74_449_408
    # per (b, h, chunk of 256): 2*256*257/2*64 + 2*(2*256*128*64); plus C B^T per (b, chunk)
    assert bench.algorithmic_flops(inputs.MAMBA2_1B) == 13_036_421_120


def test_algorithmic_bytes_backward():
    # float32: x, dy, dx 3 x 67.11 MB; dt, ddt 2 x 1.05 MB; B, C, dB, dC 4 x 1.05 MB;
    # init_state, dfinal, dinit 3 x 4.19 MB; A, D, dA, dD 4 x 256 B
    tok = 2 * 2048
    expect = 3 * tok * 64 * 64 * 4 + 2 * tok * 64 * 4 + 4 * tok * 128 * 4 + 3 * 2 * 64 * 64 * 128 * 4 + 4 * 64 * 4
    assert bench.bwd_bytes(inputs.BWD) == expect == 224_396_288


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


WORKER = r"""
import os, sys, json
sys.path.insert(0, {root!r})
import bench
rank, world = bench.dist_init("gloo")
bench.dist_barrier()
m = bench.dist_max(float(rank + 1) * 1.5)
print(json.dumps({{"rank": rank, "world": world, "max": m}}))
import torch.distributed as dist
dist.destroy_process_group()
"""


def test_dist_max_two_ranks_gloo(tmp_path):
    port = _free_port()
    script = tmp_path / "w.py"
    script.write_text(WORKER.format(root=ROOT))
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=120) for p in procs]
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e
    res = [json.loads(o.strip().splitlines()[-1]) for o, _ in outs]
    assert all(r["world"] == 2 and r["max"] == 3.0 for r in res)


def test_reference_arm_two_ranks_only_rank0_prints(tmp_path):
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "tiny-real-f32"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0
