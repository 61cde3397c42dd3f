"""Multi-rank host logic of the benchmark on CPU: two gloo ranks.

The layer does not shard: `bench.py --gpus N` runs N independent replicas and
the only cross-rank steps are a barrier around the timed region and a MAX
reduction of the elapsed time. These tests run that plumbing as two processes
over gloo on 127.0.0.1, with no GPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["REPO_ROOT"])
import bench
ws, rank, local = bench.dist_setup()
assert ws == 2 and rank == int(os.environ["RANK"])
bench.barrier(ws)
# rank r reports (r + 1) * 1.5 ms: every rank must see the slower rank's time
t = bench.max_over_ranks((rank + 1) * 1.5, ws)
bench.barrier(ws)

class A:  # the reference arm's arguments; ranks other than 0 must return at once
    steps, warmup, ref_tokens, workload = 1, 3, 2, "prefill8k"
ref = bench.run_reference(A, ws, rank) if rank != 0 else None
import torch.distributed as dist
dist.destroy_process_group()
print(json.dumps({"rank": rank, "max": t, "ref_is_none": ref is None}), flush=True)
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_share_barrier_and_max_time():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                   RANK=str(r), LOCAL_RANK=str(r), REPO_ROOT=ROOT, CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("gloo ranks did not finish")
        assert p.returncode == 0, e[-2000:]
        outs.append(json.loads(o.strip().splitlines()[-1]))
    assert sorted(o["rank"] for o in outs) == [0, 1]
    for o in outs:
        assert o["max"] == pytest.approx(3.0)
        assert o["ref_is_none"]

