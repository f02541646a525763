"""The multi-rank logic of bench.py on the CPU: two `gloo` ranks agree on the
slowest rank's time, and the whole-job throughput counts every rank's bytes
over that time (weak scaling: replicas)."""

import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["BENCH_ROOT"])
import bench
ctx = bench.DistCtx(backend="gloo")
ctx.init()
ms_local = 10.0 + 5.0 * ctx.rank            # rank 1 is the slow one
ms = ctx.max(ms_local)
ctx.barrier()
us, gbs_rank, value = bench.step_metrics(1_000_000, ms, 100, ctx.world)
print(json.dumps({"rank": ctx.rank, "world": ctx.world, "ms": ms, "us": us, "value": value}))
ctx.close()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_slowest_time():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), BENCH_ROOT=ROOT)
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2
        assert o["ms"] == 15.0
        assert abs(o["us"] - 150.0) < 1e-9
        # 2 ranks x 1e6 bytes per step over 150 us
        assert abs(o["value"] - 2e6 / 150e-6 / 1e9) < 1e-9


def test_single_rank_metrics():
    sys.path.insert(0, ROOT)
    import bench
    us, gbs, value = bench.step_metrics(15_423_488, 2.0, 100, 1)
    assert abs(us - 20.0) < 1e-12
    assert abs(gbs - 15_423_488 / 20e-6 / 1e9) < 1e-9
    assert value == gbs
