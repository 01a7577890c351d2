"""The benchmark's multi-process plumbing on CPU: two gloo ranks on 127.0.0.1.

bench.py runs one replica per GPU (the path has no exchange step); the only cross-rank
operations are a barrier around the timed region and a MAX all-reduce of the elapsed time.
These run here with the gloo backend, two processes, no GPU.
"""
import os
import socket
import subprocess
import sys

from tests.conftest import ROOT

RANK_SCRIPT = r"""
import json, os, sys
sys.path.insert(0, {root!r})
import bench
d = bench.Dist()
d.init("gloo")
d.barrier()
ms = 10.0 + 5.0 * d.rank          # rank 1 is the slower one
worst = d.max(ms)
d.barrier()
print(json.dumps({{"rank": d.rank, "world": d.world, "max": worst}}))
d.close()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_max_time():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", RANK_SCRIPT.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=120) for p in procs]
    for p, (out, err) in zip(procs, outs):
        assert p.returncode == 0, err
    import json
    res = sorted((json.loads(o.strip().splitlines()[-1]) for o, _ in outs), key=lambda r: r["rank"])
    assert [r["rank"] for r in res] == [0, 1]
    assert all(r["world"] == 2 and r["max"] == 15.0 for r in res)


def test_reference_arm_other_ranks_exit_quietly():
    # under torchrun only rank 0 runs and prints the reference arm; the others exit 0 at once
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
