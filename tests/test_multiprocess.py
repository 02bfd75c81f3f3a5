"""The benchmark's multi-rank plumbing on CPU: world size 2 over gloo. The
forward path shards as independent replicas, so the ranks only meet in a
barrier and a max over their timings; the reference arm runs on rank 0 alone
and the other ranks exit without output."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_RANK_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r})
import bench
d = bench.Dist()
d.init("gloo")
d.barrier()
v = d.max(float(10 + 5 * d.rank))
d.barrier()
print("RESULT", d.rank, d.world, v, flush=True)
d.close()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _launch(args_for_rank, world=2):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen(args_for_rank(r), env=env, cwd=ROOT, text=True,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    return outs


def test_barrier_and_max_over_two_gloo_ranks():
    script = _RANK_SCRIPT.format(root=ROOT)
    outs = _launch(lambda r: [sys.executable, "-c", script])
    for r, out in enumerate(outs):
        line = [l for l in out.splitlines() if l.startswith("RESULT")][0].split()
        assert int(line[1]) == r and int(line[2]) == 2
        assert float(line[3]) == 15.0  # the max over ranks, seen by both


def test_reference_arm_prints_on_rank_zero_only():
    outs = _launch(lambda r: [sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                              "reference", "--workload", "1", "--steps", "1", "--warmup", "1",
                              "--gpus", "2"])
    lines0 = [l for l in outs[0].splitlines() if l.startswith("{")]
    assert len(lines0) == 1 and json.loads(lines0[0])["n_gpus"] == 2
    assert not [l for l in outs[1].splitlines() if l.startswith("{")]
