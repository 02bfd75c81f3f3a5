"""The benchmark's reference arm (the float64 oracle on the host cores) runs
on CPU and prints one JSON line with the keys its contract requires."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "1", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["config"]["workload"].startswith("tiny")
    # the library arm prints the same static dict (bench_config) for its config
    sys.path.insert(0, ROOT)
    import bench
    import synth
    assert d["config"] == bench.bench_config(synth.WORKLOADS[1])
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["quantize"]["GB/s"] > 0  # the oracle's quantizer on a bounded sample
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


class _RecordingContext:
    """Stands in for mpe.Context: records the order of queued calls and waits
    and checks that a buffer set is never queued again before its previous
    call was waited for."""

    def __init__(self):
        self.log = []
        self.pending = {}   # buffer set id -> ticket not yet waited for
        self.next = 0

    def moe_ffn_host_async(self, xh, ih, wh, oh):
        key = id(oh)
        assert key not in self.pending, "buffer set reused while its call is in flight"
        t = self.next
        self.next += 1
        self.pending[key] = t
        self.log.append(("queue", t, key))
        return t

    def wait_host(self, t):
        self.log.append(("wait", t))
        for k, v in list(self.pending.items()):
            if v <= t:
                del self.pending[k]


def test_e2e_pipeline_queues_ahead_and_waits_every_step():
    sys.path.insert(0, ROOT)
    import bench
    ctx = _RecordingContext()
    sets = [tuple(object() for _ in range(4)) for _ in range(2)]
    bench.e2e_pipeline(ctx, sets, 7)
    queues = [e for e in ctx.log if e[0] == "queue"]
    waits = [e[1] for e in ctx.log if e[0] == "wait"]
    assert [q[1] for q in queues] == list(range(7))
    assert waits == list(range(7))  # every step's result is read back, in order
    # step i is queued before step i - 1 is waited for (one call in flight ahead)
    for i in range(1, 7):
        assert ctx.log.index(("queue", i, queues[i][2])) < ctx.log.index(("wait", i - 1))
    # the two buffer sets alternate
    assert [q[2] for q in queues] == [id(sets[i % 2][3]) for i in range(7)]
    assert not ctx.pending


def test_reference_arm_one_layer_at_one_width():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "1", "--width", "8", "--experts", "4", "--tokens", "8",
                        "--topk", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    sys.path.insert(0, ROOT)
    import bench
    wl = bench.bench_workload(1, experts=4, tokens=8, topk=2, width=8)
    assert (wl.E, wl.T, wl.k, wl.H, wl.F) == (4, 8, 2, 256, 512)
    assert d["config"] == bench.bench_config(wl, 8)
    assert d["config"]["workload"] == "tiny-layer-e4-h256-f512-t8-top2-w8"
    assert d["config"]["width"] == 8 and d["config"]["avg_bits_budget"] is None
    assert d["cpu_baseline"]["quantize"]["sample"].endswith("at 8 bits")
    # a layer of the repaging workload's shape is not the schedule
    assert not bench.is_schedule(bench.bench_workload(5, width=3))
    assert bench.is_schedule(bench.bench_workload(5))
    assert bench.bench_workload(2) is bench.bench_workload(2, None, None, None, None)


def test_layer_flags_are_checked():
    for extra in (["--variant", "prefix", "--width", "3"], ["--topk", "0"], ["--experts", "0"]):
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                            "reference", "--workload", "1", "--steps", "1"] + extra,
                           capture_output=True, text=True, timeout=120, cwd=ROOT)
        assert r.returncode == 2 and "error" in r.stderr, extra


def test_forced_path_is_in_the_config_and_limited_to_one_layer():
    sys.path.insert(0, ROOT)
    import bench
    import synth
    wl = synth.WORKLOADS[3]
    assert bench.bench_config(wl)["path"] == "streaming"
    assert bench.bench_config(wl, path_flag="prefill")["path"] == "tensor-core"
    assert bench.bench_config(synth.WORKLOADS[4], path_flag="decode")["path"] == "streaming"
    # the L2 note follows the workload, not the forced path
    assert "264 MB" not in bench.bench_config(wl, path_flag="prefill")["l2"]
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "5", "--path", "prefill", "--steps", "1"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode == 2 and "--path applies to one layer" in r.stderr
