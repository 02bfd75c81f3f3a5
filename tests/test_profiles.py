"""The committed profiler summaries: every command they give runs committed
files only, and the bench reports a recorded DRAM traffic figure only while
the kernel's sources are the ones it was captured on."""
import json
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _tracked():
    out = subprocess.run(["git", "ls-files"], capture_output=True, text=True, cwd=ROOT)
    assert out.returncode == 0
    return set(out.stdout.split())


def test_profile_commands_run_committed_files_only():
    tracked = _tracked()
    pdir = os.path.join(ROOT, "profiles")
    names = sorted(f for f in os.listdir(pdir) if f.endswith(".md"))
    assert names
    for name in names:
        text = open(os.path.join(pdir, name)).read()
        assert "_work" not in text, name
        blocks = [b.replace("\\\n", " ") for b in re.findall(r"```\n(.*?)```", text, flags=re.S)]
        assert blocks, f"{name} gives no command"
        scripts = re.findall(r"python3? (?:-m )?([\w/.-]+\.py)", "\n".join(blocks))
        assert scripts, f"{name}: no python command"
        for s in scripts:
            assert s in tracked, f"{name} runs {s}, which is not committed"
        for cmd in re.findall(r"^ncu .*$", "\n".join(blocks), flags=re.M):
            if " -i " not in cmd:
                assert "--clock-control none" in cmd, f"{name}: {cmd}"


def test_traffic_records_are_reported_only_for_current_sources(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for key, r in rec.items():
        kernel, workload = key.split(":", 1)
        assert r["command"].startswith("ncu ") and "--clock-control none" in r["command"]
        current = bench.kernel_source_hash(kernel) == r["source_hash"]
        got = (bench.recorded_traffic_ratio(kernel, workload)
               if "traffic_over_algorithmic" in r else bench.recorded_traffic(kernel, workload))
        assert (got is not None) == current, key
    # a changed source voids every record
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel: "0" * 16)
    for key, r in rec.items():
        kernel, workload = key.split(":", 1)
        assert bench.recorded_traffic_ratio(kernel, workload) is None
        assert bench.recorded_traffic(kernel, workload) is None
