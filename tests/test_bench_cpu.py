"""bench.py's host side on CPU: the reference arm (the CPU oracle timed on a
bounded sample) prints one line with the benchmark contract's keys, ranks
other than 0 print nothing and do no work, and a recorded ncu traffic figure
is reported only while the kernel's sources still hash to the digest it was
recorded under."""
import json
import os
import re
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CONTRACT_KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                 "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")
DIGEST_FILES = ("ep_layout.cu", "ep_dispatch.cu", "ep_combine.cu", "ep_device.cuh", "ep_internal.h")


def _bench(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          cwd=ROOT, env=e, timeout=600)


def _json_lines(out):
    return [json.loads(line) for line in out.splitlines() if line.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    r = _bench(["--impl", "reference", "--steps", "1", "--warmup", "3"], env={"WORLD_SIZE": "1", "RANK": "0"})
    assert r.returncode == 0, r.stderr
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert all(k in d for k in CONTRACT_KEYS), sorted(set(CONTRACT_KEYS) - set(d))
    assert d["impl"] == "reference"
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 1, 3)
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None
    assert d["config"]["workload"] == "prefill-topk-4096x7168-top8"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    r = _bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
               env={"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert _json_lines(r.stdout) == []


def test_gpus_flag_must_match_the_launcher():
    r = _bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
               env={"WORLD_SIZE": "1", "RANK": "0"})
    assert r.returncode != 0 and "WORLD_SIZE" in (r.stderr + r.stdout)


def _tree(tmp_path):
    """A copy of the files the digests cover, rooted at tmp_path."""
    csrc = tmp_path / "combine_ep_get_10_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in DIGEST_FILES:
        shutil.copy(os.path.join(ROOT, "combine_ep_get_10_b200", "csrc", name), csrc / name)
    (tmp_path / "include").mkdir()
    shutil.copy(os.path.join(ROOT, "include", "ep.h"), tmp_path / "include" / "ep.h")
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_record_is_used_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = {k: bench.source_digest(k) for k in bench.KERNEL_SOURCES}
    assert sha == {k: bench.source_digest(k) for k in bench.KERNEL_SOURCES}  # deterministic
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# a comment line\n"
        "kernel=combine source_sha=%s dram_bytes_per_launch=123 workload=w capture=c\n"
        "kernel=layout source_sha=%s dram_bytes_per_launch=7 workload=w capture=c\n" % (sha["combine"], sha["layout"]))
    assert bench.recorded_traffic("combine") == 123
    assert bench.recorded_traffic("layout") == 7
    assert bench.recorded_traffic("dispatch") is None  # no record
    # editing one kernel's file invalidates its record only
    with open(csrc / "ep_combine.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.source_digest("combine") != sha["combine"]
    assert bench.recorded_traffic("combine") is None
    assert bench.recorded_traffic("layout") == 7
    # a shared header changes every kernel's digest
    with open(csrc / "ep_device.cuh", "a") as f:
        f.write("\n// edited\n")
    assert all(bench.source_digest(k) != sha[k] for k in bench.KERNEL_SOURCES)
    assert bench.recorded_traffic("layout") is None


def test_committed_traffic_record_is_well_formed():
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    seen = set()
    for line in open(path):
        if not line.strip() or line.startswith("#"):
            continue
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        assert f["kernel"] in bench.KERNEL_SOURCES and f["kernel"] not in seen
        seen.add(f["kernel"])
        assert re.fullmatch(r"[0-9a-f]{16}", f["source_sha"])
        assert int(f["dram_bytes_per_launch"]) > 0
        assert f.get("workload") and f.get("capture")
    assert seen == set(bench.KERNEL_SOURCES)
