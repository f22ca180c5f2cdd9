"""The parts of bench.py that run without a GPU: the reference arm (the fp64 oracle on
the host cores), the rule that reads a kernel's DRAM traffic from its committed ncu
summary only while the kernel source is unchanged, and the cut of the timed steps into
blocks."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_bench(*args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          timeout=600, env=e, cwd=ROOT)


def test_reference_arm_prints_one_line_of_the_contract():
    r = _run_bench("--impl", "reference", "--steps", "2", "--warmup", "3", "--workload", "tiny_fp32")
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["steps"] == 2 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == d["value"] and cpu["cores"] >= 1 and cpu["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny_fp32"


def test_reference_arm_leaves_ranks_other_than_0_idle():
    r = _run_bench("--impl", "reference", "--steps", "1", "--workload", "tiny_fp32",
                   env={"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_warmup_is_at_least_three_steps(monkeypatch):
    seen = {}
    monkeypatch.setattr(bench, "run_gpu", lambda a: seen.setdefault("w", a.warmup) and 0)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--warmup", "1"])
    bench.main()
    assert seen["w"] == 3


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    src_dir = tmp_path / "mla_latent_kv_46_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = src_dir / "decode_2sm.cuh"
    src.write_text("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path, src


def _profile(root, sha, traffic):
    (root / "profiles" / "ncu_decode_attn_wl.md").write_text(
        f"Kernel source: decode_2sm.cuh sha256[:16]: {sha}\n"
        f"| traffic per full launch (bytes): {traffic} | x |\n")


def test_traffic_is_read_while_the_kernel_source_matches(fake_root):
    root, src = fake_root
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    _profile(root, sha, 123456789)
    assert bench.traffic_record("wl", 128, 1) == (123456789, sha)


def test_traffic_is_dropped_once_the_kernel_source_changed(fake_root):
    root, src = fake_root
    old = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    _profile(root, old, 123456789)
    src.write_text("// kernel v2\n")
    new = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    assert bench.traffic_record("wl", 128, 1) == (None, new)


def test_traffic_needs_a_summary_of_that_workload(fake_root):
    root, src = fake_root
    assert bench.traffic_record("other", 128, 1)[0] is None


def test_decode_kernel_follows_the_library_dispatch():
    assert bench.decode_kernel_of(128, 1)[0] == "decode_2sm.cuh"
    assert bench.decode_kernel_of(64, 2)[0] == "decode_2sm.cuh"
    assert bench.decode_kernel_of(64, 1)[0] == "decode_2sm.cuh"
    assert bench.decode_kernel_of(192, 1)[0] == "decode_tc.cuh"


@pytest.mark.parametrize("steps", [1, 2, 3, 4, 5, 7, 50, 200, 201])
def test_timing_blocks_cover_every_step_once(steps):
    """The timed steps are cut into at most four blocks of near-equal size (each followed
    by as many bracketed steps): together exactly `steps`, sizes one apart at most."""
    b = bench.timing_blocks(steps)
    assert sum(b) == steps and 1 <= len(b) <= 4 and min(b) >= 1 and max(b) - min(b) <= 1

