"""Host-side helpers of bench.py (no GPU): the profile-summary traffic lookup
and its source hashing, workload accounting, and the reference arm's JSON
line on the chunk workload."""
import json
import os
import subprocess
import sys

import pytest

import bench
from structured_attention_video_monarch_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_region_hash_covers_only_the_marked_launch_code(tmp_path, monkeypatch):
    csrc = tmp_path / "structured_attention_video_monarch_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("kernel v1\n")
    (csrc / "host.cu").write_text("entry A\n// <launch>\nlaunch v1\n// </launch>\nentry B\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "kern", ("k.cuh", "host.cu#launch"))
    h0 = bench.kernel_sources_sha256("kern")
    # code outside the region does not change the hash ...
    (csrc / "host.cu").write_text("entry A changed\n// <launch>\nlaunch v1\n// </launch>\nentry C\n")
    assert bench.kernel_sources_sha256("kern") == h0
    # ... the region and the kernel's own file do
    (csrc / "host.cu").write_text("entry A\n// <launch>\nlaunch v2\n// </launch>\nentry B\n")
    h1 = bench.kernel_sources_sha256("kern")
    assert h1 != h0
    (csrc / "k.cuh").write_text("kernel v2\n")
    assert bench.kernel_sources_sha256("kern") != h1
    # a missing region is an error, not a silent hash of nothing
    (csrc / "host.cu").write_text("no markers\n")
    with pytest.raises(ValueError):
        bench.kernel_sources_sha256("kern")


def test_captured_traffic_requires_a_matching_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "structured_attention_video_monarch_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cuh").write_text("kernel\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "kern", ("k.cuh",))
    h = bench.kernel_sources_sha256("kern")
    summary = tmp_path / "profiles" / "kern_wl.md"
    summary.write_text(f"# x\n\n    kernel_sources_sha256: {h}\n    traffic_bytes_per_launch: 1234\n")
    assert bench.captured_traffic("wl", "kern") == 1234.0
    assert bench.captured_traffic("other", "kern") is None   # no summary for that workload
    (csrc / "k.cuh").write_text("kernel changed\n")
    assert bench.captured_traffic("wl", "kern") is None      # counters predate the change


def test_committed_profiles_name_their_hash_and_traffic():
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        if not name.endswith(".md"):
            continue
        text = open(os.path.join(ROOT, "profiles", name)).read()
        assert "kernel_sources_sha256:" in text and "traffic_bytes_per_launch:" in text, name
        assert "--clock-control none" in text, name


@pytest.mark.parametrize("name", sorted(workloads.BY_NAME))
def test_workload_accounting(name):
    wl = workloads.BY_NAME[name]
    bhd = wl.B * wl.heads * wl.d
    es = 4 if wl.dtype == "f32" else 2
    if wl.grad:  # 10*d FLOPs per (query, key) pair; read Q, K, V, dO, write dQ, dK, dV
        assert wl.flops == 10.0 * wl.N * (wl.m + wl.b) * bhd
        assert wl.io_bytes == 7 * wl.N * bhd * es
        return
    assert wl.flops == 4.0 * wl.N * (wl.m + wl.b) * bhd
    extra = wl.N + 2 * wl.N_ctx if wl.T_ctx else 0
    assert wl.io_bytes == (4 * wl.N + extra) * bhd * es
    if wl.fact == workloads.FACT_ROW:
        assert (wl.m, wl.b) == (wl.W, wl.T * wl.H)


def test_reference_arm_line_for_the_chunk_workload():
    # the reference arm times the oracle's chunk form on whole heads; one short step
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "4"))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "chunk_ar_bf16", "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and "head(s) of the chunk" in line["cpu_baseline"]["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert "context frames" in line["config"]["workload"]


def test_traffic_source_explains_a_null_traffic(tmp_path, monkeypatch):
    csrc = tmp_path / "structured_attention_video_monarch_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cuh").write_text("kernel\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "kern", ("k.cuh",))
    assert bench.traffic_source("wl", "kern").startswith("none: no ncu summary")
    h = bench.kernel_sources_sha256("kern")
    (tmp_path / "profiles" / "kern_wl.md").write_text(
        f"    kernel_sources_sha256: {h}\n    traffic_bytes_per_launch: 5\n")
    assert bench.traffic_source("wl", "kern").startswith("profiles/kern_wl.md")
    (csrc / "k.cuh").write_text("kernel changed\n")
    assert "earlier sources" in bench.traffic_source("wl", "kern")
