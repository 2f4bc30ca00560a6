"""Host-side logic of bench.py (no GPU): the committed DRAM-traffic entries and
their source hashes, the peak lookup, and the reference arm (the oracle alone,
on host-built samples)."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_every_traffic_entry_names_a_known_kernel_and_its_capture():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)["entries"]
    assert entries
    for key, e in entries.items():
        workload, kernel = key.split(":", 1)
        assert workload in bench.WORKLOADS, key
        assert kernel.split(" ")[0] in bench.KERNEL_SOURCES, key
        assert os.path.exists(os.path.join(ROOT, e["capture"])), key
        assert e["dram_bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"], key


def test_traffic_is_reported_only_while_the_sources_are_unchanged(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)["entries"]
    key = "kv:decode_kernel"
    e = entries[key]
    monkeypatch.setattr(bench, "source_hash", lambda files: e["source_hash"])
    assert bench.traffic_for("kv", "decode_kernel") == e["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "source_hash", lambda files: "0" * 16)
    assert bench.traffic_for("kv", "decode_kernel") is None
    assert bench.traffic_for("kv", "no_such_kernel") is None


def test_source_hash_follows_code_not_comments(tmp_path, monkeypatch):
    d = tmp_path / "entropy_coded_kv_b200" / "csrc"
    d.mkdir(parents=True)
    f = d / "k.cu"
    f.write_text("// header\nint a = 1; /* note */\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.source_hash(["k.cu"])
    f.write_text("// a longer header\n/* two\n   lines */\n\nint a = 1;   // why\n")
    assert bench.source_hash(["k.cu"]) == h0
    f.write_text("int a = 2;\n")
    assert bench.source_hash(["k.cu"]) != h0


def test_source_hash_covers_every_listed_file():
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "entropy_coded_kv_b200", "csrc", f)), (kernel, f)
        assert len(bench.source_hash(files)) == 16


@pytest.mark.parametrize("content,want", [
    ('{"hbm_gbs": 6532.5}', (6532.5, "measured")),
    ('{"hbm_gbs": {"value": 6400}}', (6400.0, "measured")),
    ('{"bf16_tflops": 1500}', None),
    ('{"hbm_gbs": "n/a"}', None),
    ('not json', None),
])
def test_peak_file_forms(tmp_path, monkeypatch, content, want):
    (tmp_path / "MEASURED_PEAKS.json").write_text(content)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    value, source = bench.peaks()
    if want is None:
        assert value == bench.FALLBACK_HBM_GBS and source.startswith("fallback")
    else:
        assert (value, source) == want


def test_peak_comes_from_the_measured_file_when_present():
    value, source = bench.peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            assert value == float(json.load(f)["hbm_gbs"]) and source == "measured"
    else:
        assert (value, source) == (bench.FALLBACK_HBM_GBS, "fallback")


def test_attention_workload_defaults_to_the_staged_path():
    assert bench.AttnWorkload.path == "staged"


_RUN_AND_LIST_LIBS = (
    "import runpy, sys; sys.argv = ['bench.py'] + sys.argv[1:]; "
    "runpy.run_path('bench.py', run_name='__main__'); "
    "maps = open('/proc/self/maps').read(); "
    "print('LIBS', int('libecco_b200' in maps), int('libecco_oracle' in maps))")


@pytest.mark.parametrize("workload", [None, "c1", "attn"])
def test_reference_arm_runs_the_oracle_alone(workload):
    """The reference arm times the oracle on a host-built sample: it needs no
    device and never maps the product library."""
    args = ["--impl", "reference", "--steps", "1", "--warmup", "1"]
    if workload:
        args += ["--workload", workload]
    r = subprocess.run([sys.executable, "-c", _RUN_AND_LIST_LIBS] + args, capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    out = r.stdout.strip().splitlines()
    line = json.loads(out[-2])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    want = bench.WORKLOADS[workload or "longctx"]
    if want is not bench.AttnWorkload:
        assert line["config"]["workload"] == want.desc
    assert out[-1] == "LIBS 0 1"


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    """Launched the way the scaling run launches it (torchrun, 2 ranks, gloo
    on the host): rank 0 alone times the oracle and prints, the other rank
    exits 0, and the line counts both ranks."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "c1", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
