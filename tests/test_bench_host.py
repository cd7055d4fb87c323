"""bench.py pieces that run without a GPU: the environment record every
result carries, the CPU-baseline leg's shape, the traffic lookup keyed by the
kernel sources, and the algorithmic byte counts the roofline divides by."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_environment_record():
    env = bench.environment()
    for key in ("torch", "cuda_runtime", "kernel_sources_sha256", "command", "driver", "nvcc"):
        assert key in env
    assert len(env["kernel_sources_sha256"]) == 64


def test_cpu_baseline_reports_all_core_and_single_thread_figures():
    w = bench.workload("large_f32")
    r = bench.cpu_baseline(w, 0.5)
    assert r["kind"] == "oracle" and r["unit"] == "elements/s"
    assert r["cores"] == (os.cpu_count() or 1)
    assert r["value"] > 0 and r["single_thread_value"] > 0
    assert "single-threaded oracle" in r["sample"]


def test_traffic_lookup_follows_the_kernel_sources(tmp_path):
    """The committed DRAM figure is used only for the kernel sources it was
    captured from, and scaled from the captured element count."""
    key = "step_kernel/f32_adam"
    rec = {"kernel_source_sha256": bench.kernel_source_sha256(), "captured_numel": 16777216,
           "dram_bytes_read_per_launch": 268.9e6, "dram_bytes_write_per_launch": 145.0e6}
    p = tmp_path / "dram_traffic.json"
    p.write_text(json.dumps({key: rec}))
    got = bench.traffic_for(key, 268435456, str(p))
    assert got == pytest.approx((268.9e6 + 145.0e6) * 16)
    p.write_text(json.dumps({key: dict(rec, kernel_source_sha256="0" * 64)}))
    assert bench.traffic_for(key, 268435456, str(p)) is None     # other sources: no figure
    assert bench.traffic_for("no/such/kernel", 1, str(p)) is None
    committed = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    for k, r in committed.items():
        assert "captured_numel" in r and r["captured_numel"] <= 1 << 26, k   # small-case captures only


def test_algorithmic_bytes_per_element():
    from elementwise_optimizer_b200 import synth
    assert bench.algorithmic_bytes(synth.large_f32()) == 28 * 268_435_456
    tr = synth.transformer_bf16()
    assert bench.algorithmic_bytes(tr) == 30 * tr.numel
    sc = synth.small_collection()
    assert bench.algorithmic_bytes(sc) == sum(n * (28 if d == "f32" else 22)
                                              for n, d in zip(sc.sizes, sc.dtypes))


def test_source_hash_ignores_comments_but_not_code():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "x//y/*z*/";\n'
    assert bench.strip_c_comments(src) == bench.strip_c_comments(
        'int a = 1;\n/* other words */ const char* s = "x//y/*z*/"; // more\n')
    assert bench.strip_c_comments(src) != bench.strip_c_comments(src.replace("a = 1", "a = 2"))
    assert '"x//y/*z*/"' in bench.strip_c_comments(src)
