"""Host-side logic of bench.py that needs no GPU: the source hash that keys
recorded ncu counters, the reference arm's per-step sample size, the
per-rank helpers' arithmetic and the roofline's algorithmic bytes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads  # noqa: E402


def test_comment_stripping_keeps_code_and_strings():
    src = 'int a; // tail\n/* block\n comment */ const char *s = "a//b/*c*/\\"d"; int b;\n\n'
    out = bench._strip_comments(src)
    assert "tail" not in out and "block" not in out and "comment" not in out
    assert '"a//b/*c*/\\"d"' in out
    assert "int a;" in out and "int b;" in out


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "block_causal_linear_rope_b200" / "csrc"
    csrc.mkdir(parents=True)
    f = csrc / "k.cuh"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f.write_text("int x = 1; // one\n")
    h1 = bench.kernel_source_hash()
    f.write_text("int x = 1; // a different comment\n/* and a block */\n")
    assert bench.kernel_source_hash() == h1
    f.write_text("int x = 2; // one\n")
    assert bench.kernel_source_hash() != h1


def test_recorded_traffic_requires_matching_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "block_causal_linear_rope_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("int y;\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    import json
    doc = {"source_hash": bench.kernel_source_hash(), "per_launch_bytes": {"480p": {"output": 123}}}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(doc))
    assert bench.recorded_traffic("output", "480p") == 123
    (csrc / "k.cu").write_text("int y, z;\n")
    assert bench.recorded_traffic("output", "480p") is None


@pytest.mark.parametrize("ranks,units,ms,want", [(1, 1000, 1.0, 1e6), (4, 1000, 2.0, 2e6)])
def test_job_throughput_counts_every_rank(ranks, units, ms, want):
    assert bench.job_throughput(units, ranks, ms) == pytest.approx(want)


@pytest.mark.parametrize("name,mb", [("480p", 587.1), ("720p", 1354.8), ("wide", 2147.0), ("decode", 83.9)])
def test_algorithmic_bytes_per_step_match_the_workload_table(name, mb):
    """The roofline numerator: Q, K, V read once and O written once per token*head, summed
    over the launches that move per-token bytes (for decode: one block of 3 frames)."""
    import block_causal_linear_rope_b200 as blin
    w = workloads.CONFIGS[name]
    tokens = w.F * w.HW if name == "decode" else w.N
    elem = 2 if w.dtype == "bf16" else 4
    units = w.B * w.H * tokens
    total = sum(blin.KERNEL_BYTES_PER_UNIT[k] * w.d * elem * units for k in blin.KERNEL_BYTES_PER_UNIT)
    assert total == units * 4 * w.d * elem
    assert round(total / 1e6, 1) == mb
