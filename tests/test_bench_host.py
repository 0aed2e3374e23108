"""bench.py's host-side bookkeeping, on CPU: the step it times (the decode
pass's launches and their weight bytes), the workload name, and the key under
which profiler-recorded DRAM traffic is matched to kernel code."""
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import oracle  # noqa: E402


def test_qwen3_8b_step_is_the_decode_pass():
    shapes = bench.step_shapes("qwen3-8b", 36)
    assert len(shapes) == 36 * 4 + 1
    assert shapes[:4] == [("L0.qkv", 6144, 4096), ("L0.o", 4096, 4096), ("L0.gate_up", 24576, 4096),
                          ("L0.down", 4096, 12288)]
    assert shapes[-1] == ("lm_head", 151936, 4096)
    # weight bytes of one binary pass: 36 layers of 24.1 M weights + the head, at 1.125 bits per weight
    wbytes = sum(oracle.codes_bytes("q1g128", n, k) + oracle.scales_bytes(n, k) for _, n, k in shapes)
    assert wbytes == 1064263680


def test_27b_step_shapes():
    shapes = bench.step_shapes("27b", 64)
    assert len(shapes) == 64 * 4 + 1
    assert shapes[:4] == [("L0.qkv", 8192, 5120), ("L0.o", 5120, 6144), ("L0.gate_up", 34816, 5120),
                          ("L0.down", 5120, 17408)]
    assert shapes[-1] == ("lm_head", 248320, 5120)
    name = bench.workload_name("27b", "t2g128", 1, 64)
    assert "64 x (q|k|v 8192x5120" in name and "LM head 248320x5120" in name


def test_traffic_key_ignores_comments_not_code(tmp_path, monkeypatch):
    src = os.path.join(ROOT, "ternary_g128_weight_b200", "csrc")
    fake = tmp_path / "ternary_g128_weight_b200" / "csrc"
    fake.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(src, name), fake / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    f = fake / "bq_gemv_rows.cu"
    f.write_text(f.read_text() + "\n// a comment\n/* and a block\n   comment */\n")
    assert bench.kernel_source_hash() == h0
    f.write_text(f.read_text().replace("kMaxSlots = 8", "kMaxSlots = 7", 1))
    assert bench.kernel_source_hash() != h0


def test_recorded_traffic_matches_only_its_workload_and_code():
    rec = bench.recorded_traffic("qwen3-8b", "q1g128", 1, 36)
    if rec is None:
        pytest.skip("no record for the current kernel code")
    assert rec > 1064263680                                    # at least the weight bytes
    assert bench.recorded_traffic("qwen3-8b", "t2g128", 1, 36) is None
    assert bench.recorded_traffic("qwen3-8b", "q1g128", 8, 36) is None
