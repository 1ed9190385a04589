"""The measurement arithmetic of bench.py, without a GPU: the algorithmic byte counts the
roofline fractions divide by (checked against the per-token and per-step figures they are
built from), and the lookup that attaches a recorded DRAM capture to a kernel only while
that kernel's code is unchanged."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_prefill_bytes_per_token_and_state():
    # per token at Hk = Hv = 48, d = 128: q, k, v bf16 (3 x 48 x 128 x 2 = 36,864), a, b bf16
    # (2 x 48 x 2 = 192), o fp32 (48 x 128 x 4 = 24,576): 61,632 B; the final state fp32
    # 48 x 128 x 128 x 4 = 3,145,728 B
    per_token = 36864 + 192 + 24576
    assert per_token == 61632
    assert bench.prefill_alg_bytes(1, 8192, 48, 48, 128, 128) == 8192 * per_token + 3145728
    assert bench.prefill_alg_bytes(1, 8192, 48, 48, 128, 128) == 508035072
    # grouped keys (Hk = 16 shared by Hv = 48): q, k shrink to a third
    per_token_gqa = 2 * 16 * 128 * 2 + 48 * 128 * 2 + 2 * 48 * 2 + 48 * 128 * 4
    assert per_token_gqa == 45248
    assert bench.prefill_alg_bytes(1, 1000, 16, 48, 128, 128) == 1000 * 45248 + 3145728


def test_decode_bytes_per_step():
    # B = 64, H = 48, d = 128: the fp32 state read and written (2 x 64 x 48 x 64 KiB) plus
    # one token's inputs and fp32 output per (sequence, head)
    state = 2 * 64 * 48 * 128 * 128 * 4
    assert bench.decode_state_bytes(64, 48, 128, 128) == state
    inputs = 64 * (2 * 48 * 128 * 2 + 48 * 128 * 2 + 2 * 48 * 2 + 48 * 128 * 4)
    assert bench.decode_alg_bytes(64, 48, 48, 128, 128) == state + inputs == 406597632


def test_source_hash_ignores_comments_and_layout_only():
    code = "int f(int x) {\n    return x + 1;  // one more\n}\n/* block */\n"
    h = bench.kernel_source_hash("x.cu", code)
    assert bench.kernel_source_hash("x.cu", "int f(int x) { return x + 1; }") == h
    assert bench.kernel_source_hash("x.cu", code.replace("// one more", "// comment")) == h
    assert bench.kernel_source_hash("x.cu", code.replace("x + 1", "x + 2")) != h


def test_recorded_traffic_follows_the_code(tmp_path, monkeypatch):
    csrc = tmp_path / "gated_delta_rule_145_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_text("__global__ void k() {}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash("k.cu")
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# file hash bytes how\n" + f"k.cu {h} 12345 a capture\n")
    assert bench.recorded_traffic("k.cu") == 12345.0
    src.write_text("__global__ void k() {}  // a comment does not change the code\n")
    assert bench.recorded_traffic("k.cu") == 12345.0
    src.write_text("__global__ void k() { int x = 0; }\n")
    assert bench.recorded_traffic("k.cu") is None
    assert bench.recorded_traffic("other.cu") is None
