"""Host-side arithmetic of bench.py on CPU: the roofline's algorithmic work
and the gate that reports DRAM traffic only for the profiled kernel source.

The byte and flop counts are checked against values worked out by hand from
their definitions (per token: q, k in bf16, v in and o out in bf16, g and
beta in f32; per sequence: h0 read and hT written in f32; the chunk form's
flops per token and value head), so a dropped term or a wrong factor fails.
"""
import hashlib
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_prefill_bytes_of_the_4576_token_workload():
    # 4576 tokens x (2*16*128*2 + 2*48*128*2 + 2*48*4) B + 1 x 2*48*128*128*4 B
    per_token = 8192 + 24576 + 384
    per_seq = 6291456
    assert bench.prefill_alg_bytes(4576, 1, 16, 48, 128, 128) == 4576 * per_token + per_seq
    assert bench.prefill_alg_bytes(4576, 1, 16, 48, 128, 128) == 157995008


def test_prefill_bytes_scale_with_sequences_and_heads():
    one = bench.prefill_alg_bytes(100, 1, 2, 4, 64, 64)
    # a second sequence adds only its own h0/hT; doubling tokens adds only token bytes
    assert bench.prefill_alg_bytes(100, 2, 2, 4, 64, 64) - one == 8 * 4 * 64 * 64
    assert bench.prefill_alg_bytes(200, 1, 2, 4, 64, 64) - one == 100 * (4 * 2 * 64 + 4 * 4 * 64 + 8 * 4)


def test_prefill_flops_of_the_4576_token_workload():
    # per (token, v-head): (C-1) d_k  +  2C (d_k + d_v)  +  6 d_k d_v  with C = 64
    per = 63 * 128 + 2 * 64 * 256 + 6 * 128 * 128
    assert per == 139136
    assert bench.prefill_alg_flops(4576, 48, 128, 128) == 4576 * 48 * per == 30560944128


def _fake_tree(tmp_path, src_bytes, traffic_sha):
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "linear_attention_ssm_gdn_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gdn_prefill.cu").write_bytes(src_bytes)
    (tmp_path / "profiles" / "prefill_dram_traffic.txt").write_text(
        "# a comment line = with an equals sign\n"
        "bytes_per_launch_full_workload = 123456\n"
        f"source_sha256 = {traffic_sha}\n")


def test_profiled_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    src = b"// kernel source\n"
    _fake_tree(tmp_path, src, hashlib.sha256(src).hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic() == 123456.0
    # the kernel changes: the counters no longer describe it
    (tmp_path / "linear_attention_ssm_gdn_b200" / "csrc" / "gdn_prefill.cu").write_bytes(src + b" ")
    assert bench.profiled_traffic() is None


def test_profiled_traffic_missing_file_is_none(tmp_path, monkeypatch):
    src = b"x"
    _fake_tree(tmp_path, src, hashlib.sha256(src).hexdigest())
    shutil.rmtree(tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic() is None


def test_committed_traffic_file_parses():
    """The committed summary has both keys the bench reads (whether its hash
    matches the current source is the bench's business, not this test's)."""
    vals = {}
    with open(os.path.join(ROOT, "profiles", "prefill_dram_traffic.txt")) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                vals[k.strip()] = v.split()[0]
    assert int(vals["bytes_per_launch_full_workload"]) > 0
    assert len(vals["source_sha256"]) == 64
