"""The committed profile summaries: text only, every ncu command leaves the clocks alone, and the
DRAM traffic record is self-consistent (each weight byte read once per call)."""
import json
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def _files():
    return sorted(os.listdir(PROFILES))


def test_profiles_hold_text_only():
    for f in _files():
        assert f.endswith((".md", ".txt", ".json")), f
        assert os.path.getsize(os.path.join(PROFILES, f)) < 64 * 1024, f


def test_every_ncu_command_leaves_clocks_alone():
    n = 0
    for f in _files():
        if not f.endswith(".md"):
            continue
        text = open(os.path.join(PROFILES, f)).read().replace("\\\n", " ")
        for line in text.splitlines():
            if line.startswith("#"):
                continue  # the title names the capture, not a command
            if re.search(r"(^|\s|`)ncu\s+--", line):
                n += 1
                assert "--clock-control none" in line, (f, line)
    assert n >= len([f for f in _files() if f.endswith(".md")])


def test_traffic_record_is_consistent():
    t = json.load(open(os.path.join(PROFILES, "traffic.json")))
    for rec in (t, t["b8"]):
        assert rec["bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
        # weight + x is at most the algorithmic bytes (which add y); reads stay within 0.2% of
        # them: no re-reads of the weights
        assert 0.99 * rec["algorithmic_bytes"] <= rec["dram_bytes_read"] <= 1.002 * rec["algorithmic_bytes"]
    assert re.fullmatch(r"[0-9a-f]{16}", t["rows_kernel_hash"])
    assert re.fullmatch(r"[0-9a-f]{16}", t["b8"]["mma_kernel_hash"])
    # the headline record is the Q4_K 17408 x 5120 call at B = 1: W + x + y bytes
    N, K = 17408, 5120
    assert t["algorithmic_bytes"] == N * K // 256 * 144 + 2 * K + 4 * N
    assert t["b8"]["algorithmic_bytes"] == N * K // 256 * 144 + 2 * K * 8 + 4 * N * 8
