"""Host-side logic of bench.py that needs no GPU: the comment-insensitive kernel source
hash and the rule that a committed DRAM-traffic figure is reported only while the kernel's
sources still hash to the value recorded with it."""
import json
import os

import bench


def test_code_only_ignores_comments_and_blank_space():
    a = "int x = 1; // one\n/* block\ncomment */\n\n   float  y = 2;\n"
    b = "int x = 1;\nfloat y = 2;   // two\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(b.replace("2", "3"))


def test_committed_traffic_is_reported_while_the_hash_matches(monkeypatch):
    """Each committed figure names its capture summary, and is returned exactly when the
    sources hash to the recorded value."""
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        d = json.load(f)
    for key in bench.KERNEL_SOURCES:
        assert key in d, key
        assert os.path.exists(os.path.join(bench.ROOT, d[key]["capture"])), d[key]["capture"]
        monkeypatch.setattr(bench, "kernel_source_hash", lambda k, h=d[key]["source_hash"]: h)
        assert bench.committed_traffic(key) == float(d[key]["bytes_per_launch"])


def test_committed_traffic_is_null_for_other_sources(monkeypatch):
    monkeypatch.setattr(bench, "kernel_source_hash", lambda key: "0000000000000000")
    for key in bench.KERNEL_SOURCES:
        assert bench.committed_traffic(key) is None
