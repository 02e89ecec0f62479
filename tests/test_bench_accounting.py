"""Host logic of bench.py's roofline accounting (CPU): the visible (query, key) pairs the
attention's FLOPs are counted on, the algorithmic bytes of the decode launches, and the
rule that a committed DRAM-traffic record is used only while the kernel's sources match
the ones the counters were taken on."""
import json
import os

import pytest

import bench
import synth


def _brute_pairs(Tp, m, W):
    n = 0
    for i in range(Tp):
        for j in range(i + 1):
            if W <= 0 or j < m or i - j < W:
                n += 1
    return n


@pytest.mark.parametrize("Tp,m,W", [(1, 0, 0), (9, 0, 0), (17, 3, 4), (40, 8, 16), (33, 0, 1), (12, 12, 5)])
def test_visible_pairs_match_brute_force(Tp, m, W):
    """The count the attention's FLOPs are taken on: key j visible to query i iff j <= i
    and (j < m or i - j < W), W <= 0 global."""
    assert bench.visible_pairs(Tp, m, W) == _brute_pairs(Tp, m, W)


def test_visible_pairs_closed_forms():
    """Global causal: Tp (Tp + 1) / 2. A window of W with no meta rows: row i sees
    min(i + 1, W) keys, so W (W + 1) / 2 over the first W rows and W for each later one."""
    assert bench.visible_pairs(100, 0, 0) == 100 * 101 // 2
    Tp, W = 100, 8
    assert bench.visible_pairs(Tp, 0, W) == W * (W + 1) // 2 + (Tp - W) * W
    # window 1 and no meta: only the diagonal
    assert bench.visible_pairs(37, 0, 1) == 37


def test_decode_work_of_the_combined_launch():
    """The combined attention + SSM decode launch is counted as the sum of its parts; the
    attention's bytes are K and V of every cache slot of every (sequence, KV head)."""
    cfg = synth.workload("hymba15_decode_pair_b64_p4096")["cfg"]
    B, cap = 64, cfg.n_meta + cfg.window
    w = bench.decode_work(cfg, B, cap)
    assert w["attn_decode"] == ("hbm", B * cfg.n_kv_heads * cap * (cfg.head_dim + cfg.v_head_dim) * 2.0)
    assert w["attn_ssm_decode"][1] == w["attn_decode"][1] + w["ssm_decode"][1]
    assert all(bound == "hbm" for bound, _ in w.values())
    # the 1.5B pair: 141.6 MB of K/V per attention launch
    assert abs(w["attn_decode"][1] - 141557760.0) < 1.0


def test_traffic_record_is_dropped_when_a_source_changes(tmp_path, monkeypatch):
    """A record keyed on a source file and headers stays valid while their bytes match
    and reads as None once any of them changes."""
    root = tmp_path
    for rel in ("k.cu", "h.cuh"):
        (root / rel).write_text("// " + rel + "\n")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    monkeypatch.setattr(bench, "TRAFFIC_HEADERS", ("h.cuh",))
    bench.record_traffic("kern", "wl", "k.cu", 12345, "counters", "summary.md")
    assert bench.kernel_traffic("kern", "wl") == 12345
    assert bench.kernel_traffic("kern", "other_workload") is None
    (root / "h.cuh").write_text("// changed\n")
    assert bench.kernel_traffic("kern", "wl") is None
    rec = json.load(open(root / "profiles" / "dram_traffic.json"))["kern"]
    assert rec["sources"] == ["k.cu", "h.cuh"] and rec["bytes_per_launch"] == 12345


def test_committed_traffic_record_names_its_sources():
    """The committed record lists existing files and the summary it came from."""
    recs = json.load(open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")))
    for name, rec in recs.items():
        for rel in rec["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, rel)), (name, rel)
        assert os.path.exists(os.path.join(bench.ROOT, rec["summary"])), (name, rec["summary"])
        assert rec["bytes_per_launch"] > 0
