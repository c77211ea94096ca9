"""Host-side pieces of bench.py that need no GPU: the clock-sample summary,
the workload description for one and several ranks, the algorithmic counts
behind the roofline numbers, and the rule that a recorded DRAM traffic figure
is dropped once the kernel's sources change."""
import json

import numpy as np
import pytest

import bench
import synth


def test_clock_summary_reports_median_and_reasons():
    rows = [
        "2026/12/03 05:40:00.100, 0, 1965, 1965, 650.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 05:40:00.150, 0, 1965, 1965, 700.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 05:40:00.200, 0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "2026/12/03 05:40:00.250, 0, [N/A], 1965, 1.0, x, Not Active, Not Active, Not Active, Not Active",
    ]
    r = bench.Clocks.parse(rows)
    assert r["samples"] == 3
    assert r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    assert bench.Clocks.parse([])["sm_mhz"] is None


def test_clock_summary_windows_by_timestamp():
    """Only samples inside the clock window count; those inside the timed
    region are counted apart."""
    rows = [f"2026/12/03 05:40:0{i}.000, 0, {1900 + i}, 1965, 700.0, 0x0, Not Active, Not Active, "
            f"Not Active, Not Active" for i in range(6)]
    t = [bench.Clocks._stamp(f"2026/12/03 05:40:0{i}.000") for i in range(6)]
    r = bench.Clocks.parse(rows, window=(t[1], t[4]), timed=(t[1], t[2]))
    assert r["samples"] == 4 and r["samples_in_timed_region"] == 2
    assert r["sm_mhz"] == 1902.5


def test_workload_config_single_and_multi_rank():
    w = synth.make("tiny")
    one = bench.workload_config(w, 1)
    four = bench.workload_config(w, 4)
    assert one["parallelism"] == "single" and one["global_batch"] == w.B
    assert four["parallelism"] == "dp4" and four["global_batch"] == 4 * w.B
    assert "seeds 1003..1006" in four["workload"]


def test_algorithmic_counts_match_a_direct_count():
    w = synth.make("small")
    sel, win = bench.algorithmic_counts(w)
    # selected slots: the causal and document rules applied to idx, directly
    P = w.S // w.cr
    t = np.arange(w.S)[None, :, None]
    j = w.idx
    ok = (j >= 0) & (j < P) & ((j + 1) * w.cr - 1 <= t)
    if w.doc_start is not None:
        d0 = np.clip(w.doc_start, 0, np.arange(w.S)[None, :])[:, :, None]
        ok &= j * w.cr >= d0
    assert sel == int(ok.sum())
    # window keys: min(W, t - d0 + 1) per token
    d0 = np.zeros((w.B, w.S), dtype=np.int64) if w.doc_start is None else \
        np.clip(w.doc_start, 0, np.arange(w.S)[None, :])
    tt = np.arange(w.S)[None, :]
    assert win == int(np.minimum(w.W, tt - np.maximum(d0, tt - w.W + 1) + 1).sum())


def test_traffic_record_is_dropped_when_sources_change(tmp_path, monkeypatch):
    root = tmp_path
    csrc = root / "sparse_attention_indexer_window_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    (csrc / "k.cu").write_text("kernel v1")
    import hashlib
    h = hashlib.sha256(b"kernel v1").hexdigest()[:16]
    (root / "profiles" / "traffic.json").write_text(json.dumps(
        {"k.cu": {"sources": ["k.cu"], "src_sha256_16": h, "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.traffic_record("k.cu") == 123
    (csrc / "k.cu").write_text("kernel v2")
    assert bench.traffic_record("k.cu") is None
    assert bench.traffic_record("other.cu") is None


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("small", {}), ("packed", {"B": 2, "S": 256, "K": 16})])
def test_candidate_blocks_match_a_direct_count(name, kw):
    """The selection line's read bytes count every (token, block) pair with
    the block wholly at or before the token and inside its document."""
    w = synth.make(name, **kw)
    P = w.S // w.cr
    n = 0
    for b in range(w.B):
        for t in range(w.S):
            d0 = 0 if w.doc_start is None else min(max(int(w.doc_start[b, t]), 0), t)
            n += sum(1 for j in range(P) if (j + 1) * w.cr - 1 <= t and j * w.cr >= d0)
    assert bench.candidate_blocks(w) == n
