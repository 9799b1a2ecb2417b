"""Host-side pieces of bench.py that need no GPU: the byte model, the L2
notes, the traffic lookup keyed by kernel sources, and the peaks."""
import json

import torch

import bench
from block_sparse_attention_decode_b200 import synth


def test_l2_notes_follow_the_cache_size():
    big, big_e2e = bench.l2_notes(5_400_000_000)
    assert "5.4 GB > 126 MB L2" in big and big_e2e == "no L2 flush (inputs > L2)"
    small, small_e2e = bench.l2_notes(44_000_000)
    assert "fit in the 126 MB L2" in small and "stay there" in small_e2e


def test_algorithmic_bytes_counts_union_of_selected_visible_tokens():
    w = synth.make_workload("bytes", 2, [300, 129], 2, paged=True, seed=7)
    sel = torch.full((2, 2, 4, 16), -1, dtype=torch.int32)
    sel[0, 0, 0, :2] = torch.tensor([0, 2])      # sequence 0, group 0: blocks {0, 2} over
    sel[0, 1, 0, :1] = torch.tensor([2])         # its two tokens (block 2 holds 44 tokens)
    sel[1, 0, 3, :1] = torch.tensor([1])         # sequence 1, group 3: block 1 (1 token)
    b = bench.algorithmic_bytes(w, sel)
    assert b["index_scan"] == (300 + 129) * 72
    assert b["kv_tokens"] == 128 + 44 + 1
    assert b["kv_selected"] == (128 + 44 + 1) * 144
    assert b["queries"] == 2 * 2 * (64 * 128 + 4 * 128)
    assert b["output"] == 2 * 2 * 64 * 128 * 2
    assert b["total"] == b["index_scan"] + b["kv_selected"] + b["queries"] + b["output"]


def test_traffic_is_read_only_for_unchanged_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "probe_kernel", ["k.cu"])
    sha = bench.source_sha(["k.cu"])
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"probe_kernel": {"workload": "wl", "bytes_per_launch": 1234, "source_sha": sha}}))
    assert bench.dram_traffic("probe_kernel", "wl") == 1234
    assert bench.dram_traffic("probe_kernel", "other_workload") is None
    src.write_text("kernel v2")                   # the kernel changed since the capture
    assert bench.dram_traffic("probe_kernel", "wl") is None


def test_measured_peaks_come_from_the_file(tmp_path, monkeypatch):
    """The HBM peak is the driver-written measurement when the file exists,
    else the stated fallback, labelled as such."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peak, src = bench.measured_peaks()
    assert src == "fallback" and peak == bench.FALLBACK_HBM_GBS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6540.2}))
    peak, src = bench.measured_peaks()
    assert src == "measured" and peak == 6540.2


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the oracle on the host cores) prints one JSON
    line with the contract's keys; a small workload keeps it quick."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "ctx4k_b1_t1", "--steps", "1", "--warmup", "0"],
                       cwd=bench.ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["warmup"] >= 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
