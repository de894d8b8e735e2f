"""bench.py's bookkeeping on CPU: the ncu traffic record applies only to the
kernel source it was taken on and to its workload; peaks fall back when the
measured file is absent; the algorithmic FLOP count equals the visible-pair
count the oracle pins."""
from __future__ import annotations

import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_traffic_record_needs_matching_kernel_and_workload(tmp_path, monkeypatch):
    import bench

    rec = tmp_path / "traffic.txt"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    rec.write_text(f"# comment\nkernel_sha256_16: {bench.kernel_hash()}\nworkload_id: 3\ndram_bytes_per_launch: 12345\n")
    assert bench.recorded_traffic(3) == 12345.0
    assert bench.recorded_traffic(4) is None              # another workload
    rec.write_text("kernel_sha256_16: 0000000000000000\nworkload_id: 3\ndram_bytes_per_launch: 12345\n")
    assert bench.recorded_traffic(3) is None              # taken on another kernel source
    rec.unlink()
    assert bench.recorded_traffic(3) is None              # no record


def test_kernel_hash_tracks_the_attention_sources():
    import bench

    h = bench.kernel_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    assert all(os.path.exists(os.path.join(ROOT, f)) for f in bench.KERNEL_SOURCES)


def test_step_flops_is_four_d_h_per_visible_pair():
    """The bench's FLOP count per layer step is 4 d H per visible (query, key)
    pair, the pair counts the golden file holds for every step workload."""
    import bench
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS

    with open(os.path.join(ROOT, "tests", "golden", "visible_pairs.json")) as f:
        golden = json.load(f)
    for wid in (1, 2, 3, 4):
        wl = WORKLOADS[wid]
        assert bench.step_flops(wl) == pytest.approx(4.0 * wl.d * wl.H * golden[str(wid)]["step_pairs"])


def test_peaks_fall_back_without_the_measured_file(monkeypatch, tmp_path):
    import bench

    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks


def test_verify_flops_match_the_golden_pair_count():
    import bench
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS

    with open(os.path.join(ROOT, "tests", "golden", "visible_pairs.json")) as f:
        golden = json.load(f)
    wl = WORKLOADS[5]
    assert bench.verify_flops(wl) == pytest.approx(4.0 * wl.d * wl.H * golden["2"]["verify_pairs"])


def test_insert_bytes_follow_the_definition():
    """Algorithmic insert bytes per layer step: read the step's K and V and
    write them into the ring, 4 N_new Hkv d bytes of bf16 (7,995,392 at the
    driving shape); the kernel's own traffic adds the fp16 operand rows."""
    import bench
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS

    wl = WORKLOADS[3]
    assert bench.insert_algorithmic_bytes(wl) == 4 * wl.step_tokens * wl.Hkv * wl.d * 2 == 7995392
    impl = bench.insert_implementation_bytes(wl)
    assert impl >= 1.75 * bench.insert_algorithmic_bytes(wl)


def test_frame_flops_count_the_frame_pairs():
    """Encoder attention: every token of a view's frame sees the whole frame,
    so a call does 4 d H n^2 per view; checked against a brute-force count of
    the (query, key) pairs of the oracle's per-view mask."""
    import numpy as np

    import bench
    from streaming_kv_cache_stream_b200.inputs import Workload

    wl = Workload("f", 3, 2, 5, 0, H=4, Hkv=2, d=8)
    heads = dict(H=4, Hkv=2, d=8)
    view = np.repeat(np.arange(wl.views), wl.tok_per_frame)
    pairs = int((view[:, None] == view[None, :]).sum())
    assert bench.frame_flops(wl, heads) == 4.0 * heads["d"] * heads["H"] * pairs
