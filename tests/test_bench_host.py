"""Host-side logic of bench.py, on CPU: the algorithmic byte count the
roofline divides by, and the reference arm (the CPU oracle timed on the
host cores), which must print the contract's JSON line without a GPU."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_tiny_prefill_by_hand():
    """2 requests of 5 and 3 tokens from position 0, C = 8, W = 4, fp32:
    x 8*8*4 + (insert + out) 2*8*8*4 + no history + weight 8*4*4 + 24 B of
    metadata per token = 1088 bytes."""
    wl = workloads.tiny_prefill_f32()
    assert bench.algorithmic_bytes(wl) == 256 + 512 + 128 + 24 * 8


def test_algorithmic_bytes_counts_history_rows_and_block_entries():
    """One request, 2 new tokens after 9 cached ones, N = 4, W = 4: three
    history rows (positions 6, 7, 8) over two logical blocks (1 and 2)."""
    wl = workloads.build("h", dtype="bf16", H=1, D=8, ws=8, off_s=0, W=4, N=4, hist=[9],
                         new=[2], act=None, residual=False, seed=3)
    C, e = 8, 2
    expect = 2 * C * e + 2 * 2 * C * e + 3 * C * e + C * 4 * e + 24 * 2 + 4 * 2
    assert bench.algorithmic_bytes(wl) == expect


def test_algorithmic_bytes_skips_pad_rows_for_writes():
    wl = workloads.spec_decode_bf16()
    live = int((wl.slot_mapping != -1).sum())
    assert live == wl.T - int(0.1 * wl.T)
    b = bench.algorithmic_bytes(wl)
    # x is read for every row, inserts and outputs only for live rows
    assert b > wl.T * wl.C * 2 + 2 * live * wl.C * 2
    assert b < wl.T * wl.C * 2 + 2 * wl.T * wl.C * 2 + 3 * wl.R * wl.C * 2 + (1 << 20)


@pytest.mark.timeout(600)
def test_reference_arm_prints_the_contract_line_on_cpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=540)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["steps"] == 1 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("decode_bf16")
    assert np.isfinite(line["ms_per_step"])


class _Sets:
    def __init__(self, alg_bytes):
        self.alg_bytes = alg_bytes
        self.sets = [None] * len(alg_bytes)


def test_l2_statement_for_fewer_steps_than_sets():
    """K timed steps on K distinct sets: the statement says the region is
    preceded by a flush and counts only the K sets' bytes."""
    s = bench.l2_statement(_Sets([3_000_000] * 96), 20)
    assert "flushed" in s and "none repeats" in s and "60 MB" in s


def test_l2_statement_names_the_untimed_lead_steps():
    """Short runs time K steps after LEAD_STEPS untimed ones in the same
    graph; the statement says those read other sets."""
    s = bench.l2_statement(_Sets([3_000_000] * 96), 20)
    assert f"the {bench.LEAD_STEPS} untimed steps ahead of them read other sets" in s
    assert "untimed" not in bench.l2_statement(_Sets([3_000_000] * 96), 95)


def test_config_timing_says_which_form_ran():
    short = bench.config_block(1, "l2", 20)["timing"]
    assert "untimed steps" in short and "graph nodes" in short
    long = bench.config_block(1, "l2", bench.EVENT_GRAPH_MAX_STEPS + 1)["timing"]
    assert "rotation" in long
    assert "timing" not in bench.config_block(1, "l2")


def test_l2_statement_for_rotations():
    big = bench.l2_statement(_Sets([3_000_000] * 96), 500)
    assert "288 MB > 126 MB L2" in big
    small = bench.l2_statement(_Sets([1_000_000] * 8), 500)
    assert "NOT above the 126 MB L2" in small


def test_profiled_traffic_reads_the_json_record(tmp_path, monkeypatch):
    """The roofline's traffic comes from profiles/fused_sconv_<workload>.json
    and only while its source hash matches the kernel sources."""
    (tmp_path / "profiles").mkdir()
    rec = {"traffic_bytes_per_launch": 1234, "kernel_source_sha256_16": "abc"}
    (tmp_path / "profiles" / "fused_sconv_w.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.profiled_traffic("w") == 1234
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "changed")
    assert bench.profiled_traffic("w") is None
    assert bench.profiled_traffic("missing") is None


def test_algorithmic_bytes_taps_by_hand():
    """One request, 2 new tokens after 9 cached ones, W = 4, C = 8, bf16: x,
    insert and out of both tokens, three history rows, the weights, and per
    token the slot (8 B) and a table row of three 8-byte entries."""
    wl = workloads.build("h", dtype="bf16", H=1, D=8, ws=8, off_s=0, W=4, N=4, hist=[9],
                         new=[2], act=None, residual=False, seed=3)
    C, e = 8, 2
    expect = 2 * C * e + 2 * 2 * C * e + 3 * C * e + C * 4 * e + (8 + 24) * 2
    assert bench.algorithmic_bytes_taps(wl) == expect


def test_algorithmic_bytes_resolve_by_hand():
    """One request, 2 new tokens after 9 cached ones, W = 4, N = 4: per
    token 16 B read (position, slot) and 8 + 24 B written (seq_idx,
    query_start, table row); query_start_loc 2 entries; the three history
    rows (positions 6, 7, 8) lie in two logical blocks."""
    wl = workloads.build("h", dtype="bf16", H=1, D=8, ws=8, off_s=0, W=4, N=4, hist=[9],
                         new=[2], act=None, residual=False, seed=3)
    assert bench.algorithmic_bytes_resolve(wl) == 16 * 2 + 4 * 2 + 4 * 2 + 32 * 2
