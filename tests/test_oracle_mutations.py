"""The pins must catch plausible mistakes in the oracle (CPU only).

Each mutant is a copy of the oracle's C source with one plausible slip
planted (a reversed or shifted tap, a wrong comparison, a swapped index, a
dropped term, a transposed write).  It is compiled on the CPU, and the pin
suites (tests/test_oracle_pins.py, tests/test_oracle_pins_dense.py and
tests/test_oracle_pins_taps.py) are run against it in a child process; they must fail for every mutant.  Every planted slip keeps all memory
accesses inside their buffers, so a mutant fails by assertion, not by crash.
"""
from __future__ import annotations

import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sconv_oracle.c")

# (name, text to replace, replacement); the first occurrence is replaced.
MUTANTS = [
    ("tap_orientation_reversed",
     "#define TAP_POSITION(pos, W, k) ((pos) - ((W) - 1) + (k))",
     "#define TAP_POSITION(pos, W, k) ((pos) - (k))"),
    ("tap_window_shifted",
     "#define TAP_POSITION(pos, W, k) ((pos) - ((W) - 1) + (k))",
     "#define TAP_POSITION(pos, W, k) ((pos) - (W) + (k))"),
    ("same_forward_strict",
     "            if (row >= q0) {",
     "            if (row > q0) {"),
    ("logical_block_mod",
     "                int64_t logical = src / N;",
     "                int64_t logical = (src % N) % max_blocks;"),
    ("block_offset_div",
     "                                  (src % N) * cache_strides[2] +",
     "                                  ((src / N) % N) * cache_strides[2] +"),
    ("read_lane_ignores_off_s",
     "                                  (off_s + j) * cache_strides[3];",
     "                                  (j) * cache_strides[3];"),
    ("read_head_dropped",
     "                                  h * cache_strides[1] +\n                                  (src % N)",
     "                                  0 * cache_strides[1] +\n                                  (src % N)"),
    ("insert_offset_div",
     "(slot % N) * cache_strides[2] + (off_s + j) * cache_strides[3];",
     "((slot / N) % N) * cache_strides[2] + (off_s + j) * cache_strides[3];"),
    ("insert_lane_ignores_off_s",
     "(slot % N) * cache_strides[2] + (off_s + j) * cache_strides[3];",
     "(slot % N) * cache_strides[2] + (j) * cache_strides[3];"),
    ("weight_taps_reversed",
     "load_value(weight, dtype, c * w_stride_c + k * w_stride_k)",
     "load_value(weight, dtype, c * w_stride_c + (W - 1 - k) * w_stride_k)"),
    ("epilogue_residual_inside_act",
     "(((silu) ? (conv) / (1.0 + exp(-(conv))) : (conv)) + ((resid) ? (xv) : 0.0))",
     "(((silu) ? ((conv) + ((resid) ? (xv) : 0.0)) / (1.0 + exp(-((conv) + ((resid) ? (xv) : 0.0)))) : (conv) + ((resid) ? (xv) : 0.0)))"),
    ("residual_dropped",
     "+ ((resid) ? (xv) : 0.0))",
     "+ 0.0)"),
    ("silu_sign",
     "(conv) / (1.0 + exp(-(conv)))",
     "(conv) / (1.0 + exp((conv)))"),
    ("pad_not_skipped",
     "        if (slot == -1) continue; /* PAD",
     "        if (slot == -2) continue; /* PAD"),
    ("metadata_strict",
     "            if (query_start_loc[r] <= t) found = r;",
     "            if (query_start_loc[r] < t) found = r;"),
    ("extract_window_shifted",
     "int64_t p = (int64_t)abs_positions[i] - d_conv + k;",
     "int64_t p = (int64_t)abs_positions[i] - d_conv + k + 1;"),
    ("extract_not_transposed",
     "int64_t dst = i * out_slot_stride + c * d_conv + k;",
     "int64_t dst = i * out_slot_stride + k * conv_dim + c;"),
    ("ssm_row_reversed",
     "            copy_element(out, i * out_row_stride + e, states, row * states_row_stride + e,",
     "            copy_element(out, i * out_row_stride + e, states, row * states_row_stride + (state_flat - 1 - e),"),
    ("ssm_ignores_bad_index_check",
     "        if (row < 0 || row >= num_chunks) {",
     "        if (row < 0 || row >= num_chunks || row == 0) {"),
    ("paged_offset_shifted",
     "                                  (p % N) * cache_strides[2] + (off_s + j) * cache_strides[3];\n                    copy_element(out, dst, cache, src, dtype);",
     "                                  ((p + 1) % N) * cache_strides[2] + (off_s + j) * cache_strides[3];\n                    copy_element(out, dst, cache, src, dtype);"),
    ("paged_zero_at_position_0",
     "                if (p < 0) {\n                    memset",
     "                if (p < 1) {\n                    memset"),
    ("extract_ignores_real_count",
     "    for (int64_t i = 0; i < real_count; ++i) {",
     "    for (int64_t i = 0; i < max_count; ++i) {"),
    ("dense_bias_dropped",
     "#define BIASED(conv, b) ((conv) + (b))",
     "#define BIASED(conv, b) ((conv) + 0.0 * (b))"),
    ("dense_bias_after_activation",
     "out_ref[(q0 + t) * dim + c] = EPILOGUE(BIASED(acc, bv), 0.0, silu, 0);",
     "out_ref[(q0 + t) * dim + c] = EPILOGUE(acc, 0.0, silu, 0) + bv;"),
    ("dense_taps_from_oldest_entries",
     "int64_t i = Lh + TAP_POSITION(t, W, k); /* entry of e */",
     "int64_t i = (W - 1) + TAP_POSITION(t, W, k); /* entry of e */"),
    ("dense_has_init_ignored",
     "int from_state = states_in && has_init && has_init[b];",
     "int from_state = states_in != NULL;"),
    ("dense_line_not_shifted",
     "            int64_t j = n + i;",
     "            int64_t j = i;"),
    ("dense_zero_line_not_zeroed",
     "memset((char *)states_out + dst * (int64_t)elem_bytes(dtype), 0,",
     "memset((char *)states_out + dst * (int64_t)elem_bytes(dtype), 0x3f,"),
    ("dense_pad_not_skipped",
     "if (cache_indices && line == pad_slot_id) continue; /* padded entry */",
     "if (cache_indices && line == pad_slot_id - 1) continue; /* padded entry */"),
    ("update_ring_taps_shifted",
     "                        i = ((p % L) + L) % L;",
     "                        i = (((p + 1) % L) + L) % L;"),
    ("update_ring_store_shifted",
     "                int64_t i = ((s % L) + L) % L;",
     "                int64_t i = (((s + 1) % L) + L) % L;"),
    ("update_line_not_shifted",
     "                                 states_in, STATE_INDEX(line, c, i + 1, s_line, s_c, s_k),",
     "                                 states_in, STATE_INDEX(line, c, i, s_line, s_c, s_k),"),
    ("update_taps_from_oldest_entries",
     "                        i = L + TAP_POSITION(0, W, k);",
     "                        i = (W - 1) + TAP_POSITION(0, W, k);"),
]
MUTANTS += [
    ("resolve_same_forward_strict",
     "                if (t - d >= q0) {\n                    *e = SRC_X;",
     "                if (t - d > q0) {\n                    *e = SRC_X;"),
    ("resolve_offset_div",
     "                    *e = b * N + src % N;",
     "                    *e = b * N + (src / N) % N;"),
    ("resolve_logical_wraps",
     "                    int64_t logical = src / N;\n                    if (logical >= max_blocks) { flags |= 0x04;",
     "                    int64_t logical = (src / N) % max_blocks;\n                    if (logical >= max_blocks) { flags |= 0x04;"),
    ("resolve_block_from_token_position",
     "                    int64_t b = block_table[r * bt_row_stride + logical];",
     "                    int64_t b = block_table[r * bt_row_stride + pos / N];"),
    ("resolve_flags_on_first_lag_only",
     "            for (int64_t d = 1; d <= L; ++d) taps[t * L + d - 1] = -(flags * 256);",
     "            for (int64_t d = 1; d <= 1; ++d) taps[t * L + d - 1] = -(flags * 256);"),
    ("resolve_pad_rows_resolved",
     "        if (t >= num_actual || slot_mapping[t] == -1) continue;",
     "        if (t >= num_actual) continue;"),
    ("resolve_search_strict",
     "                    if (query_start_loc[k] <= t) r = k;",
     "                    if (query_start_loc[k] < t) r = k;"),
    ("resolve_decode_start_zero",
     "                r = t;\n                q0 = t;",
     "                r = t;\n                q0 = 0;"),
]
PIN_FILES = ["test_oracle_pins.py", "test_oracle_pins_dense.py", "test_oracle_pins_taps.py"]


def _run_mutant(tmp, name, old, new):
    src = open(SRC).read()
    assert old in src, f"mutant {name}: pattern not found"
    mutated = src.replace(old, new, 1)
    c_path = os.path.join(tmp, f"{name}.c")
    so_path = os.path.join(tmp, f"lib{name}.so")
    with open(c_path, "w") as f:
        f.write(mutated)
    oracle.build(force=True, src=c_path, out=so_path)
    env = dict(os.environ, SCONV_ORACLE_LIB=so_path)
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         *[os.path.join(ROOT, "tests", f) for f in PIN_FILES]],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-400:]


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
            results = list(ex.map(lambda m: _run_mutant(tmp, *m), MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc != 1]
    assert not survivors, f"mutants not caught by a failing assertion: {survivors}"


def test_unmutated_oracle_passes_in_child():
    """Control: the same child-process run passes on the real oracle."""
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         *[os.path.join(ROOT, "tests", f) for f in PIN_FILES]],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
