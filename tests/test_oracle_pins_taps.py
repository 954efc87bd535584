"""Pins of the oracle's tap resolution (CPU only).

The resolution names, for every token and lag d = 1..W-1, where the tap at
position pos - d comes from ("vllm.models.inkling.nvidia.ops.sconv", module
docstring and fused_sconv argument comments): the same-forward x row
(-2), zero before position 0 (-1), or the flat cache slot block*N + offset
through block_table[req][src // N].  It is pinned here by
  * hand-worked tables (tests/golden/resolve_taps_w4.txt),
  * brute force: every position of every request is given an identity and
    placed in an identity cache by the block table's own layout; each
    resolved slot must hold the identity of (request, pos - d), each x entry
    must name a row of the same request at pos - d, and a zero entry must
    mean pos - d < 0;
  * the metadata it returns against numpy's searchsorted,
  * the bounds policy: each bad index gives its flag bits at every lag of
    its token, and nothing else changes.
"""
from __future__ import annotations

import os

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "resolve_taps_w4.txt")


def _golden():
    cases = {}
    for line in open(GOLDEN):
        if not line.strip() or line.startswith("#"):
            continue
        name, row, pos, slot, si, qs, taps = [f.strip() for f in line.split("|")]
        cases.setdefault(name, []).append(
            (int(row), int(pos), int(slot), int(si), int(qs), [int(v) for v in taps.split()]))
    return cases


def test_hand_worked_varlen_table():
    rows = _golden()["varlen"]
    pos = np.array([r[1] for r in rows[:6]], np.int64)
    slot = np.array([r[2] for r in rows[:6]], np.int64)
    bt = np.array([[5, 2, -1], [7, -1, -1], [1, -1, -1]], np.int32)
    si, qs, taps = oracle.resolve_taps(
        query_start_loc=np.array([0, 2, 5, 6], np.int32), num_reqs=3, num_actual_tokens=6,
        num_padded_tokens=8, positions=pos, slot_mapping=slot, block_table=bt, num_blocks=8,
        block_size=4, W=4)
    np.testing.assert_array_equal(si, [r[3] for r in rows])
    np.testing.assert_array_equal(qs, [r[4] for r in rows])
    np.testing.assert_array_equal(taps, [r[5] for r in rows])


def test_hand_worked_decode_table():
    rows = _golden()["decode"]
    bt = np.array([[3, 6, -1], [1, -1, -1], [0, 2, 5]], np.int32)
    si, qs, taps = oracle.resolve_taps(
        query_start_loc=None, num_reqs=3, num_actual_tokens=3,
        positions=np.array([r[1] for r in rows], np.int64),
        slot_mapping=np.array([r[2] for r in rows], np.int64), block_table=bt, num_blocks=8,
        block_size=4, W=4)
    np.testing.assert_array_equal(si, [r[3] for r in rows])
    np.testing.assert_array_equal(qs, [r[4] for r in rows])
    np.testing.assert_array_equal(taps, [r[5] for r in rows])


def _identity_cache(wl):
    """[num_blocks, N] table holding, at the block-table place of every
    position p of request r, the identity r * 2^20 + p (-1 elsewhere)."""
    ident = np.full((wl.num_blocks, wl.N), -1, np.int64)
    for r in range(wl.R):
        for p in range(int(wl.hist[r] + wl.new[r])):
            ident[wl.block_table[r, p // wl.N], p % wl.N] = (r << 20) + p
    return ident


def _check_brute_force(wl, taps):
    ident = _identity_cache(wl)
    W = wl.W
    for t in range(wl.T):
        if wl.slot_mapping[t] == -1:
            assert (taps[t] == -1).all()
            continue
        r, pos = int(wl.seq_idx[t]), int(wl.positions[t])
        first = int(wl.query_start_loc[r])
        for d in range(1, W):
            e = int(taps[t, d - 1])
            src = pos - d
            if t - d >= first:
                assert e == oracle.SRC_X, (t, d, e)
                assert wl.seq_idx[t - d] == r and wl.positions[t - d] == src
            elif src < 0:
                assert e == oracle.SRC_ZERO, (t, d, e)
            else:
                assert e >= 0, (t, d, e)
                assert ident[e // wl.N, e % wl.N] == (r << 20) + src, (t, d, e)


@pytest.mark.parametrize("seed", range(60))
def test_brute_force_against_identity_cache(seed):
    wl = workloads.random_case(seed, max_new=30, max_hist=40)
    si, qs, taps = oracle.resolve_taps(
        query_start_loc=wl.query_start_loc, num_reqs=wl.R, num_actual_tokens=wl.T,
        positions=wl.positions, slot_mapping=wl.slot_mapping, block_table=wl.block_table,
        num_blocks=wl.num_blocks, block_size=wl.N, W=wl.W)
    assert taps.shape == (wl.T, wl.W - 1)
    np.testing.assert_array_equal(si, wl.seq_idx)
    np.testing.assert_array_equal(qs, wl.query_start)
    qsl = np.asarray(wl.query_start_loc)
    ref = np.searchsorted(qsl[:-1], np.arange(wl.T), side="right") - 1
    np.testing.assert_array_equal(si, ref)
    _check_brute_force(wl, taps)


@pytest.mark.parametrize("seed", range(8))
def test_brute_force_decode_form(seed):
    """Token b is request b: the same identities, read without query_start_loc."""
    wl = workloads.decode_bf16(seed=200 + seed, R=48, max_hist=300)
    si, qs, taps = oracle.resolve_taps(
        query_start_loc=None, num_reqs=wl.R, num_actual_tokens=wl.T, positions=wl.positions,
        slot_mapping=wl.slot_mapping, block_table=wl.block_table, num_blocks=wl.num_blocks,
        block_size=wl.N, W=wl.W)
    np.testing.assert_array_equal(si, np.arange(wl.T))
    np.testing.assert_array_equal(qs, np.arange(wl.T))
    _check_brute_force(wl, taps)


def test_long_window_and_block_size_one():
    """W = 8 with N = 1: every pre-forward tap in a block of its own."""
    rng = np.random.default_rng(5)
    wl = workloads.build("w8n1", dtype="bf16", H=1, D=8, ws=8, off_s=0, W=8, N=1,
                         hist=rng.integers(0, 12, size=5), new=rng.integers(1, 9, size=5),
                         act=None, residual=False, seed=5, num_pad=3, rng=rng)
    _, _, taps = oracle.resolve_taps(
        query_start_loc=wl.query_start_loc, num_reqs=wl.R, num_actual_tokens=wl.T,
        positions=wl.positions, slot_mapping=wl.slot_mapping, block_table=wl.block_table,
        num_blocks=wl.num_blocks, block_size=wl.N, W=wl.W)
    _check_brute_force(wl, taps)


def test_w1_has_no_taps():
    _, _, taps = oracle.resolve_taps(
        query_start_loc=np.array([0, 2], np.int32), num_reqs=1, num_actual_tokens=2,
        positions=np.array([3, 4]), slot_mapping=np.array([3, 4]),
        block_table=np.array([[0, 1]], np.int32), num_blocks=2, block_size=4, W=1)
    assert taps.shape == (2, 0)


def _bad_case():
    """Request 1 has one token at position 20 reading three history taps."""
    rng = np.random.default_rng(40)
    return workloads.build("err", dtype="bf16", H=1, D=8, ws=8, off_s=0, W=4, N=8,
                           hist=np.array([5, 20, 0, 9]), new=np.array([6, 1, 7, 2]),
                           act=None, residual=False, seed=40, rng=rng)


def _resolve(wl, qsl, pos, slot, bt, num_reqs=None):
    return oracle.resolve_taps(query_start_loc=qsl, num_reqs=num_reqs or wl.R,
                               num_actual_tokens=wl.T, positions=pos, slot_mapping=slot,
                               block_table=bt, num_blocks=wl.num_blocks, block_size=wl.N, W=wl.W)


@pytest.mark.parametrize("kind,flag", [("logical", 0x04), ("block", 0x08), ("position", 0x20)])
def test_bad_index_gives_its_flags_at_every_lag(kind, flag):
    wl = _bad_case()
    qsl = np.asarray(wl.query_start_loc, np.int32)
    pos, slot, bt = wl.positions.copy(), wl.slot_mapping.copy(), wl.block_table.copy()
    row = int(qsl[1])
    _, _, good = _resolve(wl, qsl, pos, slot, bt)
    if kind == "logical":
        pos[row] = bt.shape[1] * wl.N + 2          # history beyond the table
    elif kind == "block":
        bt[1, (int(pos[row]) - 1) // wl.N] = wl.num_blocks + 7
    else:
        pos[row] = -3
    _, _, taps = _resolve(wl, qsl, pos, slot, bt)
    assert (taps[row] == -flag * 256).all()
    others = np.arange(wl.T) != row
    np.testing.assert_array_equal(taps[others], good[others])


def test_flags_are_the_union_over_the_taps():
    """One tap past the table (0x04) and another on a bad block (0x08)."""
    wl = workloads.build("u", dtype="bf16", H=1, D=8, ws=8, off_s=0, W=4, N=4,
                         hist=np.array([7]), new=np.array([1]), act=None, residual=False,
                         seed=1)
    bt = np.array([[1, -5]], np.int32)       # positions 4..7 in a bad block; 8.. past the table
    pos = np.array([9], np.int64)            # taps at 8 (past), 7 and 6 (bad block)
    _, _, taps = _resolve(wl, np.array([0, 1], np.int32), pos, wl.slot_mapping, bt)
    assert (taps[0] == -(0x04 | 0x08) * 256).all()


def test_request_and_query_start_flags():
    wl = _bad_case()
    # decode form with fewer block-table rows than tokens: token t >= rows has no request
    _, _, taps = _resolve(wl, None, wl.positions, wl.slot_mapping, wl.block_table, num_reqs=4)
    assert (taps[4:] == -0x02 * 256).all()
    # a query_start_loc that starts past 0 puts the first rows' start after them
    qsl = np.asarray(wl.query_start_loc, np.int32).copy()
    qsl[0] = 3
    _, qs, taps = _resolve(wl, qsl, wl.positions, wl.slot_mapping, wl.block_table)
    assert (qs[:3] == 3).all() and (taps[:3] == -0x10 * 256).all()


def test_pad_rows_are_never_flagged():
    """A PAD row's other metadata may be anything: it resolves to -1."""
    wl = _bad_case()
    pos, slot = wl.positions.copy(), wl.slot_mapping.copy()
    pos[2], slot[2] = -99, -1
    _, _, taps = _resolve(wl, np.asarray(wl.query_start_loc, np.int32), pos, slot,
                          wl.block_table)
    assert (taps[2] == -1).all()
