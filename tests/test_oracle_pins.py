"""Pins of the CPU oracle against things other than itself (CPU only).

Each test checks the oracle against what the pages and the mathematics fix:
hand-worked examples, a library depthwise conv1d over dense sequences (brute
force), closed forms and special cases, and invariants of the method
("vllm.models.inkling.nvidia.ops.sconv": module docstring, fused_sconv,
sconv_seq_metadata; "core.ssm.ops.intermediate_extraction":
scatter_intermediate_conv).
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._cases import bf16_round, dense_case, textbook_conv, to64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def run_fused(wl, t, **kw):
    args = dict(dtype=wl.dtype, x=t["x"], weight=t["weight"], cache=t["cache"],
                positions=t["positions"], block_table=t["block_table"],
                seq_idx=t["seq_idx"], slot_mapping=t["slot_mapping"],
                query_start=t["query_start"], **wl.kwargs())
    args.update(kw)
    return oracle.fused(**args)


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            nm, w, x, res, exp = [s.strip() for s in line.split("|")]
            rows.append((nm, [float(v) for v in w.split()], [float(v) for v in x.split()],
                         bool(int(res)), [float(v) for v in exp.split()]))
    return rows


# --------------------------------------------------------------------------
# hand-worked examples

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("split", [0, 2, 4])
def test_hand_worked_examples(dtype, split):
    """tests/golden/hand_worked_w4.txt, with the first ``split`` tokens
    already in the cache (history) and the rest in this step."""
    for name, w, x, res, exp in read_golden("hand_worked_w4.txt"):
        seq = np.asarray(x, np.float64)[:, None]
        wl, t = dense_case([seq], [split], dtype=dtype, W=4, N=4, weight=w,
                           residual=res)
        out, state, _, skipped = run_fused(wl, t)
        assert skipped == 0 and state.all()
        assert out[:, 0].tolist() == exp[split:], name


def test_hand_worked_as_decode_steps():
    """The ramp example fed one token per call, each call reading the cache
    the previous call wrote (decode from zero history)."""
    w = [1.0, 2.0, 3.0, 4.0]
    xs = [1.0, 2.0, 3.0, 4.0, 5.0]
    expected = [4.0, 11.0, 20.0, 30.0, 40.0]
    wl, t = dense_case([np.asarray(xs)[:, None]], [0], W=4, N=2, weight=w)
    cache = t["cache"]
    for p in range(len(xs)):
        sl = slice(p, p + 1)
        out, state, cache_np, _ = run_fused(
            wl, t, x=t["x"][sl], positions=t["positions"][sl], seq_idx=t["seq_idx"][sl],
            slot_mapping=t["slot_mapping"][sl], query_start=np.zeros(1, np.int32),
            cache=cache)
        cache = torch.from_numpy(cache_np)
        assert out[0, 0] == expected[p]


# --------------------------------------------------------------------------
# brute force: a library conv1d over dense sequences

def _random_dense(rng, dtype, R, W, H, ws, max_len=24):
    C = H * ws
    seqs, hist = [], []
    for _ in range(R):
        L = int(rng.integers(1, max_len))
        s = rng.standard_normal((L, C))
        seqs.append(bf16_round(s) if dtype == "bf16" else s.astype(np.float32))
        hist.append(int(rng.integers(0, L)))
    w = rng.standard_normal((C, W)) * 0.5
    w = bf16_round(w) if dtype == "bf16" else w.astype(np.float32)
    return seqs, hist, w


@pytest.mark.parametrize("seed", range(12))
def test_against_library_conv1d(seed):
    rng = np.random.default_rng(seed)
    dtype = "bf16" if seed % 2 else "f32"
    W = int(rng.integers(1, 9))
    H = int(rng.integers(1, 4))
    ws = int(rng.integers(1, 6))
    off_s = int(rng.integers(0, 3))
    N = int(rng.choice([1, 2, 3, 4, 8]))
    R = int(rng.integers(1, 5))
    act = "silu" if seed % 3 else None
    residual = bool(seed % 4 < 2)
    seqs, hist, w = _random_dense(rng, dtype, R, W, H, ws)
    wl, t = dense_case(seqs, hist, dtype=dtype, H=H, ws=ws, off_s=off_s,
                       D=off_s + ws + 2, W=W, N=N, weight=w, act=act,
                       residual=residual, seed=seed)
    out, state, _, skipped = run_fused(wl, t)
    assert skipped == 0 and state.all()
    row = 0
    for s, h in zip(seqs, hist):
        ref = textbook_conv(np.asarray(s, np.float64), np.asarray(w, np.float64), act,
                            residual)
        n = len(s) - h
        np.testing.assert_allclose(out[row: row + n], ref[h:], rtol=1e-12, atol=1e-12)
        row += n


def test_pad_rows_feed_neighbours_but_produce_nothing():
    """A PAD row (slot -1) is skipped: no output row, no cache write; its x
    is still the same-forward tap of the next tokens of its request."""
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((6, 4)) * 0.5).astype(np.float32)
    seqs = [rng.standard_normal((9, 6)).astype(np.float32),
            rng.standard_normal((7, 6)).astype(np.float32)]
    hist = [2, 0]
    pad = [3, 8]  # rows of x: request 0 owns rows 0..6, request 1 rows 7..13
    wl, t = dense_case(seqs, hist, H=2, ws=3, W=4, N=4, weight=w, pad_rows=pad,
                       residual=True, act="silu")
    out, state, cache_out, _ = run_fused(wl, t)
    assert state.tolist() == [0 if r in pad else 1 for r in range(wl.T)]
    assert not out[pad].any()
    ref0 = textbook_conv(seqs[0].astype(np.float64), w.astype(np.float64), "silu", True)[2:]
    ref1 = textbook_conv(seqs[1].astype(np.float64), w.astype(np.float64), "silu", True)
    ref = np.concatenate([ref0, ref1])
    keep = [r for r in range(wl.T) if r not in pad]
    np.testing.assert_allclose(out[keep], ref[keep], rtol=1e-12, atol=1e-12)
    # No cache element was written for the PAD rows' positions.
    for r in pad:
        req = int(wl.seq_idx[r])
        p = int(wl.positions[r])
        b = int(wl.block_table[req, p // wl.N])
        np.testing.assert_array_equal(cache_out[b, :, p % wl.N],
                                      t["cache"][b, :, p % wl.N].numpy())


# --------------------------------------------------------------------------
# closed forms and special cases

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_tap_is_a_scaling(dtype):
    """W = 1: out = weight[c] * x[t, c] (+ x), with no history involved."""
    wl = workloads.random_case(3, dtype=dtype)
    wl = workloads.build("w1", dtype=dtype, H=wl.H, D=wl.D, ws=wl.ws, off_s=wl.off_s,
                         W=1, N=wl.N, hist=wl.hist, new=wl.new, act=None,
                         residual=True, seed=3)
    t = wl.tensors()
    out, state, _, _ = run_fused(wl, t)
    expect = to64(t["x"]) * to64(t["weight"])[:, 0][None, :] + to64(t["x"])
    np.testing.assert_array_equal(out[state == 1], expect[state == 1])


@pytest.mark.parametrize("seed", range(4))
def test_zero_weight_residual_is_identity(seed):
    wl = workloads.random_case(seed)
    wl.act = None
    wl.residual = True
    t = wl.tensors()
    t["weight"] = torch.zeros_like(t["weight"])
    out, state, _, _ = run_fused(wl, t)
    np.testing.assert_array_equal(out[state == 1], to64(t["x"])[state == 1])


@pytest.mark.parametrize("seed", range(4))
def test_epilogue_order(seed):
    """act(conv) + x: the SiLU result (torch's silu) of the plain conv, plus
    x, equals the oracle's silu+residual output."""
    wl = workloads.random_case(100 + seed)
    t = wl.tensors()
    plain, s0, _, _ = run_fused(wl, t, activation=None, use_residual=False)
    both, s1, _, _ = run_fused(wl, t, activation="silu", use_residual=True)
    assert (s0 == s1).all()
    ref = torch.nn.functional.silu(torch.from_numpy(plain)).numpy() + to64(t["x"])
    np.testing.assert_allclose(both[s1 == 1], ref[s1 == 1], rtol=1e-14, atol=1e-15)
    zero = np.zeros_like(plain)
    assert (torch.nn.functional.silu(torch.from_numpy(zero)).numpy() == 0).all()


# --------------------------------------------------------------------------
# invariants

def _apply_in_chunks(wl, t, cuts):
    """Run the step as successive calls over request-aligned token chunks
    whose later chunks read what the earlier ones inserted."""
    cache = t["cache"]
    outs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sub = workloads.build(
            "chunk", dtype=wl.dtype, H=wl.H, D=wl.D, ws=wl.ws, off_s=wl.off_s, W=wl.W,
            N=wl.N, hist=wl.hist + a, new=np.full(wl.R, b - a), act=wl.act,
            residual=wl.residual, seed=0)
        # reuse the full step's block table so the chunks address the same blocks
        m = sub.metadata()
        bt = torch.from_numpy(wl.block_table)
        pos = m["positions"]
        slot = (bt[m["seq_idx"].long(), (pos // wl.N)].long() * wl.N + pos % wl.N)
        rows = torch.cat([torch.arange(int(wl.query_start_loc[r]) + a,
                                       int(wl.query_start_loc[r]) + b)
                          for r in range(wl.R)])
        out, state, cache_np, _ = oracle.fused(
            dtype=wl.dtype, x=t["x"][rows], weight=t["weight"], cache=cache,
            positions=pos, block_table=bt, seq_idx=m["seq_idx"], slot_mapping=slot,
            query_start=m["query_start"], **wl.kwargs())
        cache = cache_np
        outs.append((rows, out))
    return outs, cache


@pytest.mark.parametrize("seed", range(6))
def test_chunked_prefill_equals_one_shot(seed):
    """Prefill split into chunks (each later chunk reading the cache the
    earlier ones wrote) gives exactly the one-shot result and cache."""
    rng = np.random.default_rng(seed)
    L = int(rng.integers(6, 20))
    R = int(rng.integers(1, 4))
    dtype = "bf16" if seed % 2 else "f32"
    wl = workloads.build("full", dtype=dtype, H=2, D=12, ws=5, off_s=3,
                         W=int(rng.integers(2, 8)), N=int(rng.choice([1, 3, 4])),
                         hist=rng.integers(0, 9, size=R), new=np.full(R, L),
                         act="silu" if seed % 3 else None, residual=bool(seed % 2),
                         seed=seed)
    t = wl.tensors()
    one, state, cache_one, _ = run_fused(wl, t)
    inner = sorted(set(int(c) for c in rng.integers(1, L, size=3)))
    outs, cache_chunked = _apply_in_chunks(wl, t, [0, *inner, L])
    for rows, out in outs:
        np.testing.assert_array_equal(out, one[rows.numpy()])
    np.testing.assert_array_equal(cache_chunked, cache_one)


@pytest.mark.parametrize("seed", range(3))
def test_zero_history_decode_equals_prefill(seed):
    """Token-by-token decode from an empty history reproduces the one-shot
    prefill of the same tokens exactly."""
    rng = np.random.default_rng(50 + seed)
    L = 9
    wl = workloads.build("full", dtype="f32", H=3, D=8, ws=2, off_s=1, W=4, N=2,
                         hist=np.zeros(2, np.int64), new=np.full(2, L), act="silu",
                         residual=True, seed=seed)
    t = wl.tensors()
    one, _, _, _ = run_fused(wl, t)
    outs, _ = _apply_in_chunks(wl, t, list(range(L + 1)))
    for rows, out in outs:
        np.testing.assert_array_equal(out, one[rows.numpy()])


@pytest.mark.parametrize("seed", range(6))
def test_cache_holds_x_at_every_written_position(seed):
    """After the step, the element for (request r, absolute position p,
    head h, lane j) -- found through the block table -- is x's element, for
    every non-PAD token; every other element of the cache is unchanged."""
    wl = workloads.random_case(200 + seed, pad_frac=0.3)
    t = wl.tensors()
    _, state, cache_out, _ = run_fused(wl, t)
    raw_in = oracle._float_array(t["cache"], wl.dtype)
    after = cache_out.copy()
    xs = oracle._float_array(t["x"], wl.dtype)
    expected_written = np.zeros(raw_in.shape, bool)
    for row in range(wl.T):
        if wl.slot_mapping[row] == -1:
            continue
        r, p = int(wl.seq_idx[row]), int(wl.positions[row])
        b = int(wl.block_table[r, p // wl.N])
        for h in range(wl.H):
            lanes = slice(wl.off_s, wl.off_s + wl.ws)
            np.testing.assert_array_equal(after[b, h, p % wl.N, lanes],
                                          xs[row, h * wl.ws:(h + 1) * wl.ws])
            expected_written[b, h, p % wl.N, lanes] = True
    np.testing.assert_array_equal(after[~expected_written], raw_in[~expected_written])


def test_bad_indices_skip_the_token():
    """Out-of-range slot, request, block-table entry or query_start: that
    token is skipped whole and counted; the others are unaffected."""
    wl = workloads.random_case(11, pad_frac=0.0, max_hist=20)
    t = wl.tensors()
    base, s0, _, _ = run_fused(wl, t)
    assert s0.all()
    bad = {}
    slot = t["slot_mapping"].clone()
    slot[0] = wl.num_blocks * wl.N  # past the pool
    bad[0] = ("slot_mapping", slot)
    for row, (name, val) in bad.items():
        out, state, _, skipped = run_fused(wl, t, **{name: val})
        assert skipped == 1 and state[row] == 2
        keep = state == 1
        np.testing.assert_array_equal(out[keep], base[keep])
    sid = t["seq_idx"].clone()
    sid[-1] = wl.R
    out, state, _, skipped = run_fused(wl, t, seq_idx=sid)
    assert skipped == 1 and state[-1] == 2


# --------------------------------------------------------------------------
# seq metadata

@pytest.mark.parametrize("seed", range(8))
def test_seq_metadata_against_searchsorted_and_layout(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 40))
    lens = rng.integers(0, 6, size=R)  # includes empty requests
    if lens.sum() == 0:
        lens[-1] = 1
    qsl = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(qsl[-1])
    padded = T + int(rng.integers(0, 9))
    si, qs = oracle.seq_metadata(qsl, R, T, padded)
    t = np.arange(T)
    ref = np.searchsorted(qsl[:R], t, side="right") - 1
    np.testing.assert_array_equal(si[:T], ref)
    np.testing.assert_array_equal(qs[:T], qsl[ref])
    assert not si[T:].any() and not qs[T:].any()
    # the generator's by-construction layout agrees
    wl = workloads.build("m", dtype="f32", H=1, D=1, ws=1, off_s=0, W=2, N=4,
                         hist=np.zeros(R, np.int64), new=lens, act=None,
                         residual=False, seed=seed)
    np.testing.assert_array_equal(si[:T], wl.seq_idx)
    np.testing.assert_array_equal(qs[:T], wl.query_start)


# --------------------------------------------------------------------------
# window extraction

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d_conv", [1, 3, 4])
def test_extract_windows_against_padded_slicing(dtype, d_conv):
    seq_len, conv_dim, max_count, real = 23, 10, 9, 6
    src, pos, rc, out = workloads.extraction_inputs(
        5, seq_len, conv_dim, max_count, d_conv, real, dtype=dtype, lo=0,
        hi=seq_len + d_conv)
    got = oracle.extract_windows(dtype=dtype, src=src, abs_positions=pos,
                                 real_count=real, out=out, d_conv=d_conv)
    raw_src = oracle._float_array(src, dtype)
    raw_out = oracle._float_array(out, dtype)
    padded = np.concatenate([np.zeros((d_conv, conv_dim), raw_src.dtype), raw_src,
                             np.zeros((d_conv, conv_dim), raw_src.dtype)])
    for i in range(max_count):
        if i < real:
            p = int(pos[i])
            window = padded[p: p + d_conv]  # rows p-d_conv .. p-1 of src
            np.testing.assert_array_equal(got[i], window.T)
        else:
            np.testing.assert_array_equal(got[i], raw_out[i])


def test_extract_windows_edges():
    """End positions 0..d_conv-1 and past seq_len read zeros outside src."""
    src = torch.arange(1, 13, dtype=torch.float32).reshape(6, 2)
    pos = np.array([0, 1, 3, 6, 8], np.int32)
    out = torch.full((5, 2, 3), -7.0)
    got = oracle.extract_windows(dtype="f32", src=src, abs_positions=pos,
                                 real_count=5, out=out, d_conv=3)
    # channel 0 of src is 1,3,5,7,9,11 at positions 0..5
    assert got[0, 0].tolist() == [0, 0, 0]
    assert got[1, 0].tolist() == [0, 0, 1]
    assert got[2, 0].tolist() == [1, 3, 5]
    assert got[3, 1].tolist() == [8, 10, 12]
    assert got[4, 0].tolist() == [11, 0, 0]


def test_extract_real_count_bounds():
    """real_count 0 writes nothing; a real_count above max_count is clamped."""
    src, pos, rc, out = workloads.extraction_inputs(1, 12, 3, 5, 2, 0, dtype="f32")
    raw = oracle._float_array(out, "f32").view(np.uint32)
    none = oracle.extract_windows(dtype="f32", src=src, abs_positions=pos,
                                  real_count=0, out=out, d_conv=2)
    np.testing.assert_array_equal(none.view(np.uint32), raw)
    full = oracle.extract_windows(dtype="f32", src=src, abs_positions=pos,
                                  real_count=99, out=out, d_conv=2)
    assert not (full.view(np.uint32) == raw).any()


# --------------------------------------------------------------------------
# the generator's workloads meet the one-launch preconditions

@pytest.mark.parametrize("name", ["tiny_prefill_f32", "spec_decode_bf16"])
def test_named_workloads_are_well_formed(name):
    wl = workloads.NAMED[name]()
    assert oracle.check_preconditions(
        W=wl.W, block_size=wl.N, positions=wl.positions, seq_idx=wl.seq_idx,
        slot_mapping=wl.slot_mapping, query_start=wl.query_start,
        block_table=wl.block_table) == 0


def test_named_workload_sizes():
    wl = workloads.tiny_prefill_f32()
    assert (wl.T, wl.C, wl.num_blocks, wl.block_table.shape) == (8, 8, 8, (2, 4))
    assert sorted(wl.block_table.ravel().tolist()) == list(range(8))
    wl = workloads.spec_decode_bf16()
    assert wl.T == 512 and wl.num_pad == 51 and wl.C == 2048
    assert wl.cache_elems * wl.elem_bytes > 2**31  # byte offsets exceed int32
    wl = workloads.decode_bf16()
    assert wl.T == 256 and wl.C == 1024 and wl.off_s == 32
    assert wl.cache_elems * wl.elem_bytes > 2**31  # byte offsets exceed int32


@pytest.mark.parametrize("seed", range(20))
def test_random_cases_are_well_formed(seed):
    wl = workloads.random_case(seed)
    assert oracle.check_preconditions(
        W=wl.W, block_size=wl.N, positions=wl.positions, seq_idx=wl.seq_idx,
        slot_mapping=wl.slot_mapping, query_start=wl.query_start,
        block_table=wl.block_table) == 0


def test_precondition_checker_detects_violations():
    wl = workloads.random_case(4, pad_frac=0.0, max_hist=30)
    kw = dict(W=wl.W, block_size=wl.N, positions=wl.positions, seq_idx=wl.seq_idx,
              slot_mapping=wl.slot_mapping, query_start=wl.query_start,
              block_table=wl.block_table)
    dup = wl.slot_mapping.copy()
    if wl.T >= 2:
        dup[1] = dup[0]
        assert oracle.check_preconditions(**{**kw, "slot_mapping": dup}) == 2
    pos = wl.positions.copy()
    pos[-1] += 1
    if wl.new[-1] >= 2:
        assert oracle.check_preconditions(**{**kw, "positions": pos}) == 1


# --------------------------------------------------------------------------
# several streams of one layer

def _two_stream_case(seed, dtype="bf16"):
    rng = np.random.default_rng(seed)
    wl = workloads.build("kv", dtype=dtype, H=3, D=24, ws=8, off_s=0, W=4, N=4,
                         hist=rng.integers(0, 12, size=3), new=rng.integers(1, 9, size=3),
                         act="silu", residual=True, seed=seed, num_pad=2, rng=rng)
    t = wl.tensors()
    g = torch.Generator().manual_seed(seed + 1)
    streams = [
        dict(x=t["x"], weight=t["weight"], off_s=0, ws=8, activation="silu", use_residual=True),
        dict(x=torch.randn(wl.T, 3 * 6, generator=g).to(t["x"].dtype),
             weight=(torch.randn(18, 4, generator=g) * 0.5).to(t["x"].dtype),
             off_s=10, ws=6, activation=None, use_residual=False),
    ]
    return wl, t, streams


@pytest.mark.parametrize("seed", range(4))
def test_streams_equal_sequential_single_stream_calls(seed):
    """With disjoint lane ranges, applying the streams one after another
    (each later stream reading the cache the earlier ones wrote) gives the
    same outputs and cache as the combined definition."""
    wl, t, streams = _two_stream_case(seed)
    md = dict(positions=wl.positions, block_table=wl.block_table, seq_idx=wl.seq_idx,
              slot_mapping=wl.slot_mapping, query_start=wl.query_start)
    outs, states, cache_all, _ = oracle.fused_streams(
        dtype=wl.dtype, streams=streams, cache=t["cache"], block_size=wl.N, **md)
    cache = t["cache"]
    for sd, out_c in zip(streams, outs):
        out, st, cache_np, _ = oracle.fused(
            dtype=wl.dtype, x=sd["x"], weight=sd["weight"], cache=cache, off_s=sd["off_s"],
            ws=sd["ws"], block_size=wl.N, activation=sd["activation"],
            use_residual=sd["use_residual"], **md)
        np.testing.assert_array_equal(out, out_c)
        cache = cache_np
    np.testing.assert_array_equal(cache, cache_all)
    # and every stream's written lanes hold its own x (read back by 4-D indexing)
    for sd in streams:
        xs = oracle._float_array(sd["x"], wl.dtype)
        for row in range(wl.T):
            if wl.slot_mapping[row] == -1:
                continue
            r, p = int(wl.seq_idx[row]), int(wl.positions[row])
            b = int(wl.block_table[r, p // wl.N])
            for h in range(wl.H):
                np.testing.assert_array_equal(
                    cache_all[b, h, p % wl.N, sd["off_s"]:sd["off_s"] + sd["ws"]],
                    xs[row, h * sd["ws"]:(h + 1) * sd["ws"]])


# --------------------------------------------------------------------------
# SSM state gather and window extraction from the paged cache

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("real", [0, 3, 7, 20])
def test_scatter_ssm_against_fancy_indexing(dtype, real):
    rng = np.random.default_rng(real)
    states = torch.randn(11, 3, 5).to(workloads.TORCH_DTYPE[dtype])
    idx = rng.integers(0, 11, size=7).astype(np.int64)
    idx[2] = 11  # out of range: that slot is skipped
    out = workloads.sentinel((7, 3, 5), dtype)
    got, skipped = oracle.scatter_ssm(dtype=dtype, states=states, chunk_indices=idx,
                                      real_count=real, out=out)
    raw_s = oracle._float_array(states, dtype)
    raw_o = oracle._float_array(out, dtype)
    expect = raw_o.copy()
    rc = min(real, 7)
    for i in range(rc):
        if 0 <= idx[i] < 11:
            expect[i] = raw_s[idx[i]]
    np.testing.assert_array_equal(got.view(np.uint8), expect.view(np.uint8))
    assert skipped == (1 if rc > 2 else 0)


def _paged_windows_by_indexing(cache_raw, bt, req, pos, d_conv, off_s, ws, N, out_raw):
    H = cache_raw.shape[1]
    out = out_raw.copy()
    for i, (r, p_end) in enumerate(zip(req, pos)):
        for k in range(d_conv):
            p = int(p_end) - d_conv + k
            for h in range(H):
                if p < 0:
                    out[i, h * ws:(h + 1) * ws, k] = 0
                else:
                    out[i, h * ws:(h + 1) * ws, k] = cache_raw[bt[r, p // N], h, p % N,
                                                               off_s:off_s + ws]
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d_conv", [1, 4, 6])
def test_extract_windows_paged_against_indexing(dtype, d_conv):
    wl = workloads.random_case(61 + d_conv, dtype=dtype, max_hist=30)
    t = wl.tensors()
    rng = np.random.default_rng(d_conv)
    n = 9
    req = rng.integers(0, wl.R, size=n).astype(np.int32)
    lengths = wl.hist + wl.new
    pos = np.array([rng.integers(0, lengths[r] + 1) for r in req], np.int32)
    out = workloads.sentinel((n, wl.C, d_conv), dtype)
    got, skipped = oracle.extract_windows_paged(
        dtype=dtype, cache=t["cache"], block_table=wl.block_table, request=req,
        abs_positions=pos, real_count=6, out=out, d_conv=d_conv, off_s=wl.off_s, ws=wl.ws)
    assert skipped == 0
    raw_o = oracle._float_array(out, dtype)
    expect = _paged_windows_by_indexing(oracle._float_array(t["cache"], dtype),
                                        wl.block_table, req[:6], pos[:6], d_conv, wl.off_s,
                                        wl.ws, wl.N, raw_o)
    np.testing.assert_array_equal(got.view(np.uint8), expect.view(np.uint8))


def test_extract_windows_paged_equals_dense_after_prefill():
    """Prefill sequences from position 0 (the fused oracle inserts every
    token into the paged cache); windows read back from the cache equal the
    dense extraction from the same x rows."""
    wl = workloads.build("pf", dtype="bf16", H=3, D=20, ws=6, off_s=7, W=4, N=4,
                         hist=[0, 0], new=[13, 9], act="silu", residual=False, seed=5)
    t = wl.tensors()
    _, _, cache_after, _ = run_fused(wl, t)
    d_conv, rng = 4, np.random.default_rng(5)
    for r in range(2):
        a, b = int(wl.query_start_loc[r]), int(wl.query_start_loc[r + 1])
        pos = rng.integers(0, b - a + 1, size=5).astype(np.int32)
        out = workloads.sentinel((5, wl.C, d_conv), "bf16")
        paged, _ = oracle.extract_windows_paged(
            dtype="bf16", cache=cache_after, block_table=wl.block_table,
            request=np.full(5, r, np.int32), abs_positions=pos, real_count=5, out=out,
            d_conv=d_conv, off_s=wl.off_s, ws=wl.ws)
        dense = oracle.extract_windows(dtype="bf16", src=t["x"][a:b], abs_positions=pos,
                                       real_count=5, out=out, d_conv=d_conv)
        np.testing.assert_array_equal(paged, dense)


def test_extract_windows_paged_bad_indices_skip_the_slot():
    wl = workloads.random_case(70, dtype="f32", max_hist=20)
    t = wl.tensors()
    req = np.array([0, wl.R, 0], np.int32)  # slot 1: no such request
    pos = np.array([1, 1, 1], np.int32)
    out = workloads.sentinel((3, wl.C, 2), "f32")
    got, skipped = oracle.extract_windows_paged(
        dtype="f32", cache=t["cache"], block_table=wl.block_table, request=req,
        abs_positions=pos, real_count=3, out=out, d_conv=2, off_s=wl.off_s, ws=wl.ws)
    assert skipped == 1
    assert (got[1].view(np.uint32) == 0xFFFFFFFF).all()
