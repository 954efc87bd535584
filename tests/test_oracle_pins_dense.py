"""Pins of the dense-state oracle functions (CPU only).

oracle.conv1d_fwd / oracle.conv1d_update follow causal_conv1d_fwd and
causal_conv1d_update on "Implementation:Sgl project Sglang Mamba Ops".  They
are pinned against hand-worked examples, a library depthwise conv1d over the
extended input of every sequence, the independently written paged-cache
oracle (fused_sconv, "vllm.models.inkling.nvidia.ops.sconv") on equivalent
inputs, and invariants: chunked prefill equals one-shot prefill, a decode
update equals a one-token prefill, and the circular line equals the shifted
line read in rotated order.
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
W3 = [1.0, 2.0, 3.0]


def _nums(field):
    return [] if field == "-" else [float(v) for v in field.split()]


def read_dense_golden():
    rows = []
    with open(os.path.join(GOLDEN, "hand_worked_dense_w3.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            nm, op, bias, L, st, init, s, x, y, new = [v.strip() for v in line.split("|")]
            rows.append(dict(name=nm, op=op, bias=float(bias), L=int(L), line=_nums(st),
                             init=None if init == "-" else bool(int(init)),
                             s=None if s == "-" else int(s), x=_nums(x), y=_nums(y),
                             new=_nums(new)))
    return rows


def _t(values, dtype, shape):
    return torch.tensor(values, dtype=torch.float32).reshape(shape).to(
        workloads.TORCH_DTYPE[dtype])


def _f64(a, dtype):
    return oracle.to_f64(a, dtype)


# --------------------------------------------------------------------------
# hand-worked examples

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_hand_worked_dense(dtype):
    for r in read_dense_golden():
        w = _t(W3, dtype, (1, 3))
        b = _t([r["bias"]], dtype, (1,))
        st = _t(r["line"], dtype, (1, 1, r["L"]))
        if r["op"] == "fwd":
            n = len(r["x"])
            x = _t(r["x"], dtype, (n, 1))
            out, rs, new, sk = oracle.conv1d_fwd(
                dtype=dtype, x=x, weight=w, bias=b, conv_states=st,
                query_start_loc=np.array([0, n], np.int32),
                has_initial_state=np.array([r["init"]]))
            assert sk == 0 and (rs == 1).all(), r["name"]
        else:
            x = _t(r["x"], dtype, (1, 1))
            seqlens = None if r["s"] is None else np.array([r["s"]], np.int32)
            out, rs, new, sk = oracle.conv1d_update(
                dtype=dtype, x=x, conv_state=st, weight=w, bias=b, cache_seqlens=seqlens)
            assert sk == 0 and rs.tolist() == [1], r["name"]
        assert out[:, 0].tolist() == r["y"], r["name"]
        assert _f64(new, dtype).reshape(-1).tolist() == r["new"], r["name"]


# --------------------------------------------------------------------------
# library conv1d over the extended input of every sequence

def _library_fwd(d, dtype, W, L, silu):
    """Per sequence: e = (line or zeros) ++ x rows, a valid depthwise conv1d
    (torch.nn.functional.conv1d, groups = dim) of e, the last n outputs;
    the new line = e[-L:]."""
    x = torch.from_numpy(_f64(d["x"], dtype))
    w = torch.from_numpy(_f64(d["weight"], dtype))
    dim = x.shape[1]
    bias = None if d["bias"] is None else torch.from_numpy(_f64(d["bias"], dtype))
    states = torch.from_numpy(_f64(d["conv_states"], dtype))
    qsl = d["query_start_loc"].tolist()
    lines = d["cache_indices"].tolist()
    init = d["has_initial_state"].tolist()
    out = torch.zeros_like(x)
    new = states.clone()
    for b in range(len(lines)):
        if lines[b] == d["pad_slot_id"]:
            continue
        hist = states[lines[b]] if init[b] else torch.zeros(dim, L, dtype=torch.float64)
        e = torch.cat([hist, x[qsl[b]:qsl[b + 1]].T], dim=1)         # [dim, L + n]
        y = F.conv1d(e[None], w[:, None, :], bias, groups=dim)[0]   # [dim, L + n - W + 1]
        n = qsl[b + 1] - qsl[b]
        y = y[:, y.shape[1] - n:].T
        out[qsl[b]:qsl[b + 1]] = F.silu(y) if silu else y
        new[lines[b]] = e[:, e.shape[1] - L:]
    return out.numpy(), new.numpy()


def _fwd(d, dtype, act):
    return oracle.conv1d_fwd(
        dtype=dtype, x=d["x"], weight=d["weight"], bias=d["bias"], conv_states=d["conv_states"],
        query_start_loc=d["query_start_loc"], cache_indices=d["cache_indices"],
        has_initial_state=d["has_initial_state"], activation=act, pad_slot_id=d["pad_slot_id"])


@pytest.mark.parametrize("seed", range(8))
def test_fwd_against_library_conv1d(seed):
    rng = np.random.default_rng(seed)
    dtype = ["f32", "bf16"][seed % 2]
    W = int(rng.integers(2, 9))
    L = W - 1 + int(rng.integers(0, 3))
    lens = rng.integers(0, 12, size=int(rng.integers(1, 6)))
    d = workloads.dense_conv_inputs(seed, dtype=dtype, dim=int(rng.integers(1, 7)), W=W,
                                    state_len=L, lens=lens, num_pad=int(len(lens) > 2),
                                    bias=bool(seed % 3))
    act = "silu" if seed % 2 else None
    out, rs, new, sk = _fwd(d, dtype, act)
    ref_out, ref_new = _library_fwd(d, dtype, W, L, act == "silu")
    assert sk == 0
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-12)
    assert np.array_equal(_f64(new, dtype), ref_new)
    lines = d["cache_indices"].tolist()
    qsl = d["query_start_loc"].tolist()
    for b, line in enumerate(lines):
        assert (rs[qsl[b]:qsl[b + 1]] == (0 if line == -1 else 1)).all()


def test_no_states_is_zero_history():
    d = workloads.dense_conv_inputs(7, dtype="f32", dim=5, W=4, state_len=3, lens=[4, 7, 1])
    out, rs, new, _ = oracle.conv1d_fwd(
        dtype="f32", x=d["x"], weight=d["weight"], bias=d["bias"],
        query_start_loc=d["query_start_loc"], activation="silu")
    assert new is None and rs.all()
    d["has_initial_state"] = torch.zeros(3, dtype=torch.bool)
    d["cache_indices"] = torch.arange(3, dtype=torch.int32)
    ref, _ = _library_fwd(d, "f32", 4, 3, True)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# the paged-cache oracle on equivalent inputs

@pytest.mark.parametrize("seed", range(6))
def test_fwd_equals_paged_oracle(seed):
    """Sequence b as request b of fused_sconv (no bias, no residual): with
    an initial state its L line entries are the cached positions 0..L-1
    and its tokens start at position L; without one it starts at position
    0.  Outputs agree exactly and the new line is the cache's last L
    positions."""
    rng = np.random.default_rng(100 + seed)
    dtype = ["bf16", "f32"][seed % 2]
    W = int(rng.integers(2, 7))
    L = W - 1 + int(rng.integers(0, 3))
    N = int(rng.choice([1, 2, 4, 8]))
    lens = rng.integers(1, 10, size=int(rng.integers(1, 5)))
    dim = int(rng.integers(1, 6))
    d = workloads.dense_conv_inputs(200 + seed, dtype=dtype, dim=dim, W=W, state_len=L,
                                    lens=lens, bias=False)
    act = "silu" if seed % 3 else None
    out, rs, new, _ = _fwd(d, dtype, act)

    B = len(lens)
    init = d["has_initial_state"].numpy()
    lines = d["cache_indices"].numpy()
    hist = np.where(init, L, 0)
    total = hist + lens
    nblk = -(-total // N)
    perm = rng.permutation(int(nblk.sum()))
    bt = np.full((B, int(nblk.max())), -1, np.int32)
    cache = torch.zeros((int(nblk.sum()), 1, N, dim), dtype=workloads.TORCH_DTYPE[dtype])
    states = d["conv_states"]
    pos, sid, slot, qs = [], [], [], []
    k = 0
    for b in range(B):
        bt[b, :nblk[b]] = perm[k:k + nblk[b]]
        k += nblk[b]
        for p in range(hist[b]):
            cache[bt[b, p // N], 0, p % N, :] = states[lines[b], :, p]
        for i in range(lens[b]):
            p = hist[b] + i
            pos.append(p)
            sid.append(b)
            slot.append(int(bt[b, p // N]) * N + p % N)
            qs.append(int(d["query_start_loc"][b]))
    f_out, f_rs, f_cache, _ = oracle.fused(
        dtype=dtype, x=d["x"], weight=d["weight"], cache=cache,
        positions=np.array(pos, np.int64), block_table=bt, seq_idx=np.array(sid, np.int32),
        slot_mapping=np.array(slot, np.int64), query_start=np.array(qs, np.int32),
        off_s=0, ws=dim, block_size=N, activation=act, use_residual=False)
    assert rs.all() and f_rs.all()
    assert np.array_equal(out, f_out)
    fc = _f64(torch.from_numpy(f_cache).view(workloads.TORCH_DTYPE[dtype]) if dtype == "bf16"
              else f_cache, dtype)
    nw = _f64(new, dtype)
    for b in range(B):
        for i in range(L):
            p = total[b] - L + i
            want = 0.0 if p < 0 else fc[bt[b, p // N], 0, p % N, :]
            np.testing.assert_array_equal(nw[lines[b], :, i], want)


# --------------------------------------------------------------------------
# invariants

@pytest.mark.parametrize("seed", range(6))
def test_chunked_fwd_equals_one_shot(seed):
    rng = np.random.default_rng(300 + seed)
    dtype = ["bf16", "f32"][seed % 2]
    W = int(rng.integers(2, 9))
    L = W - 1 + int(rng.integers(0, 2))
    lens = rng.integers(0, 14, size=4)
    d = workloads.dense_conv_inputs(300 + seed, dtype=dtype, dim=3, W=W, state_len=L,
                                    lens=lens, num_pad=1)
    out, _, new, _ = _fwd(d, dtype, "silu")
    cut = np.array([int(rng.integers(0, n + 1)) for n in lens])
    qsl = d["query_start_loc"].numpy()
    first = np.concatenate([np.arange(qsl[b], qsl[b] + cut[b]) for b in range(4)]).astype(int)
    second = np.concatenate([np.arange(qsl[b] + cut[b], qsl[b + 1]) for b in range(4)]).astype(int)
    d1 = dict(d, x=d["x"][first], query_start_loc=torch.from_numpy(
        np.concatenate([[0], np.cumsum(cut)]).astype(np.int32)))
    o1, _, s1, _ = _fwd(d1, dtype, "silu")
    d2 = dict(d, x=d["x"][second], conv_states=torch.from_numpy(s1).view(d["x"].dtype)
              if dtype == "bf16" else torch.from_numpy(s1),
              query_start_loc=torch.from_numpy(
                  np.concatenate([[0], np.cumsum(lens - cut)]).astype(np.int32)),
              has_initial_state=torch.ones(4, dtype=torch.bool))
    # sequences whose first part was empty keep their original has_initial_state
    d2["has_initial_state"] = torch.from_numpy((cut > 0) | d["has_initial_state"].numpy())
    o2, _, s2, _ = _fwd(d2, dtype, "silu")
    assert np.array_equal(out[first], o1) and np.array_equal(out[second], o2)
    assert np.array_equal(s2.view(np.uint8), new.view(np.uint8))


@pytest.mark.parametrize("seed", range(4))
def test_update_equals_one_token_fwd(seed):
    rng = np.random.default_rng(400 + seed)
    dtype = ["bf16", "f32"][seed % 2]
    W = int(rng.integers(2, 9))
    L = W - 1 + int(rng.integers(0, 3))
    u = workloads.dense_update_inputs(400 + seed, dtype=dtype, batch=6, dim=4, W=W,
                                      state_len=L, num_pad=1)
    out, rs, new, sk = oracle.conv1d_update(
        dtype=dtype, x=u["x"], conv_state=u["conv_state"], weight=u["weight"], bias=u["bias"],
        activation="silu", conv_state_indices=u["conv_state_indices"])
    f_out, f_rs, f_new, _ = oracle.conv1d_fwd(
        dtype=dtype, x=u["x"], weight=u["weight"], bias=u["bias"], conv_states=u["conv_state"],
        query_start_loc=np.arange(7, dtype=np.int32), cache_indices=u["conv_state_indices"],
        has_initial_state=np.ones(6, bool), activation="silu")
    assert sk == 0 and rs.sum() == 5
    assert np.array_equal(rs, f_rs) and np.array_equal(out, f_out)
    assert np.array_equal(new.view(np.uint8), f_new.view(np.uint8))


@pytest.mark.parametrize("seed", range(4))
def test_ring_update_equals_shift_update_in_rotated_order(seed):
    """With cache_seqlens = s the circular line, read oldest first from
    entry s mod L, is the shifted line; after the update it reads, from
    entry (s+1) mod L, as the shifted line after its update."""
    rng = np.random.default_rng(500 + seed)
    dtype = ["f32", "bf16"][seed % 2]
    W = int(rng.integers(2, 9))
    L = W - 1 + int(rng.integers(0, 3))
    u = workloads.dense_update_inputs(500 + seed, dtype=dtype, batch=5, dim=3, W=W,
                                      state_len=L, ring=True, max_seqlen=50)
    s = u["cache_seqlens"].numpy()
    lines = u["conv_state_indices"].numpy()
    out, _, new, _ = oracle.conv1d_update(
        dtype=dtype, x=u["x"], conv_state=u["conv_state"], weight=u["weight"], bias=u["bias"],
        cache_seqlens=s, conv_state_indices=lines)
    ring = u["conv_state"]
    shifted = ring.clone()
    for b in range(5):
        idx = (s[b] + np.arange(L)) % L
        shifted[lines[b]] = ring[lines[b]][:, idx]
    s_out, _, s_new, _ = oracle.conv1d_update(
        dtype=dtype, x=u["x"], conv_state=shifted, weight=u["weight"], bias=u["bias"],
        conv_state_indices=lines)
    assert np.array_equal(out, s_out)
    for b in range(5):
        idx = (s[b] + 1 + np.arange(L)) % L
        assert np.array_equal(np.ascontiguousarray(new[lines[b]][:, idx]).view(np.uint8),
                              s_new[lines[b]].view(np.uint8))


def test_older_line_entries_only_shift_through():
    """Entries older than the W-1 taps never reach an output; with fewer
    than L new rows they move to the front of the new line."""
    d = workloads.dense_conv_inputs(9, dtype="f32", dim=4, W=3, state_len=5, lens=[2, 1],
                                    has_init=[True, True])
    out, _, new, _ = _fwd(d, "f32", None)
    d2 = dict(d, conv_states=d["conv_states"].clone())
    d2["conv_states"][:, :, :3] = 99.0
    out2, _, _, _ = _fwd(d2, "f32", None)
    assert np.array_equal(out, out2)
    line0 = int(d["cache_indices"][0])
    np.testing.assert_array_equal(new[line0][:, :3], d["conv_states"][line0][:, 2:].numpy())


def test_pad_entries_and_bad_lines():
    d = workloads.dense_conv_inputs(11, dtype="bf16", dim=4, W=4, state_len=3,
                                    lens=[3, 2, 4], num_lines=4, has_init=[1, 1, 1])
    d["cache_indices"] = torch.tensor([-1, 7, 2], dtype=torch.int32)
    out, rs, new, sk = _fwd(d, "bf16", "silu")
    assert sk == 1
    assert rs.tolist() == [0, 0, 0, 2, 2, 1, 1, 1, 1]
    before = oracle._float_array(d["conv_states"], "bf16")
    for line in (0, 1, 3):
        assert np.array_equal(new[line], before[line])
    assert not np.array_equal(new[2], before[2])
    u = workloads.dense_update_inputs(12, dtype="f32", batch=3, dim=2, W=3, state_len=2,
                                      num_lines=2)
    out, rs, new, sk = oracle.conv1d_update(
        dtype="f32", x=u["x"], conv_state=u["conv_state"], weight=u["weight"],
        conv_state_indices=np.array([5, -1, 1], np.int32))
    assert sk == 1 and rs.tolist() == [2, 0, 1]
    assert np.array_equal(new[0], u["conv_state"][0].numpy())


def test_empty_sequence_line():
    """An empty sequence keeps its line when it starts from it and zeroes
    the line when it does not (the last L entries of e)."""
    d = workloads.dense_conv_inputs(13, dtype="f32", dim=3, W=4, state_len=3, lens=[0, 0],
                                    has_init=[True, False])
    _, rs, new, _ = _fwd(d, "f32", None)
    l0, l1 = d["cache_indices"].tolist()
    assert rs.size == 0
    assert np.array_equal(new[l0], d["conv_states"][l0].numpy())
    assert not new[l1].any()


@pytest.mark.parametrize("name", ["dense_prefill_bf16", "dense_decode_bf16"])
def test_dense_named_workloads_are_well_formed(name):
    d = workloads.DENSE_NAMED[name]()
    if "query_start_loc" in d:
        qsl = d["query_start_loc"].numpy()
        assert qsl[0] == 0 and (np.diff(qsl) >= 1).all() and qsl[-1] == d["x"].shape[0]
        lines = d["cache_indices"].numpy()
        states = d["conv_states"]
    else:
        lines = d["conv_state_indices"].numpy()
        states = d["conv_state"]
    live = lines[lines != d["pad_slot_id"]]
    assert len(set(live.tolist())) == len(live)
    assert ((live >= 0) & (live < states.shape[0])).all()
    assert states.shape[1] == d["x"].shape[1] and d["weight"].shape == (d["x"].shape[1], 4)
