"""GPU parity of sconv_causal_conv1d_fwd / sconv_causal_conv1d_update (the
dense-state interface of "Implementation:Sgl project Sglang Mamba Ops")
against the CPU oracle on the same seeded inputs.

Outputs of computed rows within the path's tolerance; rows of skipped or
padded sequences, and every state line byte, bit-exact.  The cases cover the
tiled kernel at every column width (1, 2, 4 and 8 packs, chosen by the grid
rule from the batch and dim), several tiles with ragged tails, the
any-layout kernel (channel-major x, odd dims), the in-place and out-of-place
forms, both state layouts, no state lines, padded and bad lines, and the
shifted and circular update.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import assert_close, hs, raw

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t, dtype):
    return oracle._float_array(t.cpu(), dtype).view(np.uint8)


def _to(d, device):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _run_fwd(d, dtype, silu, *, in_place=True, with_states=True, err=None):
    g = _to(d, DEV)
    # The device copy keeps x's strides (channel-major stays channel-major).
    if not d["x"].is_contiguous():
        g["x"] = d["x"].t().contiguous().to(DEV).t()
    states = g["conv_states"] if with_states else None
    if with_states and not d["conv_states"].is_contiguous():
        g["conv_states"] = d["conv_states"].transpose(1, 2).contiguous().to(DEV).transpose(1, 2)
        states = g["conv_states"]
    x_before = g["x"].cpu()
    out = None
    if not in_place:
        out = workloads.sentinel(tuple(g["x"].shape), dtype, DEV)
        if not g["x"].is_contiguous():
            out = workloads.sentinel(tuple(g["x"].t().shape), dtype, DEV).t()
    res = hs().sconv_causal_conv1d_fwd(
        g["x"], g["weight"], g["bias"], states, g["query_start_loc"], g["cache_indices"],
        g["has_initial_state"], silu, d["pad_slot_id"], out=out, err_flag=err)
    torch.cuda.synchronize()
    ref, rs, st_ref, sk = oracle.conv1d_fwd(
        dtype=dtype, x=x_before, weight=d["weight"], bias=d["bias"],
        conv_states=d["conv_states"] if with_states else None,
        query_start_loc=d["query_start_loc"], cache_indices=d["cache_indices"],
        has_initial_state=d["has_initial_state"], activation="silu" if silu else None,
        pad_slot_id=d["pad_slot_id"])
    got = res.cpu()
    rows = rs == 1
    assert_close(oracle.to_f64(got, dtype)[rows], ref[rows], dtype, "dense fwd out")
    untouched = torch.from_numpy(~rows)
    want = raw(x_before)[untouched] if in_place else torch.full_like(raw(got)[untouched], -1)
    assert torch.equal(raw(got)[untouched], want), "rows outside computed sequences changed"
    if with_states:
        np.testing.assert_array_equal(_bits(states, dtype), st_ref.view(np.uint8),
                                      err_msg="state lines differ")
    return sk


@pytest.mark.parametrize("batch,dim,expect_pp", [(40, 512, 8), (10, 1024, 4), (5, 1024, 2),
                                                 (1, 256, 1)])
@pytest.mark.parametrize("W", [2, 4, 7])
def test_fwd_tile_every_column_width(batch, dim, expect_pp, W):
    """Tiles of 256 / PP rows: lengths up to 600 give several tiles and a
    ragged last one at every width."""
    rng = np.random.default_rng(batch * 100 + W)
    lens = rng.integers(0, 601, size=batch)
    d = workloads.dense_conv_inputs(batch * 10 + W, dtype="bf16", dim=dim, W=W,
                                    state_len=W - 1 + int(rng.integers(0, 3)), lens=lens,
                                    num_pad=batch // 5)
    assert _run_fwd(d, "bf16", silu=W != 7) == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fwd_tile_many_sequences(dtype):
    """More sequences than the longest-first ordering ranks (64): blocks
    interleave the sequences instead; short and empty sequences, pads."""
    rng = np.random.default_rng(77)
    lens = rng.integers(0, 90, size=150)
    d = workloads.dense_conv_inputs(77, dtype=dtype, dim=64, W=4, state_len=5, lens=lens,
                                    num_pad=12, num_lines=200)
    assert _run_fwd(d, dtype, silu=True) == 0


@pytest.mark.parametrize("seed", range(16))
def test_fwd_random(seed):
    rng = np.random.default_rng(700 + seed)
    dtype = ["bf16", "f32"][seed % 2]
    W = int(rng.integers(2, 9))
    L = int(rng.integers(W - 1, 17))
    vec = seed % 4 != 3
    V = 8 if dtype == "bf16" else 4
    dim = V * int(rng.integers(1, 40)) if vec else int(rng.choice([1, 3, 13, 37]))
    lens = rng.integers(0, 300, size=int(rng.integers(1, 9)))
    d = workloads.dense_conv_inputs(
        700 + seed, dtype=dtype, dim=dim, W=W, state_len=L, lens=lens,
        num_pad=int(rng.integers(0, 2)) if len(lens) > 1 else 0, bias=bool(seed % 3),
        x_layout="channel_major" if seed % 5 == 4 else "token_major",
        state_layout="c_contig" if seed % 2 else "k_contig")
    assert _run_fwd(d, dtype, silu=bool(seed % 2), in_place=seed % 3 != 1,
                    with_states=seed % 7 != 6) == 0


@pytest.mark.parametrize("W", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fwd_channel_major(W, dtype):
    """Channel-major x (token stride 1): the warp-per-channel kernel over
    sequences longer than its 4 x 128-token load window, starts that are and
    are not multiples of the 4-token vector, every line length from W-1."""
    rng = np.random.default_rng(40 + W)
    lens = np.concatenate([rng.integers(0, 1200, size=5), [1, 2, 129, 512, 513]])
    L = int(rng.integers(W - 1, 17))
    d = workloads.dense_conv_inputs(1000 + W, dtype=dtype, dim=37, W=W, state_len=L,
                                    lens=lens, num_pad=1, x_layout="channel_major",
                                    state_layout="c_contig" if W % 2 else "k_contig")
    assert _run_fwd(d, dtype, silu=W != 5, in_place=W != 3) == 0


def test_fwd_in_place_equals_out_of_place():
    d = workloads.dense_conv_inputs(801, dtype="bf16", dim=256, W=4, state_len=3,
                                    lens=[700, 3, 0, 129])
    a = _to(d, DEV)
    b = _to(d, DEV)
    b["conv_states"] = a["conv_states"].clone()
    out = torch.empty_like(a["x"])
    hs().sconv_causal_conv1d_fwd(a["x"], a["weight"], a["bias"], a["conv_states"],
                                 a["query_start_loc"], a["cache_indices"],
                                 a["has_initial_state"], True)
    hs().sconv_causal_conv1d_fwd(b["x"], b["weight"], b["bias"], b["conv_states"],
                                 b["query_start_loc"], b["cache_indices"],
                                 b["has_initial_state"], True, out=out)
    torch.cuda.synchronize()
    assert torch.equal(raw(a["x"]), raw(out))
    assert torch.equal(raw(a["conv_states"]), raw(b["conv_states"]))


def test_fwd_tile_and_generic_agree_bitwise():
    """The same values in token-major (tiled kernel) and channel-major
    (any-layout kernel) storage give the same bits: both sum oldest tap
    first from the bias."""
    d = workloads.dense_conv_inputs(802, dtype="bf16", dim=64, W=4, state_len=5,
                                    lens=[300, 17, 1], has_init=[1, 0, 1])
    tok = _to(d, DEV)
    chm = _to(d, DEV)
    chm["x"] = d["x"].t().contiguous().to(DEV).t()
    chm["conv_states"] = tok["conv_states"].clone()
    for g in (tok, chm):
        hs().sconv_causal_conv1d_fwd(g["x"], g["weight"], g["bias"], g["conv_states"],
                                     g["query_start_loc"], g["cache_indices"],
                                     g["has_initial_state"], True)
    torch.cuda.synchronize()
    assert torch.equal(raw(tok["x"].contiguous()), raw(chm["x"].contiguous()))
    assert torch.equal(raw(tok["conv_states"]), raw(chm["conv_states"]))


def test_fwd_bad_line_and_query_start_set_flags():
    d = workloads.dense_conv_inputs(803, dtype="f32", dim=16, W=3, state_len=2,
                                    lens=[5, 6, 7], num_lines=4)
    d["cache_indices"] = torch.tensor([2, 9, 0], dtype=torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert _run_fwd(d, "f32", silu=False, err=err) == 1
    assert int(err.item()) == hs().EFLAG_SLOT
    g = _to(d, DEV)
    g["query_start_loc"] = torch.tensor([0, 5, 4, 19], dtype=torch.int32, device=DEV)
    err.zero_()
    before = g["x"].clone()
    hs().sconv_causal_conv1d_fwd(g["x"], g["weight"], g["bias"], g["conv_states"],
                                 g["query_start_loc"], None, None, False, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == hs().EFLAG_QUERY_START
    assert torch.equal(raw(g["x"][5:]), raw(before[5:]))


def test_fwd_graph_replay():
    d = workloads.dense_conv_inputs(804, dtype="bf16", dim=512, W=4, state_len=3,
                                    lens=[40, 300, 5])
    g = _to(d, DEV)
    x0, s0 = g["x"].clone(), g["conv_states"].clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        hs().sconv_causal_conv1d_fwd(g["x"], g["weight"], g["bias"], g["conv_states"],
                                     g["query_start_loc"], g["cache_indices"],
                                     g["has_initial_state"], True)
    torch.cuda.current_stream().wait_stream(s)
    eager_x, eager_s = g["x"].clone(), g["conv_states"].clone()
    graph = torch.cuda.CUDAGraph()
    g["x"].copy_(x0)
    g["conv_states"].copy_(s0)
    with torch.cuda.graph(graph):
        hs().sconv_causal_conv1d_fwd(g["x"], g["weight"], g["bias"], g["conv_states"],
                                     g["query_start_loc"], g["cache_indices"],
                                     g["has_initial_state"], True)
    g["x"].copy_(x0)
    g["conv_states"].copy_(s0)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(raw(g["x"]), raw(eager_x))
    assert torch.equal(raw(g["conv_states"]), raw(eager_s))
    del graph


# --------------------------------------------------------------------------
# decode update

def _run_update(u, dtype, silu, *, in_place=True, err=None):
    g = _to(u, DEV)
    if not u["conv_state"].is_contiguous():
        g["conv_state"] = u["conv_state"].transpose(1, 2).contiguous().to(DEV).transpose(1, 2)
    out = None if in_place else workloads.sentinel(tuple(g["x"].shape), dtype, DEV)
    res = hs().sconv_causal_conv1d_update(
        g["x"], g["conv_state"], g["weight"], g["bias"], silu, g["cache_seqlens"],
        g["conv_state_indices"], u["pad_slot_id"], out=out, err_flag=err)
    torch.cuda.synchronize()
    ref, rs, st_ref, sk = oracle.conv1d_update(
        dtype=dtype, x=u["x"], conv_state=u["conv_state"], weight=u["weight"], bias=u["bias"],
        activation="silu" if silu else None, cache_seqlens=u["cache_seqlens"],
        conv_state_indices=u["conv_state_indices"], pad_slot_id=u["pad_slot_id"])
    got = res.cpu()
    rows = rs == 1
    assert_close(oracle.to_f64(got, dtype)[rows], ref[rows], dtype, "dense update out")
    untouched = torch.from_numpy(~rows)
    want = raw(u["x"])[untouched] if in_place else torch.full_like(raw(got)[untouched], -1)
    assert torch.equal(raw(got)[untouched], want)
    np.testing.assert_array_equal(_bits(g["conv_state"], dtype), st_ref.view(np.uint8))
    return sk


@pytest.mark.parametrize("seed", range(16))
def test_update_random(seed):
    rng = np.random.default_rng(900 + seed)
    dtype = ["bf16", "f32"][seed % 2]
    W = int(rng.integers(2, 9))
    L = int(rng.integers(W - 1, 17))
    V = 8 if dtype == "bf16" else 4
    dim = V * int(rng.integers(1, 200)) if seed % 4 != 3 else int(rng.choice([1, 5, 33]))
    u = workloads.dense_update_inputs(900 + seed, dtype=dtype, batch=int(rng.integers(1, 300)),
                                      dim=dim, W=W, state_len=L, num_pad=int(seed % 3 == 0),
                                      ring=bool(seed % 2 == 0), bias=bool(seed % 5),
                                      state_layout="c_contig" if seed % 3 == 2 else "k_contig")
    assert _run_update(u, dtype, silu=bool(seed % 2), in_place=seed % 4 != 1) == 0


def test_update_bad_line_sets_flag():
    u = workloads.dense_update_inputs(950, dtype="bf16", batch=6, dim=64, W=4, state_len=3,
                                      num_lines=8)
    u["conv_state_indices"] = torch.tensor([0, 1, 8, -5, 4, 5], dtype=torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert _run_update(u, "bf16", True, err=err) == 2
    assert int(err.item()) == hs().EFLAG_SLOT


def test_prefill_then_decode_chain():
    """A prefill followed by three decode updates on the same lines equals
    the oracle's chain and the one-shot prefill of all the tokens."""
    rng = np.random.default_rng(960)
    lens = rng.integers(1, 50, size=6)
    d = workloads.dense_conv_inputs(960, dtype="bf16", dim=128, W=4, state_len=3,
                                    lens=lens + 3, has_init=np.zeros(6, bool), bias=True)
    qsl = d["query_start_loc"].numpy()
    pre = np.concatenate([np.arange(qsl[b], qsl[b] + lens[b]) for b in range(6)])
    g = _to(d, DEV)
    x_pre = g["x"][torch.from_numpy(pre).to(DEV)].contiguous()
    q_pre = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).to(DEV)
    hs().sconv_causal_conv1d_fwd(x_pre, g["weight"], g["bias"], g["conv_states"], q_pre,
                                 g["cache_indices"], g["has_initial_state"], True)
    outs = [x_pre]
    for step in range(3):
        rows = torch.from_numpy(qsl[:-1] + lens + step).to(DEV)
        xs = g["x"][rows].contiguous()
        hs().sconv_causal_conv1d_update(xs, g["conv_states"], g["weight"], g["bias"], True,
                                        None, g["cache_indices"])
        outs.append(xs)
    torch.cuda.synchronize()
    ref, _, st_ref, _ = oracle.conv1d_fwd(
        dtype="bf16", x=d["x"], weight=d["weight"], bias=d["bias"], conv_states=d["conv_states"],
        query_start_loc=d["query_start_loc"], cache_indices=d["cache_indices"],
        has_initial_state=d["has_initial_state"], activation="silu")
    assert_close(oracle.to_f64(outs[0].cpu(), "bf16"), ref[pre], "bf16", "chain prefill")
    for step in range(3):
        assert_close(oracle.to_f64(outs[step + 1].cpu(), "bf16"),
                     ref[qsl[:-1] + lens + step], "bf16", f"chain decode {step}")
    np.testing.assert_array_equal(_bits(g["conv_states"], "bf16"), st_ref.view(np.uint8))


# --------------------------------------------------------------------------
# benchmark sizes, checked on channel slices (the convolution is depthwise:
# channel c of the result depends on channel c of the inputs only)

def _slice_check(d, dtype, silu, chans, x_before, states_before, got_x, got_states):
    for c0, c1 in chans:
        ref, rs, st_ref, _ = oracle.conv1d_fwd(
            dtype=dtype, x=x_before[:, c0:c1], weight=d["weight"][c0:c1].cpu(),
            bias=None if d["bias"] is None else d["bias"][c0:c1].cpu(),
            conv_states=states_before[:, c0:c1], query_start_loc=d["query_start_loc"].cpu(),
            cache_indices=d["cache_indices"].cpu(),
            has_initial_state=d["has_initial_state"].cpu(), activation="silu" if silu else None,
            pad_slot_id=d["pad_slot_id"])
        rows = rs == 1
        assert_close(oracle.to_f64(got_x[:, c0:c1], dtype)[rows], ref[rows], dtype,
                     f"channels {c0}:{c1}")
        np.testing.assert_array_equal(
            oracle._float_array(got_states[:, c0:c1].contiguous(), dtype).view(np.uint8),
            st_ref.view(np.uint8))


@pytest.mark.parametrize("name", ["dense_prefill_bf16", "dense_long_prefill_bf16"])
def test_benchmark_sizes_on_channel_slices(name):
    d = workloads.DENSE_NAMED[name](device=DEV)
    x_before = d["x"].cpu()
    states_before = d["conv_states"].cpu()
    hs().sconv_causal_conv1d_fwd(d["x"], d["weight"], d["bias"], d["conv_states"],
                                 d["query_start_loc"], d["cache_indices"],
                                 d["has_initial_state"], True)
    torch.cuda.synchronize()
    dim = d["x"].shape[1]
    chans = [(0, 24), (dim // 2 - 8, dim // 2 + 24), (dim - 40, dim)]
    _slice_check(d, "bf16", True, chans, x_before, states_before, d["x"].cpu(),
                 d["conv_states"].cpu())


def test_decode_benchmark_size_full():
    """The benchmark's decode update (256 sequences, dim 1024, L 3) against
    the oracle element by element, lines bit-exact."""
    u = workloads.dense_decode_bf16()
    assert _run_update(u, "bf16", silu=True) == 0
