"""GPU parity of the resolved-tap path through the C ABI: the per-step tap
table (sconv_seq_metadata_taps) against the oracle's resolution, bit for
bit, and the fused step that reads it (sconv_fused_taps) against the
oracle's fused step and, bit for bit, against sconv_fused on the metadata
the table was built from ("vllm.models.inkling.nvidia.ops.sconv", module
docstring and fused_sconv)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import (assert_close, check_full_size, check_small, hs, oracle_fused, raw,
                        run_fused)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def resolve(wl, t, *, decode_form=False, ahead=False, num_padded=None, with_metadata=True):
    """The GPU table (and, unless decode_form, seq_idx / query_start)."""
    npad = wl.T if num_padded is None else num_padded
    si = torch.full((npad,), -7, dtype=torch.int32, device=DEV) if with_metadata else None
    qs = torch.full((npad,), -7, dtype=torch.int32, device=DEV) if with_metadata else None
    fn = hs().sconv_seq_metadata_taps_ahead if ahead else hs().sconv_seq_metadata_taps
    taps = fn(None if decode_form else t["query_start_loc"],
              wl.block_table.shape[0] if decode_form else wl.R, wl.T, t["positions"],
              t["slot_mapping"], t["block_table"], wl.num_blocks, wl.N, wl.W,
              seq_idx_out=si, query_start_out=qs, num_padded_tokens=npad)
    return si, qs, taps


def oracle_resolve(wl, decode_form=False, num_padded=None, md=None):
    md = md or {k: v.numpy() for k, v in wl.metadata("cpu").items()}
    return oracle.resolve_taps(
        query_start_loc=None if decode_form else md["query_start_loc"],
        num_reqs=wl.block_table.shape[0] if decode_form else wl.R, num_actual_tokens=wl.T,
        num_padded_tokens=num_padded, positions=md["positions"],
        slot_mapping=md["slot_mapping"], block_table=md["block_table"],
        num_blocks=wl.num_blocks, block_size=wl.N, W=wl.W)


def run_taps(wl, t, out=None, err=None, ready=True, decode_form=False):
    """Table, then the fused step reading it.  With ready, the stream is
    ordered between the two (a host synchronisation), which is the
    precondition of reading the table before the launch's wait."""
    _, _, taps = resolve(wl, t, decode_form=decode_form, with_metadata=False)
    if ready:
        torch.cuda.synchronize()
    return hs().sconv_fused_taps(t["x"], t["weight"], t["cache"], t["slot_mapping"], taps,
                                 out=out, err_flag=err, metadata_ready=ready, **wl.kwargs())


@pytest.mark.parametrize("ahead", [False, True])
@pytest.mark.parametrize("seed", range(24))
def test_table_matches_oracle_random(seed, ahead):
    wl = workloads.random_case(seed)
    t = wl.tensors(DEV)
    npad = wl.T + 5
    si, qs, taps = resolve(wl, t, ahead=ahead, num_padded=npad)
    rsi, rqs, rtaps = oracle_resolve(wl, num_padded=npad)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(si.cpu().numpy(), rsi)
    np.testing.assert_array_equal(qs.cpu().numpy(), rqs)
    np.testing.assert_array_equal(taps.cpu().numpy(), rtaps)


@pytest.mark.parametrize("name", ["decode_bf16", "spec_decode_bf16", "chunked_prefill_bf16"])
def test_table_matches_oracle_named(name):
    wl = workloads.NAMED[name]()
    md = wl.metadata(DEV)
    si, qs, taps = resolve(wl, md)
    rsi, rqs, rtaps = oracle_resolve(wl)
    np.testing.assert_array_equal(si.cpu().numpy(), rsi)
    np.testing.assert_array_equal(qs.cpu().numpy(), rqs)
    np.testing.assert_array_equal(taps.cpu().numpy(), rtaps)


def test_table_decode_form():
    wl = workloads.decode_bf16(seed=31, R=200, max_hist=5000)
    md = wl.metadata(DEV)
    si, qs, taps = resolve(wl, md, decode_form=True)
    rsi, rqs, rtaps = oracle_resolve(wl, decode_form=True)
    np.testing.assert_array_equal(taps.cpu().numpy(), rtaps)
    np.testing.assert_array_equal(si.cpu().numpy(), np.arange(wl.T))
    np.testing.assert_array_equal(qs.cpu().numpy(), np.arange(wl.T))


def test_table_many_requests_unstaged():
    """More requests than the shared-memory stage holds: the search reads
    query_start_loc from global memory."""
    rng = np.random.default_rng(8)
    R = 5000
    wl = workloads.build("many", dtype="bf16", H=1, D=8, ws=8, off_s=0, W=4, N=16,
                         hist=rng.integers(0, 30, size=R), new=rng.integers(0, 3, size=R),
                         act=None, residual=False, seed=8, num_pad=50, rng=rng)
    md = wl.metadata(DEV)
    si, qs, taps = resolve(wl, md)
    rsi, rqs, rtaps = oracle_resolve(wl)
    np.testing.assert_array_equal(si.cpu().numpy(), rsi)
    np.testing.assert_array_equal(qs.cpu().numpy(), rqs)
    np.testing.assert_array_equal(taps.cpu().numpy(), rtaps)


@pytest.mark.parametrize("ready", [False, True])
@pytest.mark.parametrize("seed", range(24))
def test_fused_taps_random_small(seed, ready):
    """Outputs within tolerance of the oracle, cache and PAD rows bit-exact,
    and every byte equal to sconv_fused's on the same step."""
    wl = workloads.random_case(seed)
    t = wl.tensors(DEV)
    cache0 = t["cache"].clone()
    ref_out = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    run_fused(wl, t, out=ref_out)
    ref_cache = t["cache"].clone()
    t["cache"].copy_(cache0)
    out = check_small(wl, DEV, t=t, run=lambda wl_, t_, out: run_taps(wl_, t_, out=out,
                                                                      ready=ready))
    assert torch.equal(raw(out), raw(ref_out))
    assert torch.equal(raw(t["cache"]), raw(ref_cache))


@pytest.mark.parametrize("W", range(1, 9))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_taps_every_window_length(W, dtype):
    rng = np.random.default_rng(50 + W)
    wl = workloads.build(f"taps_w{W}", dtype=dtype, H=4, D=64, ws=32, off_s=16, W=W, N=4,
                         hist=rng.integers(0, 12, size=6), new=rng.integers(1, 30, size=6),
                         act="silu", residual=True, seed=W, num_pad=5, rng=rng)
    check_small(wl, DEV, run=lambda wl_, t_, out: run_taps(wl_, t_, out=out))


@pytest.mark.parametrize("name,decode_form", [("decode_bf16", False), ("decode_bf16", True),
                                              ("spec_decode_bf16", False),
                                              ("chunked_prefill_bf16", False)])
def test_fused_taps_full_size(name, decode_form):
    """The decode, speculative-decode and chunked-prefill workloads at full
    size (decode caches of 4.2 / 2.1 GB, element offsets past 2^31; the
    prefill through the TMA-pipelined form): sampled tokens against the
    oracle, inserts element by element, the whole cache by the holds-x
    invariant, PAD rows untouched."""
    wl = workloads.NAMED[name]()
    check_full_size(wl, DEV, run=lambda wl_, t_, out, err: run_taps(
        wl_, t_, out=out, err=err, decode_form=decode_form))


def _tiled_case(W, dtype, seed, num_pad=9, residual=True):
    """A step large enough for the TMA-pipelined form (T x C/VEC >= 2^19):
    six requests, some with long cached prefixes, some with none, and PAD
    rows; C = 4096."""
    rng = np.random.default_rng(seed)
    T_min = 1100 if dtype == "bf16" else 600
    new = rng.integers(T_min // 5, T_min // 3, size=6)  # T >= 1.2 T_min
    hist = np.array([0, 3, 700, 1, 0, 2000])
    return workloads.build(f"tiled_taps_w{W}_{dtype}", dtype=dtype, H=32, D=128, ws=128,
                           off_s=0, W=W, N=16, hist=hist, new=new, act="silu",
                           residual=residual, seed=seed, num_pad=num_pad, rng=rng)


@pytest.mark.parametrize("W", range(1, 9))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_taps_tiled_every_window_length(W, dtype):
    """At prefill sizes the resolved-tap form runs the TMA-pipelined kernel
    (the table rows travel with the tile): every output row and cache byte
    against the oracle, PAD rows untouched, and every byte equal to
    sconv_fused's on the same step."""
    wl = _tiled_case(W, dtype, 900 + 10 * W + (dtype == "f32"), residual=W % 2 == 0)
    assert wl.T * wl.C // (8 if dtype == "bf16" else 4) >= 1 << 19
    t = wl.tensors(DEV)
    cache0 = t["cache"].clone()
    ref_out = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    run_fused(wl, t, out=ref_out)
    ref_cache = t["cache"].clone()
    t["cache"].copy_(cache0)
    out = check_small(wl, DEV, t=t, run=lambda wl_, t_, out: run_taps(wl_, t_, out=out))
    assert torch.equal(raw(out), raw(ref_out))
    assert torch.equal(raw(t["cache"]), raw(ref_cache))


def test_fused_taps_tiled_foreign_entries_are_checked():
    """The TMA-pipelined resolved-tap form checks a table not made by the
    resolver as the token form does: the tokens with an entry past the
    cache, a bad code or an x row before the call are skipped with
    SCONV_EFLAG_BLOCK / SCONV_EFLAG_QUERY_START, a token carrying the
    resolver's failure code reports its bits, and nothing else changes."""
    wl = _tiled_case(4, "bf16", 950, num_pad=0)
    t = wl.tensors(DEV)
    _, _, taps = resolve(wl, t)
    torch.cuda.synchronize()
    good = taps.clone()
    taps[5, 0] = wl.num_blocks * wl.N          # slot past the cache
    taps[37, 1] = -7                           # not a code
    taps[0, 2] = hs().TAP_X                    # x row -3 of this call
    taps[600, :] = -(0x04 * 256)               # the resolver's LOGICAL failure
    out = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    cache0 = t["cache"].clone()
    hs().sconv_fused_taps(t["x"], t["weight"], t["cache"], t["slot_mapping"], taps, out=out,
                          err_flag=err, **wl.kwargs())
    torch.cuda.synchronize()
    assert int(err.item()) == 0x04 | 0x08 | 0x10
    bad_rows = [0, 5, 37, 600]
    assert bool((raw(out)[bad_rows] == -1).all())
    ref = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    c2 = cache0.clone()
    hs().sconv_fused_taps(t["x"], t["weight"], c2, t["slot_mapping"], good, out=ref,
                          **wl.kwargs())
    torch.cuda.synchronize()
    keep = torch.ones(wl.T, dtype=torch.bool)
    keep[bad_rows] = False
    assert torch.equal(raw(out)[keep.to(DEV)], raw(ref)[keep.to(DEV)])


def test_fused_taps_equals_update_on_decode_form():
    wl = workloads.decode_bf16(seed=77, R=64, max_hist=300)
    t = wl.tensors(DEV)
    cache0 = t["cache"].clone()
    out_u = hs().sconv_update(t["x"], t["weight"], t["cache"], t["positions"],
                              t["block_table"], t["slot_mapping"], **wl.kwargs())
    cache_u = t["cache"].clone()
    t["cache"].copy_(cache0)
    out_t = run_taps(wl, t, decode_form=True)
    torch.cuda.synchronize()
    assert torch.equal(raw(out_u), raw(out_t))
    assert torch.equal(raw(cache_u), raw(t["cache"]))


def test_two_streams_equal_streams_call():
    """Two conv streams of a layer through one table equal
    sconv_fused_streams bit for bit, and the oracle within tolerance."""
    wl = workloads.decode_bf16(seed=90, R=96, max_hist=700)
    t = wl.tensors(DEV)
    g = torch.Generator(device="cpu").manual_seed(3)
    x2 = workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, "cpu").to(DEV)
    w2 = workloads.normal((wl.C, wl.W), 0.5, torch.bfloat16, g, "cpu").to(DEV)

    def streams():
        return [dict(x=t["x"], weight=t["weight"], off_s=wl.off_s, ws=wl.ws, activation="silu",
                     use_residual=True),
                dict(x=x2, weight=w2, off_s=0, ws=wl.ws, activation=None, use_residual=False)]
    cache0 = t["cache"].clone()
    ref = hs().sconv_fused_streams(streams(), t["cache"], t["positions"], t["block_table"],
                                   t["seq_idx"], t["slot_mapping"], t["query_start"], wl.N)
    ref_cache = t["cache"].clone()
    t["cache"].copy_(cache0)
    _, _, taps = resolve(wl, t)
    torch.cuda.synchronize()
    got = hs().sconv_fused_streams_taps(streams(), t["cache"], t["slot_mapping"], taps, wl.N,
                                        metadata_ready=True)
    torch.cuda.synchronize()
    for a, b in zip(ref, got):
        assert torch.equal(raw(a), raw(b))
    assert torch.equal(raw(ref_cache), raw(t["cache"]))
    md = wl.metadata("cpu")
    outs, states, cache_ref, skipped = oracle.fused_streams(
        dtype="bf16", streams=[dict(s, x=s["x"].cpu(), weight=s["weight"].cpu())
                               for s in streams()],
        cache=cache0.cpu(), positions=md["positions"], block_table=md["block_table"],
        seq_idx=md["seq_idx"], slot_mapping=md["slot_mapping"], query_start=md["query_start"],
        block_size=wl.N)
    assert skipped == 0
    for o, r, state in zip(got, outs, states):
        rows = state == 1
        assert_close(oracle.to_f64(o.cpu(), "bf16")[rows], r[rows], "bf16", "stream")
    np.testing.assert_array_equal(oracle._float_array(t["cache"].cpu(), "bf16"), cache_ref)


def _err_case():
    rng = np.random.default_rng(40)
    return workloads.build("err", dtype="bf16", H=4, D=32, ws=32, off_s=0, W=4, N=8,
                           hist=np.array([5, 20, 0, 9]), new=np.array([6, 1, 7, 2]),
                           act="silu", residual=True, seed=40, rng=rng)


@pytest.mark.parametrize("kind,flag", [
    ("slot", 0x01), ("logical", 0x04), ("block", 0x08), ("query_start", 0x10),
    ("position", 0x20)])
def test_bad_index_flags_equal_fused(kind, flag):
    """Each bad index skips its token and sets the bits sconv_fused sets;
    the table row carries them (bit-exact against the oracle's)."""
    wl = _err_case()
    t = wl.tensors(DEV)
    md = {k: v.clone() for k, v in wl.metadata("cpu").items()}
    row = int(wl.query_start_loc[1])
    if kind == "slot":
        md["slot_mapping"][row] = wl.num_blocks * wl.N + 3
    elif kind == "logical":
        md["positions"][row] += wl.block_table.shape[1] * wl.N
    elif kind == "block":
        md["block_table"][1, (int(wl.positions[row]) - 1) // wl.N] = wl.num_blocks + 7
    elif kind == "query_start":
        md["query_start_loc"][0] = row + 1          # rows before it start after themselves
    elif kind == "position":
        md["positions"][row] = -3
    td = dict(t, **{k: v.to(DEV) for k, v in md.items()})
    cache0 = t["cache"].clone()
    _, _, taps = resolve(wl, td)
    rtaps = oracle_resolve(wl, md={k: v.numpy() for k, v in md.items()})[2]
    np.testing.assert_array_equal(taps.cpu().numpy(), rtaps)
    torch.cuda.synchronize()
    out = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    hs().sconv_fused_taps(td["x"], td["weight"], td["cache"], td["slot_mapping"], taps,
                          out=out, err_flag=err, metadata_ready=True, **wl.kwargs())
    torch.cuda.synchronize()
    assert int(err.item()) == flag
    # the same step through sconv_fused, on the metadata the table came from
    si, qs = oracle.seq_metadata(md["query_start_loc"], wl.R, wl.T)
    cache_t = td["cache"].clone()
    td["cache"].copy_(cache0)
    out_f = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    err_f = torch.zeros(1, dtype=torch.int32, device=DEV)
    run_fused(wl, dict(td, seq_idx=torch.from_numpy(si).to(DEV),
                       query_start=torch.from_numpy(qs).to(DEV)), out=out_f, err=err_f)
    torch.cuda.synchronize()
    assert int(err_f.item()) == flag
    assert torch.equal(raw(out), raw(out_f))
    assert torch.equal(raw(cache_t), raw(td["cache"]))


def test_foreign_table_entries_are_checked():
    """A table not made by the resolver (entries out of range, a bad code,
    an x row before the call) skips those tokens with SCONV_EFLAG_BLOCK /
    SCONV_EFLAG_QUERY_START and touches nothing else."""
    wl = workloads.decode_bf16(seed=12, R=8, max_hist=200)
    t = wl.tensors(DEV)
    _, _, taps = resolve(wl, t)
    torch.cuda.synchronize()
    good = taps.clone()
    taps[1, 0] = wl.num_blocks * wl.N          # slot past the cache
    taps[2, 1] = -7                            # not a code
    taps[0, 2] = hs().TAP_X                    # x row -3 of this call
    out = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    cache0 = t["cache"].clone()
    hs().sconv_fused_taps(t["x"], t["weight"], t["cache"], t["slot_mapping"], taps, out=out,
                          err_flag=err, **wl.kwargs())
    torch.cuda.synchronize()
    assert int(err.item()) == 0x08 | 0x10
    assert bool((raw(out)[:3] == -1).all())
    ref = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    c2 = cache0.clone()
    hs().sconv_fused_taps(t["x"], t["weight"], c2, t["slot_mapping"], good, out=ref,
                          **wl.kwargs())
    torch.cuda.synchronize()
    assert torch.equal(raw(out)[3:], raw(ref)[3:])


def test_interleaved_graph_equals_plain_steps():
    """The benchmark's step schedule: on one stream, each step's table is
    built (ahead of its wait) before the previous step's convolution, and
    every convolution but the first reads its table before its wait.
    Captured in a graph and replayed with every table and output reset
    first, the outputs and the cache equal the plain sequence of
    sconv_fused steps on the same shared cache, bit for bit."""
    wls = [workloads.decode_bf16(seed=500 + i, R=64, max_hist=600) for i in range(6)]
    nb = max(w.num_blocks for w in wls)
    w0 = wls[0]
    g = torch.Generator(device="cpu").manual_seed(4)
    cache = torch.empty((nb, w0.H, w0.N, w0.D), dtype=torch.bfloat16, device=DEV)
    workloads.fill_normal_(cache, 1.0, torch.Generator(device=DEV).manual_seed(4), DEV)
    weight = workloads.normal((w0.C, w0.W), 0.5, torch.bfloat16, g, "cpu").to(DEV)
    sets = []
    for wl in wls:
        md = wl.metadata(DEV)
        md["x"] = workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, "cpu").to(DEV)
        md["out"] = torch.empty_like(md["x"])
        md["taps"] = torch.empty((wl.T, wl.W - 1), dtype=torch.int64, device=DEV)
        sets.append(md)
    cache0 = cache.clone()
    ref = [hs().sconv_fused(s["x"], weight, cache, s["positions"], s["block_table"],
                            s["seq_idx"], s["slot_mapping"], s["query_start"], **wl.kwargs())
           for wl, s in zip(wls, sets)]      # the plain sequence of steps on one cache
    torch.cuda.synchronize()
    ref_cache = cache.clone()

    def build(i):
        wl, s = wls[i], sets[i]
        hs().sconv_seq_metadata_taps_ahead(s["query_start_loc"], wl.R, wl.T, s["positions"],
                                          s["slot_mapping"], s["block_table"], wl.num_blocks,
                                          wl.N, wl.W, taps_out=s["taps"])

    def steps():
        build(0)
        for i, (wl, s) in enumerate(zip(wls, sets)):
            if i + 1 < len(wls):
                build(i + 1)
            hs().sconv_fused_taps(s["x"], weight, cache, s["slot_mapping"], s["taps"],
                                  out=s["out"], metadata_ready=i > 0, **wl.kwargs())

    def reset():
        cache.copy_(cache0)
        for s in sets:
            s["out"].fill_(0)
            s["taps"].fill_(-7)

    main = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    reset()
    with torch.cuda.stream(main):
        steps()                 # eager, and warm-up
    torch.cuda.synchronize()
    for r, s in zip(ref, sets):
        assert torch.equal(raw(r), raw(s["out"]))
    assert torch.equal(raw(cache), raw(ref_cache))
    with torch.cuda.graph(graph, stream=main):
        steps()
    for _ in range(2):
        reset()
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        for r, s in zip(ref, sets):
            assert torch.equal(raw(r), raw(s["out"]))
        assert torch.equal(raw(cache), raw(ref_cache))
    del graph


def test_stale_table_rewritten_under_the_convolution():
    """Without metadata_ready the convolution reads its table row before its
    wait only as a guess, to prefetch the cache taps it names; the taps it
    uses follow the row read after the wait.  Each step's table here first
    holds ANOTHER step's table (valid cache slots, wrong ones), then the
    builder rewrites it and the convolution follows at once on the same
    stream, so its early reads may see either.  Replayed from a graph
    several times, outputs and cache equal the plain sconv_fused steps bit
    for bit."""
    wls = [workloads.decode_bf16(seed=520 + i, R=64, max_hist=600) for i in range(6)]
    nb = max(w.num_blocks for w in wls)
    w0 = wls[0]
    g = torch.Generator(device="cpu").manual_seed(5)
    cache = torch.empty((nb, w0.H, w0.N, w0.D), dtype=torch.bfloat16, device=DEV)
    workloads.fill_normal_(cache, 1.0, torch.Generator(device=DEV).manual_seed(5), DEV)
    weight = workloads.normal((w0.C, w0.W), 0.5, torch.bfloat16, g, "cpu").to(DEV)
    sets = []
    for wl in wls:
        md = wl.metadata(DEV)
        md["x"] = workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, "cpu").to(DEV)
        md["out"] = torch.empty_like(md["x"])
        md["taps"] = torch.empty((wl.T, wl.W - 1), dtype=torch.int64, device=DEV)
        sets.append(md)
    # Another step's real table for each step, all entries valid slots here.
    stale = []
    for i in range(len(wls)):
        j = (i + 1) % len(wls)
        _, _, tj = resolve(wls[j], sets[j], decode_form=True, with_metadata=False)
        stale.append(tj)
    assert all(s.shape == stale[0].shape for s in stale)
    cache0 = cache.clone()
    ref = [hs().sconv_fused(s["x"], weight, cache, s["positions"], s["block_table"],
                            s["seq_idx"], s["slot_mapping"], s["query_start"], **wl.kwargs())
           for wl, s in zip(wls, sets)]
    torch.cuda.synchronize()
    ref_cache = cache.clone()

    def steps():
        for i, (wl, s) in enumerate(zip(wls, sets)):
            s["taps"].copy_(stale[i])
            hs().sconv_seq_metadata_taps(None, wl.block_table.shape[0], wl.T, s["positions"],
                                        s["slot_mapping"], s["block_table"], wl.num_blocks,
                                        wl.N, wl.W, taps_out=s["taps"])
            hs().sconv_fused_taps(s["x"], weight, cache, s["slot_mapping"], s["taps"],
                                  out=s["out"], metadata_ready=False, **wl.kwargs())

    def check():
        for r, s in zip(ref, sets):
            assert torch.equal(raw(r), raw(s["out"]))
        assert torch.equal(raw(cache), raw(ref_cache))

    def reset():
        cache.copy_(cache0)
        for s in sets:
            s["out"].fill_(0)

    main = torch.cuda.Stream()
    reset()
    torch.cuda.synchronize()
    with torch.cuda.stream(main):
        steps()
    torch.cuda.synchronize()
    check()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=main):
        steps()
    for _ in range(8):
        reset()
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        check()
    del graph


def _next_dict(wl, md, taps_out, decode_form=False, si=None, qs=None):
    return dict(query_start_loc=None if decode_form else md["query_start_loc"],
                num_reqs=wl.block_table.shape[0] if decode_form else wl.R,
                num_actual_tokens=wl.T, positions=md["positions"],
                slot_mapping=md["slot_mapping"], block_table=md["block_table"],
                taps_out=taps_out, seq_idx_out=si, query_start_out=qs)


@pytest.mark.parametrize("decode_form", [False, True])
def test_fused_taps_next_one_call(decode_form):
    """One launch: this step's convolution (bit for bit sconv_fused_taps on
    the same table, and the oracle's step within tolerance) and the next
    step's table (bit for bit the oracle's resolution)."""
    a = workloads.decode_bf16(seed=41, R=96, max_hist=900)
    b = workloads.spec_decode_bf16(seed=42, max_hist=700) if not decode_form else \
        workloads.decode_bf16(seed=43, R=80, max_hist=500)
    ta = a.tensors(DEV)
    # one cache serves both steps: the next step's taps are resolved against it
    nb = max(a.num_blocks, b.num_blocks)
    big = torch.empty((nb, a.H, a.N, a.D), dtype=torch.bfloat16, device=DEV)
    workloads.fill_normal_(big, 1.0, torch.Generator(device=DEV).manual_seed(41), DEV)
    big[:a.num_blocks].copy_(ta["cache"])
    ta["cache"] = big
    mdb = b.metadata(DEV)
    _, _, taps_a = resolve(a, ta)
    torch.cuda.synchronize()
    cache0 = ta["cache"].clone()
    ref = hs().sconv_fused_taps(ta["x"], ta["weight"], ta["cache"], ta["slot_mapping"], taps_a,
                                **a.kwargs())
    torch.cuda.synchronize()
    ref_cache = ta["cache"].clone()
    ta["cache"].copy_(cache0)
    taps_b = torch.full((b.T, b.W - 1), -7, dtype=torch.int64, device=DEV)
    si = torch.full((b.T,), -7, dtype=torch.int32, device=DEV)
    qs = torch.full((b.T,), -7, dtype=torch.int32, device=DEV)
    out = hs().sconv_fused_taps_next(ta["x"], ta["weight"], ta["cache"], ta["slot_mapping"],
                                     taps_a, next_step=_next_dict(b, mdb, taps_b, decode_form,
                                                                  si, qs), **a.kwargs())
    torch.cuda.synchronize()
    assert torch.equal(raw(out), raw(ref))
    assert torch.equal(raw(ta["cache"]), raw(ref_cache))
    rsi, rqs, rtaps = oracle_resolve(b, decode_form=decode_form)
    np.testing.assert_array_equal(taps_b.cpu().numpy(), rtaps)
    np.testing.assert_array_equal(si.cpu().numpy(), rsi)
    np.testing.assert_array_equal(qs.cpu().numpy(), rqs)
    refo, state, _, _ = oracle_fused(a, ta["x"].cpu(), ta["weight"].cpu(), cache0.cpu(),
                                     a.metadata("cpu"), write_cache=False)
    rows = state == 1
    assert_close(oracle.to_f64(out.cpu(), "bf16")[rows], refo[rows], "bf16", "fused_taps_next")


def test_fused_taps_next_build_only():
    """T == 0: the launch only builds the next step's table."""
    b = workloads.decode_bf16(seed=44, R=33, max_hist=200)
    mdb = b.metadata(DEV)
    x = torch.empty((0, b.C), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((b.C, b.W), dtype=torch.bfloat16, device=DEV)
    cache = torch.zeros((b.num_blocks, b.H, b.N, b.D), dtype=torch.bfloat16, device=DEV)
    taps_b = torch.full((b.T, b.W - 1), -7, dtype=torch.int64, device=DEV)
    hs().sconv_fused_taps_next(x, w, cache, torch.empty(0, dtype=torch.int64, device=DEV), None,
                               next_step=_next_dict(b, mdb, taps_b), **b.kwargs())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(taps_b.cpu().numpy(), oracle_resolve(b)[2])


def test_fused_taps_next_loop_graph_equals_plain_steps():
    """A decode loop of one launch per step, each building the next step's
    table, captured in a graph and replayed with every table reset (the
    first from the standalone builder), equals the plain sequence of
    sconv_fused steps on one shared cache, bit for bit."""
    wls = [workloads.decode_bf16(seed=600 + i, R=64, max_hist=600) for i in range(6)]
    nb = max(w.num_blocks for w in wls)
    w0 = wls[0]
    g = torch.Generator(device="cpu").manual_seed(6)
    cache = torch.empty((nb, w0.H, w0.N, w0.D), dtype=torch.bfloat16, device=DEV)
    workloads.fill_normal_(cache, 1.0, torch.Generator(device=DEV).manual_seed(6), DEV)
    weight = workloads.normal((w0.C, w0.W), 0.5, torch.bfloat16, g, "cpu").to(DEV)
    sets = []
    for wl in wls:
        md = wl.metadata(DEV)
        md["x"] = workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, "cpu").to(DEV)
        md["out"] = torch.empty_like(md["x"])
        md["taps"] = torch.empty((wl.T, wl.W - 1), dtype=torch.int64, device=DEV)
        sets.append(md)
    cache0 = cache.clone()
    ref = [hs().sconv_fused(s["x"], weight, cache, s["positions"], s["block_table"],
                            s["seq_idx"], s["slot_mapping"], s["query_start"], **wl.kwargs())
           for wl, s in zip(wls, sets)]
    torch.cuda.synchronize()
    ref_cache = cache.clone()

    def steps():
        for i, (wl, s) in enumerate(zip(wls, sets)):
            j = (i + 1) % len(wls)
            hs().sconv_fused_taps_next(s["x"], weight, cache, s["slot_mapping"], s["taps"],
                                       out=s["out"],
                                       next_step=_next_dict(wls[j], sets[j], sets[j]["taps"]),
                                       **wl.kwargs())

    def reset():
        cache.copy_(cache0)
        for s in sets:
            s["out"].fill_(0)
            s["taps"].fill_(-7)
        wl, s = wls[0], sets[0]
        hs().sconv_seq_metadata_taps(s["query_start_loc"], wl.R, wl.T, s["positions"],
                                     s["slot_mapping"], s["block_table"], wl.num_blocks, wl.N,
                                     wl.W, taps_out=s["taps"])
        torch.cuda.synchronize()

    main = torch.cuda.Stream()
    reset()
    with torch.cuda.stream(main):
        steps()
    torch.cuda.synchronize()
    for r, s in zip(ref, sets):
        assert torch.equal(raw(r), raw(s["out"]))
    assert torch.equal(raw(cache), raw(ref_cache))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=main):
        steps()
    for _ in range(2):
        reset()
        graph.replay()
        torch.cuda.synchronize()
        for r, s in zip(ref, sets):
            assert torch.equal(raw(r), raw(s["out"]))
        assert torch.equal(raw(cache), raw(ref_cache))
    del graph
