"""GPU parity of sconv_fused_streams: several conv streams of one layer
(disjoint lane ranges of one cache, shared tokens and metadata) in one
call, against one sconv_fused per stream (bit for bit) and the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import assert_close, hs, raw

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _streams(wl, t, specs, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    out = []
    for off_s, ws, act, res in specs:
        C = wl.H * ws
        out.append(dict(
            x=torch.randn(wl.T, C, generator=g).to(t["x"].dtype).to(DEV),
            weight=(torch.randn(C, wl.W, generator=g) * 0.5).to(t["x"].dtype).to(DEV),
            off_s=off_s, ws=ws, activation=act, use_residual=res))
    return out


def _check(wl, specs, seed):
    t = wl.tensors(DEV)
    streams = _streams(wl, t, specs, seed)
    cache0 = t["cache"].clone()
    md = {k: t[k] for k in ("positions", "block_table", "seq_idx", "slot_mapping", "query_start")}
    for sd in streams:
        sd["out"] = workloads.sentinel((wl.T, wl.H * sd["ws"]), wl.dtype, DEV)
    hs().sconv_fused_streams(streams, t["cache"], block_size=wl.N, **md)
    torch.cuda.synchronize()
    cache_multi = t["cache"].clone()
    # one sconv_fused per stream on the same starting cache
    t["cache"].copy_(cache0)
    for sd in streams:
        single = workloads.sentinel((wl.T, wl.H * sd["ws"]), wl.dtype, DEV)
        hs().sconv_fused(sd["x"], sd["weight"], t["cache"], off_s=sd["off_s"], ws=sd["ws"],
                         block_size=wl.N, activation=sd["activation"],
                         use_residual=sd["use_residual"], out=single, **md)
        torch.cuda.synchronize()
        assert torch.equal(raw(single), raw(sd["out"]))
    assert torch.equal(raw(t["cache"]), raw(cache_multi))
    # against the oracle
    mdc = wl.metadata("cpu")
    cpu_streams = [dict(sd, x=sd["x"].cpu(), weight=sd["weight"].cpu()) for sd in streams]
    outs, states, cache_ref, skipped = oracle.fused_streams(
        dtype=wl.dtype, streams=cpu_streams, cache=cache0.cpu(), block_size=wl.N,
        positions=mdc["positions"], block_table=mdc["block_table"], seq_idx=mdc["seq_idx"],
        slot_mapping=mdc["slot_mapping"], query_start=mdc["query_start"])
    assert skipped == 0
    for sd, ref, st in zip(streams, outs, states):
        got = sd["out"].cpu()
        rows = st == 1
        assert_close(oracle.to_f64(got, wl.dtype)[rows], ref[rows], wl.dtype, "stream out")
        assert bool((raw(got)[~torch.from_numpy(rows)] == -1).all())
    np.testing.assert_array_equal(oracle._float_array(cache_multi.cpu(), wl.dtype), cache_ref)


KV = [(0, 32, "silu", True), (32, 32, "silu", True)]
FOUR = [(0, 32, "silu", True), (32, 32, None, False), (64, 32, "silu", False), (96, 32, None, True)]


@pytest.mark.parametrize("specs", [KV, FOUR], ids=["two", "four"])
def test_decode_sizes_one_launch(specs):
    wl = workloads.decode_bf16(seed=90, R=64, max_hist=500)
    _check(wl, specs, 1)


def test_spec_decode_with_pad_rows():
    wl = workloads.spec_decode_bf16(seed=91, R=32, max_hist=300)
    wl_kv = workloads.build("spec_kv", dtype="bf16", H=16, D=128, ws=64, off_s=0, W=4, N=16,
                            hist=wl.hist, new=wl.new, act="silu", residual=True, seed=91,
                            num_pad=13)
    _check(wl_kv, [(0, 64, "silu", True), (64, 64, "silu", False)], 2)


def test_prefill_sizes_per_stream_launches():
    rng = np.random.default_rng(92)
    wl = workloads.build("prefill_kv", dtype="bf16", H=16, D=256, ws=128, off_s=0, W=4, N=16,
                         hist=rng.integers(0, 40, size=3), new=rng.integers(900, 1400, size=3),
                         act="silu", residual=False, seed=92, num_pad=3, rng=rng)
    _check(wl, [(0, 128, "silu", False), (128, 128, "silu", True)], 3)


def test_mixed_widths_and_element_path():
    """Streams of different widths, one of them not 16-byte aligned (ws=5):
    every stream takes the element path in the shared launch."""
    rng = np.random.default_rng(93)
    wl = workloads.build("mixed", dtype="f32", H=4, D=48, ws=8, off_s=0, W=3, N=8,
                         hist=rng.integers(0, 20, size=4), new=rng.integers(1, 30, size=4),
                         act="silu", residual=True, seed=93, num_pad=4, rng=rng)
    _check(wl, [(0, 8, "silu", True), (8, 5, None, True), (16, 32, "silu", False)], 4)
