"""The benchmark's pipelined decode steps compute exactly what the plain
sequence of steps computes.

Pipelining builds step i+1's metadata (sconv_seq_metadata, or
sconv_seq_metadata_taps with the tap table, "vllm.models.inkling.nvidia.ops.sconv")
beside step i's convolution: on a second stream joined by an event
("side"), or enqueued ahead of it on the same stream ("interleaved", where
the convolution then reads its table before its wait).  The convolutions
keep their order, since step i+1 reads as history what step i inserted.
Several batches share one paged cache here, so any reordering of the
convolutions or a metadata buffer read before it is complete would change
the bits.  Each case also runs with the *_ahead builders, whose lookup
runs before their wait on the stream and whose completion must still
follow the previous convolution's.
"""
from __future__ import annotations

import pytest
import torch

import bench
from tests._gpu import raw

pytestmark = pytest.mark.gpu


def _snapshot(sets_obj):
    return raw(sets_obj.cache).clone(), [raw(s["out"]).clone() for s in sets_obj.sets]


def _reset(sets_obj, cache0):
    raw(sets_obj.cache).copy_(cache0)
    for s in sets_obj.sets:
        raw(s["out"]).fill_(-1)
        s["seq_idx"].fill_(-7)
        s["query_start"].fill_(-7)
        s["taps"].fill_(-7)


@pytest.mark.parametrize("mode", ["taps", "paged"])
@pytest.mark.parametrize("ahead", [False, True])
@pytest.mark.parametrize("n", [1, 2, 6])
def test_pipelined_steps_equal_plain_steps(n, ahead, mode):
    dev = torch.device("cuda", 0)
    sets_obj = bench.DecodeSets(n, 5151, dev, max_hist=64, mode=mode)
    cache0 = raw(sets_obj.cache).clone()

    _reset(sets_obj, cache0)
    for i in range(n):
        sets_obj.step(i)
        torch.cuda.synchronize()  # fully ordered reference
    plain_cache, plain_outs = _snapshot(sets_obj)

    # back to back on one stream, with the chosen metadata builder
    sets_obj.ahead = ahead
    _reset(sets_obj, cache0)
    for i in range(n):
        sets_obj.step(i)
    torch.cuda.synchronize()
    cache, outs = _snapshot(sets_obj)
    assert torch.equal(cache, plain_cache)
    for a, b in zip(outs, plain_outs):
        assert torch.equal(a, b)

    side = torch.cuda.Stream(dev)
    _reset(sets_obj, cache0)
    bench.pipelined_steps(sets_obj, list(range(n)), side)
    torch.cuda.synchronize()
    cache, outs = _snapshot(sets_obj)
    assert torch.equal(cache, plain_cache)
    for a, b in zip(outs, plain_outs):
        assert torch.equal(a, b)

    _reset(sets_obj, cache0)
    bench.interleaved_steps(sets_obj, list(range(n)))
    torch.cuda.synchronize()
    cache, outs = _snapshot(sets_obj)
    assert torch.equal(cache, plain_cache)
    for a, b in zip(outs, plain_outs):
        assert torch.equal(a, b)

    # the same from the benchmark's graphs, replayed twice; with carry the
    # first step's metadata comes from the prologue and the graph's last
    # build is for the step after it
    stream = torch.cuda.Stream(dev)
    for schedule, carry in (("side", False), ("interleaved", False), ("side", True)):
        _reset(sets_obj, cache0)
        if carry:
            bench.carry_prologue(sets_obj, stream)
        full, tail, reps = bench.run_steps_graphs(sets_obj, n, stream, pipeline=schedule,
                                                  carry=carry)
        for _ in range(2):
            _reset(sets_obj, cache0)
            if carry:
                bench.carry_prologue(sets_obj, stream)
            with torch.cuda.stream(stream):
                bench.replay_steps(full, tail, reps)
            torch.cuda.synchronize()
            cache, outs = _snapshot(sets_obj)
            assert torch.equal(cache, plain_cache), schedule
            for a, b in zip(outs, plain_outs):
                assert torch.equal(a, b), schedule
        del full, tail
