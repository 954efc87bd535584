"""A decode step through a stack of layers, launched back to back with
programmatic dependent launch: one sconv_seq_metadata, then one sconv_fused
per layer (each its own cache and weight), layer l+1 convolving layer l's
output.  Every launch becomes resident while its predecessor runs and may
prefetch before it waits ("vllm.models.inkling.nvidia.ops.sconv": the
fused_sconv step, repeated per layer), so this checks that nothing a kernel
computes with is read before the wait: each layer against the oracle on the
input that layer actually received, bit-exact caches, and identical bits
when every launch instead waits for its predecessor to finish (layers
alternating between two streams) and when the chain replays from a graph.
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


def _layers(wl, t, n_layers, seed):
    g = torch.Generator().manual_seed(seed)
    dt = workloads.TORCH_DTYPE[wl.dtype]
    layers = []
    for _ in range(n_layers):
        cache = workloads.normal(tuple(t["cache"].shape), 1.0, dt, g, "cpu")
        weight = workloads.normal((wl.C, wl.W), 0.5, dt, g, "cpu")
        layers.append((cache, weight))
    return layers


def _run_chain(wl, t, layers_cpu, pdl):
    caches = [c.to(DEV) for c, _ in layers_cpu]
    weights = [w.to(DEV) for _, w in layers_cpu]
    # PAD rows are never written; zeros make the next layer's input defined.
    outs = [torch.zeros_like(t["x"]) for _ in layers_cpu]
    qsl = torch.from_numpy(wl.query_start_loc).to(DEV)
    seq_idx = torch.empty(wl.T, dtype=torch.int32, device=DEV)
    query_start = torch.empty(wl.T, dtype=torch.int32, device=DEV)
    side = torch.cuda.Stream()

    def step():
        main = torch.cuda.current_stream()  # the capture stream when captured
        hs().sconv_seq_metadata(qsl, wl.R, wl.T, seq_idx, query_start)
        x, cur = t["x"], main
        for l in range(len(layers_cpu)):
            target = main if (pdl or l % 2 == 0) else side
            if target is not cur:
                ev = torch.cuda.Event()
                ev.record(cur)
                target.wait_event(ev)
            with torch.cuda.stream(target):
                hs().sconv_fused(x, weights[l], caches[l], t["positions"], t["block_table"],
                                 seq_idx, t["slot_mapping"], query_start, out=outs[l],
                                 **wl.kwargs())
            cur, x = target, outs[l]
        if cur is not main:
            ev = torch.cuda.Event()
            ev.record(cur)
            main.wait_event(ev)

    return step, caches, outs


@pytest.mark.parametrize("seed", range(4))
def test_chain_matches_oracle_layer_by_layer(seed):
    wl = workloads.random_case(600 + seed, dtype="bf16", vec_friendly=True, max_hist=40,
                               pad_frac=0.1)
    t = wl.tensors(DEV)
    layers_cpu = _layers(wl, t, 4, seed)
    step, caches, outs = _run_chain(wl, t, layers_cpu, pdl=True)
    step()
    torch.cuda.synchronize()
    md = wl.metadata("cpu")
    x = t["x"].cpu()
    for l, (cache0, weight) in enumerate(layers_cpu):
        ref, state, cache_ref, skipped = oracle.fused(
            dtype=wl.dtype, x=x, weight=weight, cache=cache0, positions=md["positions"],
            block_table=md["block_table"], seq_idx=md["seq_idx"],
            slot_mapping=md["slot_mapping"], query_start=md["query_start"], **wl.kwargs())
        assert skipped == 0
        got = outs[l].cpu()
        rows = state == 1
        assert_close(oracle.to_f64(got, wl.dtype)[rows], ref[rows], wl.dtype, f"layer {l}")
        np.testing.assert_array_equal(oracle._float_array(caches[l].cpu(), wl.dtype), cache_ref,
                                      err_msg=f"layer {l} cache")
        x = got  # the input the next layer received


def test_chain_same_bits_serialised_and_from_a_graph():
    wl = workloads.decode_bf16(seed=1002, R=128, max_hist=128)
    t = wl.tensors(DEV)
    layers_cpu = _layers(wl, t, 4, 77)
    results = []
    for mode in ("pdl", "serialised", "graph"):
        step, caches, outs = _run_chain(wl, t, layers_cpu, pdl=mode != "serialised")
        if mode == "graph":
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                step()
            g.replay()
        else:
            step()
        torch.cuda.synchronize()
        results.append(([raw(o).cpu() for o in outs], [raw(c).cpu() for c in caches]))
        if mode == "graph":
            del g
    for outs, caches in results[1:]:
        for a, b in zip(outs, results[0][0]):
            assert torch.equal(a, b)
        for a, b in zip(caches, results[0][1]):
            assert torch.equal(a, b)
