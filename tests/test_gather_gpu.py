"""GPU parity of sconv_scatter_intermediate_ssm and sconv_extract_windows_paged
against the CPU oracle, bit for bit ("core.ssm.ops.intermediate_extraction":
scatter_intermediate_ssm; the window gather read through the block table of
the "vllm.models.inkling.nvidia.ops.sconv" paged cache)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import hs, raw

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ssm_case(seed, shape, num_chunks, max_count, dtype):
    g = torch.Generator().manual_seed(seed)
    states = torch.randn((num_chunks,) + shape, generator=g).to(workloads.TORCH_DTYPE[dtype])
    rng = np.random.default_rng(seed)
    idx = torch.from_numpy(rng.integers(0, num_chunks, size=max_count).astype(np.int64))
    out = workloads.sentinel((max_count,) + shape, dtype)
    return states, idx, out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(8, 16, 32), (3, 5), (64,), (7,)])
@pytest.mark.parametrize("real", [0, 5, 17, 40])
def test_scatter_ssm_against_oracle(dtype, shape, real):
    states, idx, out = _ssm_case(len(shape) + real, shape, 23, 17, dtype)
    ref, skipped = oracle.scatter_ssm(dtype=dtype, states=states, chunk_indices=idx,
                                      real_count=real, out=out)
    assert skipped == 0
    o = out.to(DEV)
    rc = torch.tensor([real], dtype=torch.int32, device=DEV)
    hs().sconv_scatter_intermediate_ssm(states.to(DEV), idx.to(DEV), rc, o)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(oracle._float_array(o.cpu(), dtype).view(np.uint8),
                                  ref.view(np.uint8))


def test_scatter_ssm_large_rows_and_bad_index():
    """2 MB fp32 state rows (the 16-byte path with many blocks per slot),
    one slot with an index past the chunks: flag set, slot untouched."""
    states, idx, out = _ssm_case(3, (64, 64, 128), 12, 8, "f32")
    idx[5] = 12
    ref, skipped = oracle.scatter_ssm(dtype="f32", states=states, chunk_indices=idx,
                                      real_count=8, out=out)
    assert skipped == 1
    o = out.to(DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    rc = torch.tensor([8], dtype=torch.int32, device=DEV)
    hs().sconv_scatter_intermediate_ssm(states.to(DEV), idx.to(DEV), rc, o, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == hs().EFLAG_REQUEST
    assert torch.equal(raw(o.cpu()), torch.from_numpy(ref.view(np.int32)))


def test_scatter_ssm_real_count_changes_between_replays():
    states, idx, out = _ssm_case(4, (32, 16), 9, 12, "bf16")
    s_d, i_d, o = states.to(DEV), idx.to(DEV), out.to(DEV)
    rc = torch.tensor([12], dtype=torch.int32, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        hs().sconv_scatter_intermediate_ssm(s_d, i_d, rc, o)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        hs().sconv_scatter_intermediate_ssm(s_d, i_d, rc, o)
    for real in (12, 3, 0, 7):
        o.copy_(out.to(DEV))
        rc.fill_(real)
        g.replay()
        torch.cuda.synchronize()
        ref, _ = oracle.scatter_ssm(dtype="bf16", states=states, chunk_indices=idx,
                                    real_count=real, out=out)
        np.testing.assert_array_equal(oracle._float_array(o.cpu(), "bf16"), ref)
    del g


def _paged_check(wl, t, req, pos, real, d_conv, err=None):
    out = workloads.sentinel((len(req), wl.C, d_conv), wl.dtype, DEV)
    before = out.cpu()
    rc = torch.tensor([real], dtype=torch.int32, device=DEV)
    hs().sconv_extract_windows_paged(t["cache"], t["block_table"], torch.from_numpy(req).to(DEV),
                                     torch.from_numpy(pos).to(DEV), rc, out, d_conv, wl.off_s,
                                     wl.ws, err_flag=err)
    torch.cuda.synchronize()
    ref, skipped = oracle.extract_windows_paged(
        dtype=wl.dtype, cache=t["cache"].cpu(), block_table=wl.block_table, request=req,
        abs_positions=pos, real_count=real, out=before, d_conv=d_conv, off_s=wl.off_s, ws=wl.ws)
    np.testing.assert_array_equal(oracle._float_array(out.cpu(), wl.dtype).view(np.uint8),
                                  ref.view(np.uint8))
    return skipped


@pytest.mark.parametrize("seed", range(12))
def test_extract_windows_paged_random(seed):
    wl = workloads.random_case(300 + seed, max_hist=40)
    t = wl.tensors(DEV)
    rng = np.random.default_rng(seed)
    d_conv = int(rng.integers(1, 9))
    n = int(rng.integers(1, 20))
    req = rng.integers(0, wl.R, size=n).astype(np.int32)
    lengths = wl.hist + wl.new
    pos = np.array([rng.integers(0, lengths[r] + 1) for r in req], np.int32)
    assert _paged_check(wl, t, req, pos, int(rng.integers(0, n + 3)), d_conv) == 0


def test_extract_windows_paged_bad_block_sets_flag():
    wl = workloads.random_case(320, dtype="bf16", vec_friendly=True, max_hist=40)
    t = wl.tensors(DEV)
    req = np.array([0, 0], np.int32)
    length = int(wl.hist[0] + wl.new[0])
    pos = np.array([length, length], np.int32)
    t["block_table"] = t["block_table"].clone()
    wl.block_table = wl.block_table.copy()
    if length >= 1:
        lb = (length - 1) // wl.N
        wl.block_table[0, lb] = wl.num_blocks + 5
        t["block_table"][0, lb] = wl.num_blocks + 5
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    skipped = _paged_check(wl, t, req, pos, 2, 4, err=err)
    if length >= 1:
        assert skipped == 2 and int(err.item()) == hs().EFLAG_BLOCK


def test_extract_windows_paged_equals_dense_after_long_prefill():
    """The long-prefill workload: after the fused step has inserted all
    65536 tokens, the windows read back from the paged cache at the 64
    extraction positions equal the dense windows of x, bit for bit."""
    wl = workloads.long_prefill_bf16()
    t = wl.tensors(DEV)
    hs().sconv_fused(t["x"], t["weight"], t["cache"], t["positions"], t["block_table"],
                     t["seq_idx"], t["slot_mapping"], t["query_start"], **wl.kwargs())
    e = wl.extra
    pos = torch.from_numpy(e["abs_positions"]).to(DEV)
    rc = torch.tensor([e["max_count"]], dtype=torch.int32, device=DEV)
    dense = workloads.sentinel((e["max_count"], wl.C, e["d_conv"]), "bf16", DEV)
    paged = workloads.sentinel((e["max_count"], wl.C, e["d_conv"]), "bf16", DEV)
    hs().sconv_extract_windows(t["x"], pos, rc, dense, e["d_conv"])
    req = torch.zeros(e["max_count"], dtype=torch.int32, device=DEV)
    hs().sconv_extract_windows_paged(t["cache"], t["block_table"], req, pos, rc, paged,
                                     e["d_conv"], wl.off_s, wl.ws)
    torch.cuda.synchronize()
    assert torch.equal(raw(dense), raw(paged))
