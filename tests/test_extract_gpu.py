"""GPU parity of sconv_extract_windows against the CPU oracle
("core.ssm.ops.intermediate_extraction", scatter_intermediate_conv): the
gathered windows and every untouched slot, bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import hs, raw

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check(src, pos, rc_value, out, d_conv, dtype):
    before = out.clone()
    rc = torch.tensor([rc_value], dtype=torch.int32, device=DEV)
    hs().sconv_extract_windows(src, pos, rc, out, d_conv)
    torch.cuda.synchronize()
    ref = oracle.extract_windows(dtype=dtype, src=src.cpu(), abs_positions=pos.cpu(),
                                 real_count=rc_value, out=before.cpu(), d_conv=d_conv)
    np.testing.assert_array_equal(oracle._float_array(out.cpu(), dtype), ref)


def test_long_prefill_extraction_full_size():
    """The long-prefill workload's extraction: 64 window ends over a
    [65536, 8192] bf16 source, real_count 40."""
    wl = workloads.long_prefill_bf16()
    e = wl.extra
    g = torch.Generator(device=DEV).manual_seed(wl.seed)
    src = workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, DEV)
    out = workloads.sentinel((e["max_count"], wl.C, e["d_conv"]), "bf16", DEV)
    pos = torch.from_numpy(e["abs_positions"]).to(DEV)
    _check(src, pos, e["real_count"], out, e["d_conv"], "bf16")
    assert bool((raw(out[e["real_count"]:]) == -1).all())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d_conv", range(1, 9))
def test_every_window_length(dtype, d_conv):
    src, pos, rc, out = workloads.extraction_inputs(
        d_conv, 300, 256, 24, d_conv, 17, dtype=dtype, device=DEV, lo=0, hi=300 + d_conv)
    _check(src, pos, 17, out, d_conv, dtype)


@pytest.mark.parametrize("conv_dim", [1, 7, 24, 100, 1032])
def test_ragged_channel_counts(conv_dim):
    src, pos, rc, out = workloads.extraction_inputs(4, 64, conv_dim, 9, 4, 6, device=DEV,
                                                    lo=0, hi=70)
    _check(src, pos, 6, out, 4, "bf16")


@pytest.mark.parametrize("real", [0, 1, 63, 64, 100, -5])
def test_real_count_bounds(real):
    src, pos, rc, out = workloads.extraction_inputs(8, 128, 64, 64, 4, 0, device=DEV)
    _check(src, pos, real, out, 4, "bf16")


def test_edge_positions_read_zero():
    src, _, _, out = workloads.extraction_inputs(9, 16, 32, 6, 4, 6, device=DEV)
    pos = torch.tensor([0, 1, 3, 4, 16, 19], dtype=torch.int32, device=DEV)
    _check(src, pos, 6, out, 4, "bf16")


def test_three_dim_source_reads_batch_zero():
    src, pos, _, out = workloads.extraction_inputs(10, 50, 40, 5, 3, 5, device=DEV)
    src3 = torch.stack([src, torch.zeros_like(src)])
    rc = torch.tensor([5], dtype=torch.int32, device=DEV)
    before = out.clone()
    hs().sconv_extract_windows(src3, pos, rc, out, 3)
    torch.cuda.synchronize()
    ref = oracle.extract_windows(dtype="bf16", src=src.cpu(), abs_positions=pos.cpu(),
                                 real_count=5, out=before.cpu(), d_conv=3)
    np.testing.assert_array_equal(oracle._float_array(out.cpu(), "bf16"), ref)


def test_real_count_changes_between_graph_replays():
    """The grid is sized by max_count at capture; the count is read on the
    device at each replay."""
    src, pos, rc, out = workloads.extraction_inputs(11, 512, 128, 32, 4, 32, device=DEV)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        hs().sconv_extract_windows(src, pos, rc, out, 4)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        hs().sconv_extract_windows(src, pos, rc, out, 4)
    for real in (32, 5, 0, 19):
        out.copy_(workloads.sentinel(tuple(out.shape), "bf16", DEV))
        before = out.clone()
        rc.fill_(real)
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.extract_windows(dtype="bf16", src=src.cpu(), abs_positions=pos.cpu(),
                                     real_count=real, out=before.cpu(), d_conv=4)
        np.testing.assert_array_equal(oracle._float_array(out.cpu(), "bf16"), ref)
    del g
