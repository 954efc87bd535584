"""GPU parity of sconv_fused / sconv_update against the CPU oracle, through
the C ABI ("vllm.models.inkling.nvidia.ops.sconv", fused_sconv)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import (assert_close, check_cache_holds_x, check_full_size, check_small, hs,
                        oracle_fused, raw, run_fused, run_update)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_tiny_prefill_f32():
    check_small(workloads.tiny_prefill_f32(), DEV)


@pytest.mark.parametrize("seed", range(40))
def test_random_small_cases(seed):
    check_small(workloads.random_case(seed), DEV)


@pytest.mark.parametrize("seed,dtype,ws,H,max_new", [
    (1, "bf16", 128, 32, 900),    # C = 4096, several tiles per request
    (2, "bf16", 72, 9, 6000),     # C = 648: a ragged channel tail (TMA tiles past C)
    (3, "f32", 64, 16, 1500),     # fp32, 4-wide packs
    (4, "bf16", 32, 32, 3000),    # many token-packs: the 8-tokens-per-thread tile
    (5, "bf16", 8, 3, 400),       # C = 24: narrow blocks
    (6, "f32", 5, 7, 700),        # one-element path
])
def test_medium_multi_tile(seed, dtype, ws, H, max_new):
    rng = np.random.default_rng(seed)
    R = 5
    wl = workloads.build(f"medium_{seed}", dtype=dtype, H=H, D=ws + 8, ws=ws, off_s=8 if ws % 8 == 0 else 3,
                         W=4, N=16, hist=rng.integers(0, 40, size=R),
                         new=rng.integers(1, max_new + 1, size=R), act="silu",
                         residual=bool(seed % 2), seed=seed, num_pad=7, rng=rng)
    check_small(wl, DEV)


@pytest.mark.parametrize("W", range(1, 9))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_every_window_length(W, dtype):
    rng = np.random.default_rng(W)
    wl = workloads.build(f"w{W}", dtype=dtype, H=4, D=64, ws=32, off_s=16, W=W, N=4,
                         hist=rng.integers(0, 12, size=6), new=rng.integers(1, 300, size=6),
                         act="silu", residual=True, seed=W, num_pad=5, rng=rng)
    check_small(wl, DEV)


@pytest.mark.parametrize("W", range(1, 9))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prefill_tile_kernel_every_window_length(W, dtype):
    """Enough token-packs (T*C/VEC >= 2^19) for the prefill form (TMA tiles
    of 32 tokens x 512 bytes, W-1 halo rows), with request starts,
    histories and PAD rows inside tiles, for every tap count and both
    dtypes."""
    rng = np.random.default_rng(100 + W)
    H = 16 if dtype == "bf16" else 8
    wl = workloads.build(f"tile_w{W}_{dtype}", dtype=dtype, H=H, D=136, ws=128, off_s=8, W=W,
                         N=16, hist=rng.integers(0, 30, size=4),
                         new=rng.integers(600, 900, size=4), act="silu",
                         residual=bool(W % 2), seed=W, num_pad=9, rng=rng)
    vec = 8 if dtype == "bf16" else 4
    assert wl.T * wl.C // vec >= 1 << 19
    check_small(wl, DEV)


@pytest.mark.parametrize("dtype,H,W", [
    ("bf16", 32, 5), ("bf16", 32, 8),   # 16 channel blocks: weights cached, 2 per block
    ("f32", 16, 6), ("f32", 16, 8),     # the same for fp32 (cached above W = 5)
    ("bf16", 18, 5),                    # 9 channel blocks: 9 cached weight sets
    ("bf16", 18, 8),                    # 9 blocks x W 8 exceed the cache: reloaded per switch
])
def test_prefill_tile_kernel_channel_block_switches(dtype, H, W):
    """The tiled prefill form's persistent blocks take (token tile, channel
    block) units in token-major order, so a block's channel block changes
    from unit to unit when the grid is not a multiple of the channel-block
    count: its weights then come from the shared-memory copy made at entry
    (W above 4 for bf16, above 5 for fp32, when they fit) or are reloaded."""
    rng = np.random.default_rng(300 + W + H)
    wl = workloads.build(f"switch_{dtype}_h{H}_w{W}", dtype=dtype, H=H, D=136, ws=128,
                         off_s=8, W=W, N=16, hist=rng.integers(0, 30, size=4),
                         new=rng.integers(500, 700, size=4), act="silu", residual=True,
                         seed=W + H, num_pad=11, rng=rng)
    vec = 8 if dtype == "bf16" else 4
    assert wl.T * wl.C // vec >= 1 << 19
    check_small(wl, DEV)


@pytest.mark.parametrize("W", [4, 5, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_unaligned_metadata_takes_the_strip_kernel(W, dtype):
    """Metadata arrays that start 8 bytes past a 16-byte boundary cannot be
    bulk-copied; the streamed strip kernel serves the same step."""
    rng = np.random.default_rng(11)
    wl = workloads.build(f"strip_unaligned_w{W}", dtype=dtype, H=16, D=128, ws=128, off_s=0,
                         W=W, N=16, hist=rng.integers(0, 30, size=4),
                         new=rng.integers(600, 900, size=4), act="silu", residual=True,
                         seed=11, num_pad=5, rng=rng)
    t = wl.tensors(DEV)
    for k in ("positions", "slot_mapping"):
        buf = torch.empty(wl.T + 1, dtype=torch.int64, device=DEV)
        buf[1:].copy_(t[k])
        t[k] = buf[1:]
    check_small(wl, DEV, t=t)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_strip_kernel_element_path(dtype):
    """The strip kernel on a layout that is not 16-byte aligned (ws = 5)."""
    rng = np.random.default_rng(7)
    wl = workloads.build("strip_elem", dtype=dtype, H=100, D=10, ws=5, off_s=3, W=4, N=8,
                         hist=rng.integers(0, 20, size=3), new=rng.integers(500, 600, size=3),
                         act="silu", residual=True, seed=7, num_pad=4, rng=rng)
    assert wl.T * wl.C >= 1 << 19
    check_small(wl, DEV)


@pytest.mark.parametrize("name", ["decode_bf16", "chunked_prefill_bf16", "spec_decode_bf16",
                                  "long_prefill_bf16"])
def test_named_workload_full_size(name):
    wl = workloads.NAMED[name]()
    check_full_size(wl, DEV)
    torch.cuda.empty_cache()


def test_empty_step_is_a_no_op():
    wl = workloads.tiny_prefill_f32()
    t = wl.tensors(DEV)
    x0 = t["x"][:0]
    out = run_fused(wl, dict(t, x=x0))
    assert out.shape == (0, wl.C)


def test_strided_layouts():
    """x and out with row strides above C, a cache carved out of a wider
    allocation (every stride differs from the dense one) and a block table
    with padding columns."""
    wl = workloads.random_case(31, dtype="bf16", vec_friendly=True, max_new=200)
    t = wl.tensors(DEV)
    C = wl.C
    xw = torch.zeros(wl.T, C + 24, dtype=t["x"].dtype, device=DEV)
    xw[:, 8:8 + C] = t["x"]
    big = torch.randn(wl.num_blocks + 1, wl.H + 1, wl.N + 2, wl.D + 16, device=DEV).to(
        t["cache"].dtype)
    cache = big[1:, 1:, 2:, 8:8 + wl.D]
    cache.copy_(t["cache"])
    btw = torch.full((wl.R, wl.block_table.shape[1] + 5), -1, dtype=torch.int32, device=DEV)
    btw[:, :wl.block_table.shape[1]] = t["block_table"]
    t2 = dict(t, x=xw[:, 8:8 + C], cache=cache, block_table=btw[:, :wl.block_table.shape[1]])
    outw = workloads.sentinel((wl.T, C + 40), wl.dtype, DEV)
    out = outw[:, 16:16 + C]
    cache_before = cache.cpu().contiguous()
    run_fused(wl, t2, out=out)
    torch.cuda.synchronize()
    md = wl.metadata("cpu")
    ref, state, cache_ref, _ = oracle_fused(wl, t["x"].cpu(), t["weight"].cpu(),
                                            cache_before, md)
    rows = state == 1
    assert_close(oracle.to_f64(out.cpu(), wl.dtype)[rows], ref[rows], wl.dtype, "strided out")
    np.testing.assert_array_equal(oracle._float_array(cache.cpu().contiguous(), wl.dtype),
                                  cache_ref)
    # nothing outside the views was touched
    assert bool((raw(outw[:, :16]) == -1).all() and (raw(outw[:, 16 + C:]) == -1).all())


def test_unaligned_base_takes_the_element_path():
    """x starting one element past a 16-byte boundary: same results."""
    wl = workloads.random_case(32, dtype="bf16", vec_friendly=True, max_new=120)
    t = wl.tensors(DEV)
    flat = torch.empty(wl.T * wl.C + 1, dtype=t["x"].dtype, device=DEV)
    xs = flat[1:].view(wl.T, wl.C)
    xs.copy_(t["x"])
    check_small(wl, DEV, t=dict(t, x=xs))


def test_weight_strides():
    """A transposed weight view (stride (1, C)) gives the same outputs."""
    wl = workloads.random_case(33, dtype="f32", vec_friendly=True)
    t = wl.tensors(DEV)
    wt = t["weight"].t().contiguous().t()
    assert wt.stride() == (1, wl.C)
    check_small(wl, DEV, t=dict(t, weight=wt))


def test_update_equals_fused_bit_exact():
    """sconv_update on a decode step equals sconv_fused with
    seq_idx = query_start = arange, bit for bit (output and cache)."""
    wl = workloads.decode_bf16(seed=77, R=64, max_hist=300)
    t = wl.tensors(DEV)
    cache0 = t["cache"].clone()
    out_f = run_fused(wl, t)
    cache_f = t["cache"].clone()
    t["cache"].copy_(cache0)
    out_u = hs().sconv_update(t["x"], t["weight"], t["cache"], t["positions"],
                              t["block_table"], t["slot_mapping"], **wl.kwargs())
    torch.cuda.synchronize()
    assert torch.equal(raw(out_f), raw(out_u))
    assert torch.equal(raw(cache_f), raw(t["cache"]))
    # and against the oracle
    ref, state, _, _ = oracle.update(dtype=wl.dtype, x=t["x"].cpu(), weight=t["weight"].cpu(),
                                     cache=cache0.cpu(), positions=wl.positions,
                                     block_table=wl.block_table, slot_mapping=wl.slot_mapping,
                                     write_cache=False, **wl.kwargs())
    assert_close(oracle.to_f64(out_u.cpu(), wl.dtype), ref, wl.dtype, "update")


def test_update_full_size_decode():
    """sconv_update on the full decode workload the benchmark times: 256
    requests over histories of up to 4096 tokens, a 4.2 GB cache whose
    element offsets pass 2^31.  The workload is in decode form (token b is
    request b), so the fused definition with its own metadata is the
    update's; every token is compared with the oracle, the inserts element
    by element and the whole cache by the holds-x invariant."""
    wl = workloads.decode_bf16()
    ar = np.arange(wl.T)
    assert np.array_equal(wl.seq_idx, ar) and np.array_equal(wl.query_start, ar)
    check_full_size(wl, DEV, run=run_update)


def test_update_with_pad_rows():
    wl = workloads.decode_bf16(seed=78, R=40, max_hist=100)
    wl.slot_mapping[[3, 17]] = -1
    t = wl.tensors(DEV)
    cache0 = t["cache"].cpu()
    out = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    hs().sconv_update(t["x"], t["weight"], t["cache"], t["positions"], t["block_table"],
                      t["slot_mapping"], out=out, **wl.kwargs())
    torch.cuda.synchronize()
    ref, state, cache_ref, _ = oracle.update(dtype=wl.dtype, x=t["x"].cpu(),
                                             weight=t["weight"].cpu(), cache=cache0,
                                             positions=wl.positions, block_table=wl.block_table,
                                             slot_mapping=wl.slot_mapping, **wl.kwargs())
    rows = state == 1
    got = out.cpu()
    assert_close(oracle.to_f64(got, wl.dtype)[rows], ref[rows], wl.dtype, "update pad")
    assert bool((raw(got)[[3, 17]] == -1).all())
    np.testing.assert_array_equal(oracle._float_array(t["cache"].cpu(), wl.dtype), cache_ref)


def _chunk_inputs(wl, t, a, b):
    """Rows [a, b) of every request's new tokens as a step of their own."""
    rows = torch.cat([torch.arange(int(wl.query_start_loc[r]) + a,
                                   int(wl.query_start_loc[r]) + b) for r in range(wl.R)])
    n = b - a
    seq_idx = torch.arange(wl.R, dtype=torch.int32).repeat_interleave(n)
    qs = (torch.arange(wl.R, dtype=torch.int32) * n).repeat_interleave(n)
    rd = rows.to(DEV)
    return dict(t, x=t["x"][rd].contiguous(), positions=t["positions"][rd].contiguous(),
                slot_mapping=t["slot_mapping"][rd].contiguous(),
                seq_idx=seq_idx.to(DEV), query_start=qs.to(DEV)), rows


@pytest.mark.parametrize("H,ws,W", [(8, 64, 4), (16, 128, 4), (16, 128, 7)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_chunked_prefill_bit_exact_on_gpu(dtype, H, ws, W):
    """Prefill split into chunks, each later chunk reading the cache the
    earlier ones wrote, equals one-shot prefill bit for bit (outputs and
    cache), on the device.  With C = 2048 the one-shot step and the larger
    chunks take the tiled prefill form and the small chunks the token form,
    so this also checks that both forms produce the same bits."""
    R, L = 4, 700
    rng = np.random.default_rng(9)
    wl = workloads.build("chunks", dtype=dtype, H=H, D=ws, ws=ws, off_s=0, W=W, N=16,
                         hist=rng.integers(0, 50, size=R), new=np.full(R, L), act="silu",
                         residual=True, seed=9, rng=rng)
    t = wl.tensors(DEV)
    cache0 = t["cache"].clone()
    one = run_fused(wl, t).clone()
    cache_one = t["cache"].clone()
    t["cache"].copy_(cache0)
    for a, b in [(0, 1), (1, 130), (130, 131), (131, 500), (500, L)]:
        tc, rows = _chunk_inputs(wl, t, a, b)
        out = run_fused(wl, tc)
        assert torch.equal(raw(out), raw(one[rows.to(DEV)])), f"chunk {a}..{b}"
    torch.cuda.synchronize()
    assert torch.equal(raw(t["cache"]), raw(cache_one))


def test_zero_history_decode_equals_prefill_on_gpu():
    R, L = 3, 40
    wl = workloads.build("zh", dtype="bf16", H=4, D=32, ws=32, off_s=0, W=4, N=8,
                         hist=np.zeros(R, np.int64), new=np.full(R, L), act="silu",
                         residual=True, seed=10)
    t = wl.tensors(DEV)
    cache0 = t["cache"].clone()
    one = run_fused(wl, t).clone()
    t["cache"].copy_(cache0)
    for a in range(L):
        tc, rows = _chunk_inputs(wl, t, a, a + 1)
        out = hs().sconv_update(tc["x"], tc["weight"], tc["cache"], tc["positions"],
                                tc["block_table"], tc["slot_mapping"], **wl.kwargs())
        assert torch.equal(raw(out), raw(one[rows.to(DEV)]))


def test_graph_replay_with_redrawn_metadata():
    """The speculative-decode step (T = 512, 10% PAD) captured once in a
    CUDA graph and replayed with new metadata and inputs copied into the
    captured buffers gives the eager results."""
    a = workloads.spec_decode_bf16(seed=1004, max_hist=2048)
    b = workloads.spec_decode_bf16(seed=2004, max_hist=2048)
    nb = max(a.num_blocks, b.num_blocks)
    ta, tb = a.tensors(DEV), b.tensors(DEV)
    cache = torch.empty((nb, a.H, a.N, a.D), dtype=torch.bfloat16, device=DEV)
    workloads.fill_normal_(cache, 1.0, torch.Generator(device=DEV).manual_seed(5), DEV)
    mb = max(a.block_table.shape[1], b.block_table.shape[1])

    def padded_bt(wl, t):
        bt = torch.full((wl.R, mb), -1, dtype=torch.int32, device=DEV)
        bt[:, :wl.block_table.shape[1]] = t["block_table"]
        return bt

    static = {k: ta[k].clone() for k in ("x", "weight", "positions", "seq_idx",
                                          "slot_mapping", "query_start")}
    static["block_table"] = padded_bt(a, ta)
    static["cache"] = cache
    out = workloads.sentinel((a.T, a.C), "bf16", DEV)
    cache0 = cache.clone()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_fused(a, static, out=out)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    cache.copy_(cache0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_fused(a, static, out=out)

    for wl, t in ((a, ta), (b, tb)):
        cache.copy_(cache0)
        out.copy_(workloads.sentinel((a.T, a.C), "bf16", DEV))
        for k in ("x", "positions", "seq_idx", "slot_mapping", "query_start"):
            static[k].copy_(t[k])
        static["block_table"].copy_(padded_bt(wl, t))
        g.replay()
        torch.cuda.synchronize()
        replay_out, replay_cache = out.clone(), cache.clone()
        cache.copy_(cache0)
        eager = workloads.sentinel((a.T, a.C), "bf16", DEV)
        run_fused(wl, dict(static, cache=cache), out=eager)
        torch.cuda.synchronize()
        assert torch.equal(raw(replay_out), raw(eager))
        assert torch.equal(raw(replay_cache), raw(cache))
        # and the replayed step against the oracle on sampled rows
        md = wl.metadata("cpu")
        md["block_table"] = static["block_table"].cpu()
        ref, state, _, _ = oracle_fused(wl, t["x"].cpu(), static["weight"].cpu(), cache0.cpu(),
                                        md, write_cache=False)
        rows = state == 1
        assert_close(oracle.to_f64(replay_out.cpu(), "bf16")[rows], ref[rows], "bf16",
                     f"replay {wl.seed}")
    del g


# --------------------------------------------------------------------------
# device-side bounds checks: bad indices skip the token and set err_flag

def _err_case():
    rng = np.random.default_rng(40)
    return workloads.build("err", dtype="bf16", H=4, D=32, ws=32, off_s=0, W=4, N=8,
                           hist=np.array([5, 20, 0, 9]), new=np.array([6, 1, 7, 2]),
                           act="silu", residual=True, seed=40, rng=rng)


@pytest.mark.parametrize("kind,flag", [
    ("slot", 0x01), ("request", 0x02), ("logical", 0x04), ("block", 0x08),
    ("query_start", 0x10), ("position", 0x20)])
def test_bad_index_sets_flag_and_skips_token(kind, flag):
    wl = _err_case()
    t = wl.tensors(DEV)
    md = wl.metadata("cpu")
    row = int(wl.query_start_loc[1])  # request 1's only token (reads three history taps)
    if kind == "slot":
        md["slot_mapping"][row] = wl.num_blocks * wl.N + 3
    elif kind == "request":
        md["seq_idx"][row] = wl.R + 2
    elif kind == "logical":
        md["block_table"] = md["block_table"].clone()
        md["positions"][row] += wl.block_table.shape[1] * wl.N  # history beyond the table
        md["query_start"][row] = row
    elif kind == "block":
        md["block_table"][1, (int(wl.positions[row]) - 1) // wl.N] = wl.num_blocks + 7
    elif kind == "query_start":
        md["query_start"][row] = row + 1
    elif kind == "position":
        md["positions"][row] = -3
    td = dict(t, **{k: v.to(DEV) for k, v in md.items()})
    cache0 = t["cache"].cpu()
    out = workloads.sentinel((wl.T, wl.C), wl.dtype, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    run_fused(wl, td, out=out, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == flag
    ref, state, cache_ref, skipped = oracle_fused(wl, t["x"].cpu(), t["weight"].cpu(), cache0,
                                                  md)
    assert skipped == 1 and state[row] == 2
    got = out.cpu()
    assert bool((raw(got)[row] == -1).all())
    rows = state == 1
    assert_close(oracle.to_f64(got, wl.dtype)[rows], ref[rows], wl.dtype, kind)
    np.testing.assert_array_equal(oracle._float_array(t["cache"].cpu(), wl.dtype), cache_ref)


def test_no_flag_on_valid_steps():
    wl = workloads.random_case(12)
    t = wl.tensors(DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    run_fused(wl, t, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
