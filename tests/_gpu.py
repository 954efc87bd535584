"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs.

Comparison rules (from the path's stated tolerances):
  * conv outputs: |gpu - ref| <= atol + rtol*|ref| with (1e-5, 1e-5) for
    fp32 data and (1e-2, 8e-3) for bf16 outputs, ref in float64;
  * cache contents, PAD / skipped output rows, extracted windows and
    untouched slots: bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

TOL = {"f32": (1e-5, 1e-5), "bf16": (1e-2, 8e-3)}
RAW = {"f32": torch.int32, "bf16": torch.int16}


def hs():
    import hybrid_sconv_b200
    return hybrid_sconv_b200


def raw(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


def assert_close(got64: np.ndarray, ref64: np.ndarray, dtype: str, what: str) -> None:
    atol, rtol = TOL[dtype]
    ok = np.abs(got64 - ref64) <= atol + rtol * np.abs(ref64)
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError(
            f"{what}: {len(bad)} of {ok.size} elements out of tolerance; first at {i}: "
            f"gpu {got64[i]!r} ref {ref64[i]!r}")


def run_fused(wl, t, out=None, err=None, **kw):
    args = wl.kwargs()
    args.update(kw)
    return hs().sconv_fused(t["x"], t["weight"], t["cache"], t["positions"],
                            t["block_table"], t["seq_idx"], t["slot_mapping"],
                            t["query_start"], out=out, err_flag=err, **args)


def run_update(wl, t, out=None, err=None, **kw):
    """sconv_update on a decode-form step (token b is request b)."""
    args = wl.kwargs()
    args.update(kw)
    return hs().sconv_update(t["x"], t["weight"], t["cache"], t["positions"],
                             t["block_table"], t["slot_mapping"], out=out, err_flag=err, **args)


def oracle_fused(wl, x, weight, cache, md, **kw):
    args = dict(dtype=wl.dtype, x=x, weight=weight, cache=cache,
                positions=md["positions"], block_table=md["block_table"],
                seq_idx=md["seq_idx"], slot_mapping=md["slot_mapping"],
                query_start=md["query_start"])
    args.update(wl.kwargs())
    args.update(kw)
    return oracle.fused(**args)


def check_small(wl, device="cuda", t=None, md_cpu=None, run=run_fused):
    """Full comparison of one step: every output row, every cache byte, and
    the untouched PAD rows.  ``run(wl, t, out=...)`` launches the step
    (sconv_fused by default).  Returns the GPU out tensor."""
    if t is None:
        t = wl.tensors(device)
    md_cpu = md_cpu or wl.metadata("cpu")
    cache_before = t["cache"].cpu()
    out = workloads.sentinel(tuple(t["x"].shape), wl.dtype, device)
    run(wl, t, out=out)
    torch.cuda.synchronize()
    ref, state, cache_ref, skipped = oracle_fused(wl, t["x"].cpu(), t["weight"].cpu(),
                                                  cache_before, md_cpu)
    assert skipped == 0
    got = out.cpu()
    rows = state == 1
    assert_close(oracle.to_f64(got, wl.dtype)[rows], ref[rows], wl.dtype, f"{wl.name} out")
    np.testing.assert_array_equal(raw(got)[~torch.from_numpy(rows)].numpy(), -1,
                                  err_msg=f"{wl.name}: PAD rows were written")
    np.testing.assert_array_equal(oracle._float_array(t["cache"].cpu(), wl.dtype), cache_ref,
                                  err_msg=f"{wl.name}: cache differs")
    return out


def sample_ranges(T, pieces=4, width=1024, seed=0):
    """Token ranges covering the start, the end and a few random places."""
    rng = np.random.default_rng(seed)
    if T <= pieces * width:
        return [(0, T)]
    starts = {0, T - width}
    starts |= set(int(s) for s in rng.integers(0, T - width, size=pieces - 2))
    return sorted((s, s + width) for s in starts)


def check_full_size(wl, device="cuda", ranges=None, t=None, run=run_fused):
    """Full-size step: the launch the benchmark times, compared with the
    oracle on sampled token ranges (outputs and the insert of each sampled
    token, element by element), plus size-independent properties over every
    token: each written element holds x, nothing else in the cache changed,
    PAD rows are untouched.  ``run`` launches the step (sconv_fused by
    default; run_update for a decode-form step)."""
    if t is None:
        t = wl.tensors(device)
    md_cpu = wl.metadata("cpu")
    x_cpu, w_cpu = t["x"].cpu(), t["weight"].cpu()
    cache_before_cpu = t["cache"].cpu()
    cache_before = t["cache"].clone()
    out = workloads.sentinel(tuple(t["x"].shape), wl.dtype, device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    run(wl, t, out=out, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.cpu()
    cache_after_flat = raw(t["cache"]).view(-1)
    x_raw = raw(x_cpu)
    for a, b in (ranges or sample_ranges(wl.T)):
        ref, state, _, skipped, widx = oracle_fused(
            wl, x_cpu, w_cpu, cache_before_cpu, md_cpu, t_range=(a, b), write_cache=False,
            write_index=True)
        assert skipped == 0
        rows = state == 1
        assert_close(oracle.to_f64(got[a:b], wl.dtype)[rows], ref[rows], wl.dtype,
                     f"{wl.name} out rows {a}..{b}")
        widx_t = torch.from_numpy(widx[rows]).to(device)
        np.testing.assert_array_equal(cache_after_flat[widx_t].cpu().numpy(),
                                      x_raw[a:b][torch.from_numpy(rows)].numpy(),
                                      err_msg=f"{wl.name}: insert of rows {a}..{b}")
    # Properties over all tokens.
    pad = torch.from_numpy(wl.slot_mapping == -1)
    assert bool((raw(got)[pad] == -1).all()), "PAD rows were written"
    check_cache_holds_x(wl, t, cache_before)
    return out


def check_cache_holds_x(wl, t, cache_before):
    """Over every token: the cache element (block_table[r, p // N], h, p % N,
    off_s + j) of each non-PAD token of request r at position p holds
    x[token, h*ws + j] bit for bit, and no other element of the cache changed
    (plain 4-D indexing of the page's layout, on the device)."""
    dev = t["cache"].device
    after, before = raw(t["cache"]), raw(cache_before)
    written = torch.zeros(t["cache"].shape, dtype=torch.bool, device=dev)
    keep = t["slot_mapping"] != -1
    r = t["seq_idx"][keep].long()
    p = t["positions"][keep]
    blk = t["block_table"][r, p // wl.N].long()
    off = p % wl.N
    lanes = torch.arange(wl.off_s, wl.off_s + wl.ws, device=dev)
    xk = raw(t["x"])[keep]
    for h in range(wl.H):
        idx = (blk[:, None], h, off[:, None], lanes[None, :])
        assert torch.equal(after[idx], xk[:, h * wl.ws:(h + 1) * wl.ws]), \
            f"cache does not hold x for head {h}"
        written[idx] = True
    assert not bool(((after != before) & ~written).any()), "cache changed outside the inserts"
