"""Seeded synthetic workloads for the fused short-convolution path.

This module only builds inputs: request mixes, block tables, per-token
metadata, and normally distributed x / weight / cache contents.  It holds
none of the method's arithmetic (no convolution, no cache insert, no tap
resolution, no window gather), so both the CUDA path and the CPU oracle can
be fed from it.

Metadata is built by construction, the way a serving engine's scheduler
would lay a step out ("vllm.models.inkling.nvidia.ops.sconv", fused_sconv
argument comments):
  * requests occupy consecutive rows of x, request r owning rows
    [query_start_loc[r], query_start_loc[r+1]);
  * a request with ``hist`` tokens already cached and ``new`` tokens in this
    step has positions hist, hist+1, ..., hist+new-1;
  * each request gets ceil((hist+new)/N) physical blocks drawn from a seeded
    permutation of the block pool, listed in its block_table row (unused
    entries are -1);
  * a token's flat slot is block*N + offset for the block holding its
    position (the engine's flat-slot convention), and PAD rows get -1.

Random numbers: metadata from numpy's PCG64 seeded with ``seed``; float data
from a ``torch.Generator`` seeded with ``seed`` as float32 N(0, 1) draws
scaled by sigma (sigma is the standard deviation) and rounded to the storage
type with round-to-nearest-even.  Float data is generated on ``gen_device``
(CPU for small cases, so the same values reach every device; the GPU for the
multi-gigabyte caches).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}
ELEM_BYTES = {"f32": 4, "bf16": 2}

# Float data of fewer elements than this is generated on the CPU.
SMALL_ELEMS = 1 << 25


@dataclass
class Workload:
    """One step of the fused sconv path: geometry, request mix, metadata."""

    name: str
    dtype: str
    H: int
    D: int
    ws: int
    off_s: int
    W: int
    N: int
    act: Optional[str]
    residual: bool
    seed: int
    hist: np.ndarray            # [R] tokens already in the cache per request
    new: np.ndarray             # [R] tokens of this step per request
    num_blocks: int
    block_table: np.ndarray     # [R, max_blocks] int32, -1 = unused
    query_start_loc: np.ndarray  # [R+1] int32
    positions: np.ndarray       # [T] int64
    seq_idx: np.ndarray         # [T] int32
    query_start: np.ndarray     # [T] int32
    slot_mapping: np.ndarray    # [T] int64, -1 = PAD
    x_sigma: float = 1.0
    w_sigma: float = 0.5
    cache_sigma: float = 1.0
    extra: dict = field(default_factory=dict)

    @property
    def C(self) -> int:
        return self.H * self.ws

    @property
    def T(self) -> int:
        return int(self.positions.shape[0])

    @property
    def R(self) -> int:
        return int(self.hist.shape[0])

    @property
    def num_pad(self) -> int:
        return int((self.slot_mapping == -1).sum())

    @property
    def elem_bytes(self) -> int:
        return ELEM_BYTES[self.dtype]

    @property
    def cache_elems(self) -> int:
        return self.num_blocks * self.H * self.N * self.D

    # -- tensors -----------------------------------------------------------
    def metadata(self, device="cpu") -> dict:
        d = torch.device(device)
        return {
            "positions": torch.from_numpy(self.positions).to(d),
            "seq_idx": torch.from_numpy(self.seq_idx).to(d),
            "query_start": torch.from_numpy(self.query_start).to(d),
            "slot_mapping": torch.from_numpy(self.slot_mapping).to(d),
            "block_table": torch.from_numpy(self.block_table).to(d),
            "query_start_loc": torch.from_numpy(self.query_start_loc).to(d),
        }

    def float_tensors(self, device="cpu", gen_device=None, cache=True) -> dict:
        """x [T, C], weight [C, W] and (optionally) the cache
        [num_blocks, H, N, D], all of ``self.dtype``, on ``device``."""
        dt = TORCH_DTYPE[self.dtype]
        if gen_device is None:
            total = self.T * self.C + self.C * self.W + (self.cache_elems if cache else 0)
            gen_device = "cpu" if total < SMALL_ELEMS else device
        g = torch.Generator(device=gen_device).manual_seed(self.seed)
        x = normal((self.T, self.C), self.x_sigma, dt, g, gen_device).to(device)
        w = normal((self.C, self.W), self.w_sigma, dt, g, gen_device).to(device)
        out = {"x": x, "weight": w}
        if cache:
            c = torch.empty((self.num_blocks, self.H, self.N, self.D), dtype=dt, device=device)
            fill_normal_(c, self.cache_sigma, g, gen_device)
            out["cache"] = c
        return out

    def tensors(self, device="cpu", gen_device=None) -> dict:
        t = self.float_tensors(device, gen_device)
        t.update(self.metadata(device))
        return t

    def kwargs(self) -> dict:
        """The scalar arguments of fused_sconv for this workload."""
        return {"off_s": self.off_s, "ws": self.ws, "block_size": self.N,
                "activation": self.act, "use_residual": self.residual}


def normal(shape, sigma, dtype, gen, gen_device) -> torch.Tensor:
    v = torch.randn(shape, generator=gen, device=gen_device, dtype=torch.float32)
    if sigma != 1.0:
        v.mul_(sigma)
    return v.to(dtype)


def fill_normal_(t: torch.Tensor, sigma, gen, gen_device, chunk=1 << 28) -> None:
    """Fill ``t`` (any device) with N(0, sigma) in chunks of ``chunk`` elements."""
    flat = t.view(-1)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        flat[s:e].copy_(normal((e - s,), sigma, t.dtype, gen, gen_device))


# --------------------------------------------------------------------------
# construction of the metadata

def build(name, *, dtype, H, D, ws, off_s, W, N, hist, new, act, residual, seed,
          num_pad=0, pad_rows=None, w_sigma=0.5, x_sigma=1.0, cache_sigma=1.0,
          deal_per_request=None, num_blocks=None, rng=None) -> Workload:
    """Lay out one step.  ``deal_per_request`` gives every request that many
    block-table entries (a permutation of the pool dealt in order) instead
    of exactly the blocks it needs; ``num_blocks`` enlarges the pool."""
    if rng is None:
        rng = np.random.default_rng(seed)
    hist = np.asarray(hist, np.int64)
    new = np.asarray(new, np.int64)
    R = hist.shape[0]
    need = -(-(hist + new) // N)  # blocks each request occupies
    if deal_per_request is not None:
        if np.any(need > deal_per_request):
            raise ValueError("deal_per_request too small")
        per = np.full(R, deal_per_request, np.int64)
    else:
        per = need
    pool = int(per.sum())
    if num_blocks is None:
        num_blocks = pool
    if num_blocks < pool:
        raise ValueError("pool too small")
    max_blocks = max(1, int(per.max()) if R else 1)
    perm = rng.permutation(num_blocks).astype(np.int32)
    bt = np.full((max(R, 1), max_blocks), -1, np.int32)
    o = 0
    for r in range(R):
        bt[r, : per[r]] = perm[o: o + per[r]]
        o += per[r]

    qsl = np.zeros(R + 1, np.int32)
    qsl[1:] = np.cumsum(new)
    T = int(qsl[-1])
    positions = np.empty(T, np.int64)
    seq_idx = np.empty(T, np.int32)
    query_start = np.empty(T, np.int32)
    slot = np.empty(T, np.int64)
    for r in range(R):
        a, b = int(qsl[r]), int(qsl[r + 1])
        p = hist[r] + np.arange(b - a, dtype=np.int64)
        positions[a:b] = p
        seq_idx[a:b] = r
        query_start[a:b] = a
        slot[a:b] = bt[r, p // N].astype(np.int64) * N + p % N
    if pad_rows is None and num_pad:
        pad_rows = np.sort(rng.choice(T, size=num_pad, replace=False))
    if pad_rows is not None:
        slot[np.asarray(pad_rows, np.int64)] = -1
    return Workload(name=name, dtype=dtype, H=H, D=D, ws=ws, off_s=off_s, W=W, N=N,
                    act=act, residual=residual, seed=seed, hist=hist, new=new,
                    num_blocks=num_blocks, block_table=bt, query_start_loc=qsl,
                    positions=positions, seq_idx=seq_idx, query_start=query_start,
                    slot_mapping=slot, x_sigma=x_sigma, w_sigma=w_sigma,
                    cache_sigma=cache_sigma)


# --------------------------------------------------------------------------
# the five named workloads (default seed 1000 + number)

def tiny_prefill_f32(seed=1001) -> Workload:
    """2 requests of 5 and 3 new tokens from position 0; H=2, D=16, ws=4,
    off_s=0, C=8, W=4, N=4, 8 blocks dealt 4 per request from a seeded
    permutation; x~N(0,1), weight~N(0,0.5); no activation, residual on."""
    return build("tiny_prefill_f32", dtype="f32", H=2, D=16, ws=4, off_s=0, W=4, N=4,
                 hist=[0, 0], new=[5, 3], act=None, residual=True, seed=seed,
                 deal_per_request=4, num_blocks=8)


def decode_bf16(seed=1002, R=256, max_hist=4096, min_hist=1) -> Workload:
    """256 single-token requests over histories of U{1..4096} cached tokens;
    H=32, D=128, stream 2 of 4 (ws=32, off_s=32), C=1024, W=4, N=16; cache
    filled with N(0,1); weight~N(0,0.5); SiLU, residual on.  min_hist =
    max_hist = 0 gives the same batch shape with no history (every token at
    position 0, no cache taps)."""
    rng = np.random.default_rng(seed)
    hist = rng.integers(min_hist, max_hist + 1, size=R)
    return build("decode_bf16", dtype="bf16", H=32, D=128, ws=32, off_s=32, W=4, N=16,
                 hist=hist, new=np.ones(R, np.int64), act="silu", residual=True,
                 seed=seed, rng=rng)


def chunked_prefill_bf16(seed=1003, R=16, max_prefix=2048, max_new=2048) -> Workload:
    """16 requests, cached prefix U{0..2048}, new tokens U{1..2048};
    H=32, D=128, ws=128, off_s=0, C=4096, W=4, N=16; SiLU, no residual."""
    rng = np.random.default_rng(seed)
    hist = rng.integers(0, max_prefix + 1, size=R)
    new = rng.integers(1, max_new + 1, size=R)
    return build("chunked_prefill_bf16", dtype="bf16", H=32, D=128, ws=128, off_s=0,
                 W=4, N=16, hist=hist, new=new, act="silu", residual=False,
                 seed=seed, rng=rng)


def spec_decode_bf16(seed=1004, R=128, draft=4, min_hist=16, max_hist=8192,
                     pad_frac=0.1) -> Workload:
    """128 requests x 4 draft tokens over histories U{16..8192}; 10% of the
    512 rows PAD (seeded subset); H=16, D=128, ws=128, off_s=0, C=2048, W=4,
    N=16; SiLU, residual on."""
    rng = np.random.default_rng(seed)
    hist = rng.integers(min_hist, max_hist + 1, size=R)
    T = R * draft
    return build("spec_decode_bf16", dtype="bf16", H=16, D=128, ws=128, off_s=0, W=4,
                 N=16, hist=hist, new=np.full(R, draft, np.int64), act="silu",
                 residual=True, seed=seed, num_pad=int(pad_frac * T), rng=rng)


def long_prefill_bf16(seed=1005, T=65536, H=64, ws=128, N=64) -> Workload:
    """One request of 65536 new tokens from position 0; H=64, ws=128,
    D=128, off_s=0, C=8192, W=4, N=64 (1024 permuted blocks);
    weight~N(0,0.3); SiLU, no residual.  ``extra`` carries the window
    extraction: 64 end positions U{4..65536}, real_count 40, d_conv 4."""
    rng = np.random.default_rng(seed)
    wl = build("long_prefill_bf16", dtype="bf16", H=H, D=ws, ws=ws, off_s=0, W=4, N=N,
               hist=[0], new=[T], act="silu", residual=False, seed=seed,
               w_sigma=0.3, rng=rng)
    d_conv, max_count = 4, 64
    wl.extra = {
        "d_conv": d_conv,
        "max_count": max_count,
        "real_count": 40,
        "abs_positions": rng.integers(d_conv, T + 1, size=max_count).astype(np.int32),
    }
    return wl


NAMED = {
    "tiny_prefill_f32": tiny_prefill_f32,
    "decode_bf16": decode_bf16,
    "chunked_prefill_bf16": chunked_prefill_bf16,
    "spec_decode_bf16": spec_decode_bf16,
    "long_prefill_bf16": long_prefill_bf16,
}


# --------------------------------------------------------------------------
# randomised small cases (parity tests across tiles and ragged tails)

def random_case(seed, dtype=None, vec_friendly=None, max_new=40, max_hist=40,
                max_reqs=6, pad_frac=None) -> Workload:
    """A small random step: W in 1..8, H 1..4, ws, off_s, N, request mix,
    histories, PAD rows.  ``vec_friendly`` forces ws and off_s to multiples
    of 8 (16-byte vectors of bf16); False forces an odd ws."""
    rng = np.random.default_rng(seed)
    if dtype is None:
        dtype = "bf16" if rng.random() < 0.6 else "f32"
    if vec_friendly is None:
        vec_friendly = bool(rng.random() < 0.7)
    W = int(rng.integers(1, 9))
    H = int(rng.integers(1, 5))
    if vec_friendly:
        ws = 8 * int(rng.integers(1, 9))
        off_s = 8 * int(rng.integers(0, 4))
    else:
        ws = int(rng.choice([1, 3, 5, 7, 9, 13]))
        off_s = int(rng.integers(0, 6))
    D = off_s + ws + int(rng.integers(0, 3)) * (8 if vec_friendly else 1)
    N = int(rng.choice([1, 2, 3, 4, 8, 16]))
    R = int(rng.integers(1, max_reqs + 1))
    hist = rng.integers(0, max_hist + 1, size=R)
    new = rng.integers(0, max_new + 1, size=R)
    if new.sum() == 0:
        new[0] = 1
    T = int(new.sum())
    if pad_frac is None:
        pad_frac = float(rng.choice([0.0, 0.1, 0.3]))
    num_pad = int(pad_frac * T)
    act = "silu" if rng.random() < 0.5 else None
    residual = bool(rng.random() < 0.5)
    extra_blocks = int(rng.integers(0, 4))
    need = int((-(-(hist + new) // N)).sum())
    return build(f"random_{seed}", dtype=dtype, H=H, D=D, ws=ws, off_s=off_s, W=W, N=N,
                 hist=hist, new=new, act=act, residual=residual, seed=seed,
                 num_pad=num_pad, num_blocks=need + extra_blocks, rng=rng)


def extraction_inputs(seed, seq_len, conv_dim, max_count, d_conv, real_count,
                      dtype="bf16", device="cpu", lo=None, hi=None):
    """src [seq_len, conv_dim] ~ N(0,1), end positions U{lo..hi} (default
    d_conv..seq_len), a device int32[1] real_count and an out buffer
    [max_count, conv_dim, d_conv] pre-filled with the all-ones bit pattern."""
    rng = np.random.default_rng(seed)
    lo = d_conv if lo is None else lo
    hi = seq_len if hi is None else hi
    pos = rng.integers(lo, hi + 1, size=max_count).astype(np.int32)
    dt = TORCH_DTYPE[dtype]
    gen_device = "cpu" if seq_len * conv_dim < SMALL_ELEMS else device
    g = torch.Generator(device=gen_device).manual_seed(seed)
    src = normal((seq_len, conv_dim), 1.0, dt, g, gen_device).to(device)
    out = sentinel((max_count, conv_dim, d_conv), dtype, device)
    rc = torch.tensor([real_count], dtype=torch.int32, device=device)
    return src, torch.from_numpy(pos).to(device), rc, out


def sentinel(shape, dtype, device="cpu") -> torch.Tensor:
    """A buffer whose every byte is 0xFF (a NaN pattern in both dtypes)."""
    dt = TORCH_DTYPE[dtype]
    raw = torch.full(shape, -1, dtype=torch.int16 if dtype == "bf16" else torch.int32,
                     device=device)
    return raw.view(dt)


# --------------------------------------------------------------------------
# the dense-state interface ("Implementation:Sgl project Sglang Mamba Ops":
# causal_conv1d_fwd / causal_conv1d_update)

def dense_conv_inputs(seed, *, dtype, dim, W, state_len, lens, num_lines=None, num_pad=0,
                      init_frac=0.5, bias=True, x_layout="token_major",
                      state_layout="k_contig", device="cpu", pad_slot_id=-1,
                      w_sigma=0.5, x_sigma=1.0, state_sigma=1.0, has_init=None):
    """Inputs of one varlen prefill over dense state lines.

    Sequence b owns x rows [query_start_loc[b], query_start_loc[b+1]) with
    lens[b] rows.  cache_indices are distinct lines drawn from a seeded
    permutation of ``num_lines`` (default batch + 3) lines, ``num_pad`` of
    them replaced by ``pad_slot_id``; has_initial_state is 1 with
    probability ``init_frac`` (or the given array).  Storage layouts:
      x_layout  "token_major": x [T, dim] contiguous;
                "channel_major": a contiguous [dim, T] buffer seen as [T, dim].
      state_layout "k_contig": conv_states [lines, dim, L] contiguous;
                   "c_contig": a contiguous [lines, L, dim] buffer seen as
                   [lines, dim, L].
    Returns a dict of tensors on ``device`` (x, weight, bias or None,
    conv_states, query_start_loc, cache_indices, has_initial_state).
    """
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int64)
    batch = len(lens)
    T = int(lens.sum())
    num_lines = batch + 3 if num_lines is None else num_lines
    qsl = np.zeros(batch + 1, np.int32)
    qsl[1:] = np.cumsum(lens)
    lines = rng.permutation(num_lines)[:batch].astype(np.int32)
    if num_pad:
        lines[rng.choice(batch, size=num_pad, replace=False)] = pad_slot_id
    if has_init is None:
        has_init = rng.random(batch) < init_frac
    dt = TORCH_DTYPE[dtype]
    big = (T + num_lines * state_len) * dim >= SMALL_ELEMS
    gen_device = device if big else "cpu"
    g = torch.Generator(device=gen_device).manual_seed(seed)
    weight = normal((dim, W), w_sigma, dt, g, gen_device).to(device)
    b = normal((dim,), w_sigma, dt, g, gen_device).to(device) if bias else None
    if x_layout == "token_major":
        x = torch.empty((T, dim), dtype=dt, device=device)
    elif x_layout == "channel_major":
        x = torch.empty((dim, T), dtype=dt, device=device).t()
    else:
        raise ValueError(x_layout)
    fill_normal_(x if x.is_contiguous() else x.t(), x_sigma, g, gen_device)
    if state_layout == "k_contig":
        cs = torch.empty((num_lines, dim, state_len), dtype=dt, device=device)
    elif state_layout == "c_contig":
        cs = torch.empty((num_lines, state_len, dim), dtype=dt, device=device).transpose(1, 2)
    else:
        raise ValueError(state_layout)
    fill_normal_(cs if cs.is_contiguous() else cs.transpose(1, 2), state_sigma, g, gen_device)
    return {
        "x": x, "weight": weight, "bias": b, "conv_states": cs,
        "query_start_loc": torch.from_numpy(qsl).to(device),
        "cache_indices": torch.from_numpy(lines).to(device),
        "has_initial_state": torch.from_numpy(np.asarray(has_init, np.bool_)).to(device),
        "pad_slot_id": pad_slot_id,
    }


def dense_update_inputs(seed, *, dtype, batch, dim, W, state_len, num_lines=None, num_pad=0,
                        ring=False, bias=True, state_layout="k_contig", device="cpu",
                        pad_slot_id=-1, max_seqlen=4096):
    """Inputs of one decode step over dense state lines: x [batch, dim],
    conv_state [lines, dim, L] (layouts as in dense_conv_inputs), distinct
    conv_state_indices with ``num_pad`` padded entries, and for ``ring``
    cache_seqlens uniform in 0..max_seqlen."""
    rng = np.random.default_rng(seed)
    num_lines = batch + 3 if num_lines is None else num_lines
    lines = rng.permutation(num_lines)[:batch].astype(np.int32)
    if num_pad:
        lines[rng.choice(batch, size=num_pad, replace=False)] = pad_slot_id
    seqlens = rng.integers(0, max_seqlen + 1, size=batch).astype(np.int32) if ring else None
    dt = TORCH_DTYPE[dtype]
    g = torch.Generator().manual_seed(seed)
    weight = normal((dim, W), 0.5, dt, g, "cpu").to(device)
    b = normal((dim,), 0.5, dt, g, "cpu").to(device) if bias else None
    x = normal((batch, dim), 1.0, dt, g, "cpu").to(device)
    if state_layout == "k_contig":
        cs = normal((num_lines, dim, state_len), 1.0, dt, g, "cpu").to(device)
    else:
        cs = normal((num_lines, state_len, dim), 1.0, dt, g, "cpu").to(device).transpose(1, 2)
    return {
        "x": x, "weight": weight, "bias": b, "conv_state": cs,
        "conv_state_indices": torch.from_numpy(lines).to(device),
        "cache_seqlens": None if seqlens is None else torch.from_numpy(seqlens).to(device),
        "pad_slot_id": pad_slot_id,
    }


def dense_prefill_bf16(seed=1011, device="cpu"):
    """Mixed varlen prefill over dense lines, the shapes of the chunked
    prefill step: 16 sequences of uniform 1-2048 new tokens, each resuming
    from its line when its cached prefix (uniform 0-2048) is non-empty;
    dim = 4096, W = 4, L = 3, bias, SiLU, lines drawn from a pool of 64."""
    rng = np.random.default_rng(seed)
    prefix = rng.integers(0, 2049, size=16)
    lens = rng.integers(1, 2049, size=16)
    return dense_conv_inputs(seed, dtype="bf16", dim=4096, W=4, state_len=3, lens=lens,
                             num_lines=64, has_init=prefix > 0, device=device)


def dense_long_prefill_bf16(seed=1012, device="cpu"):
    """One sequence of 65536 tokens from an empty line; dim = 8192 (the long
    SSM-style prefill), W = 4, L = 3, weight N(0, 0.3), bias, SiLU."""
    return dense_conv_inputs(seed, dtype="bf16", dim=8192, W=4, state_len=3, lens=[65536],
                             num_lines=1, has_init=[False], w_sigma=0.3, device=device)


def dense_decode_bf16(seed=1013, device="cpu"):
    """One decode token for each of 256 sequences, dim = 1024, W = 4, L = 3,
    shifted lines from a pool of 512, bias, SiLU."""
    return dense_update_inputs(seed, dtype="bf16", batch=256, dim=1024, W=4, state_len=3,
                               num_lines=512, device=device)


DENSE_NAMED = {
    "dense_prefill_bf16": dense_prefill_bf16,
    "dense_long_prefill_bf16": dense_long_prefill_bf16,
    "dense_decode_bf16": dense_decode_bf16,
}
