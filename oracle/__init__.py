"""CPU oracle for the fused short-convolution path -- TEST INFRASTRUCTURE ONLY.

This package wraps ``sconv_oracle.c``: a plain, scalar, double-precision
statement of what the path computes, written from the pages' definitions
("vllm.models.inkling.nvidia.ops.sconv": module docstring, fused_sconv,
sconv_seq_metadata; "core.ssm.ops.intermediate_extraction":
scatter_intermediate_conv / scatter_intermediate_ssm; "Implementation:Sgl
project Sglang Mamba Ops": causal_conv1d_fwd / causal_conv1d_update).
Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import it.  The CUDA library never calls it
and shares no code with it; the product path fails loudly without its own
extension instead of falling back here.

Every function takes numpy arrays or CPU torch tensors.  bf16 data is passed
as its raw 16-bit patterns (a torch bfloat16 tensor, or a numpy uint16 /
int16 array together with ``dtype="bf16"``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sconv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Plain build: no fast-math, no FMA contraction, so every double operation
# rounds exactly once in source order.
CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle C source into a shared library; returns its path."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, src, "-lm"], check=True)
        os.replace(tmp, out)
    return out


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int


def _bind(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    lib.oracle_fused.restype = _I64
    lib.oracle_fused.argtypes = [
        _INT, _P, _I64, _I64, _I64,            # dtype, x, x_row_stride, T, C
        _P, _I64, _I64, _INT,                  # weight, w_stride_c, w_stride_k, W
        _P, _P, _P, _I64, _I64, _I64, _I64,    # cache_in, cache_out, strides, nb, H, N, D
        _P, _P, _P, _P,                        # positions, seq_idx, slot_mapping, query_start
        _P, _I64, _I64, _I64,                  # block_table, bt_row_stride, num_reqs, max_blocks
        _I64, _I64, _INT, _INT,                # off_s, ws, silu, residual
        _I64, _I64, _P, _P, _P,                # t_begin, t_end, out_ref, row_state, write_index
    ]
    lib.oracle_seq_metadata.restype = None
    lib.oracle_seq_metadata.argtypes = [_P, _I64, _I64, _I64, _P, _P]
    lib.oracle_extract_windows.restype = None
    lib.oracle_extract_windows.argtypes = [
        _INT, _P, _I64, _I64, _I64, _I64, _P, _I64, _I64, _P, _I64, _I64]
    lib.oracle_scatter_ssm.restype = _I64
    lib.oracle_scatter_ssm.argtypes = [_INT, _P, _I64, _I64, _I64, _P, _I64, _I64, _P, _I64]
    lib.oracle_extract_windows_paged.restype = _I64
    lib.oracle_extract_windows_paged.argtypes = [
        _INT, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _I64, _I64, _I64, _P, _P, _I64,
        _I64, _P, _I64, _I64]
    lib.oracle_conv1d_fwd.restype = _I64
    lib.oracle_conv1d_fwd.argtypes = [
        _INT, _P, _I64, _I64, _I64, _I64,      # dtype, x, x_st, x_sc, total_tokens, dim
        _P, _I64, _I64, _INT, _P,              # weight, w_sc, w_sk, W, bias
        _P, _P, _I64, _I64, _I64, _I64, _I64,  # states in/out, strides, L, num_lines
        _P, _I64, _P, _P,                      # qsl, batch, cache_indices, has_init
        _INT, _I64, _P, _P,                    # silu, pad_slot_id, out_ref, row_state
    ]
    lib.oracle_conv1d_update.restype = _I64
    lib.oracle_conv1d_update.argtypes = [
        _INT, _P, _I64, _I64, _I64, _I64,      # dtype, x, x_sb, x_sc, batch, dim
        _P, _I64, _I64, _INT, _P,              # weight, w_sc, w_sk, W, bias
        _P, _P, _I64, _I64, _I64, _I64, _I64,  # states in/out, strides, L, num_lines
        _P, _P, _INT, _I64, _P, _P,            # cache_seqlens, indices, silu, pad, out, state
    ]
    lib.oracle_resolve_taps.restype = None
    lib.oracle_resolve_taps.argtypes = [
        _P, _I64, _I64, _I64,                  # query_start_loc, num_reqs, num_actual, num_padded
        _P, _P, _P, _I64, _I64, _I64, _I64,    # positions, slots, block_table, bt stride, max_blocks,
        _INT,                                  #   num_blocks, N; W
        _P, _P, _P,                            # seq_idx_out, query_start_out, taps
    ]
    lib.oracle_check_preconditions.restype = _INT
    lib.oracle_check_preconditions.argtypes = [
        _I64, _INT, _I64, _P, _P, _P, _P, _P, _I64, _I64]
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    """The oracle library.  SCONV_ORACLE_LIB names an alternative build
    (the mutation tests point it at deliberately broken copies)."""
    global _lib
    if _lib is None:
        alt = os.environ.get("SCONV_ORACLE_LIB")
        _lib = _bind(alt if alt else build())
    return _lib


# --------------------------------------------------------------------------
# array helpers

def _np(a, dtype=None):
    """Contiguous numpy view of a numpy array or CPU torch tensor."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            t = a.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                t = t.view(torch.int16)
            a = t.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if dtype is not None:
        if a.dtype != dtype:
            raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _float_array(a, dtype: str):
    """Raw element array for the oracle: float32 for 'f32', 16-bit for 'bf16'."""
    arr = _np(a)
    if dtype == "f32":
        if arr.dtype != np.float32:
            raise TypeError("f32 data must be float32")
    elif dtype == "bf16":
        if arr.dtype not in (np.int16, np.uint16):
            raise TypeError("bf16 data must be passed as 16-bit patterns")
        arr = arr.view(np.uint16)
    else:
        raise ValueError(dtype)
    return arr


def _ptr(a) -> int:
    return a.ctypes.data if a is not None else 0


_DT = {"f32": 0, "bf16": 1}


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact decode of bf16 bit patterns to float64."""
    b = _np(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def to_f64(a, dtype: str) -> np.ndarray:
    arr = _float_array(a, dtype)
    return arr.astype(np.float64) if dtype == "f32" else bf16_bits_to_f64(arr)


# --------------------------------------------------------------------------
# public oracle calls

def fused(*, dtype, x, weight, cache, positions, block_table, seq_idx,
          slot_mapping, query_start, off_s, ws, block_size, activation=None,
          use_residual=True, t_range=None, write_cache=True, write_index=False):
    """Oracle of fused_sconv ("vllm.models.inkling.nvidia.ops.sconv").

    ``cache`` is [num_blocks, H, N, D] (any strides in elements, D stride 1
    not required here).  Returns ``(out_ref, row_state, cache_out, skipped)``:
    out_ref float64 [n, C] for the tokens in ``t_range`` (default all),
    row_state uint8 [n] (1 computed, 0 PAD, 2 skipped), cache_out the cache
    after the inserts (a new array) or None when ``write_cache`` is False.
    With ``write_index`` a fifth value is returned: int64 [n, C], the flat
    cache element each (token, channel) is inserted at, -1 for none.
    """
    xa = _float_array(x, dtype)
    wa = _float_array(weight, dtype)
    ca = _float_array(cache, dtype)
    if xa.ndim != 2 or wa.ndim != 2 or ca.ndim != 4:
        raise ValueError("x [T,C], weight [C,W], cache [nb,H,N,D] expected")
    T, C = xa.shape
    W = wa.shape[1]
    nb, H, N, D = ca.shape
    if N != block_size:
        raise ValueError("cache.shape[2] must equal block_size")
    pos = _np(positions, np.int64)
    sid = _np(seq_idx, np.int32)
    slot = _np(slot_mapping, np.int64)
    qs = _np(query_start, np.int32)
    bt = _np(block_table, np.int32)
    t0, t1 = (0, T) if t_range is None else t_range
    n = t1 - t0
    out_ref = np.zeros((n, C), np.float64)
    state = np.zeros(n, np.uint8)
    cache_out = ca.copy() if write_cache else None
    widx = np.empty((n, C), np.int64) if write_index else None
    strides = np.array([s // ca.itemsize for s in ca.strides], np.int64)
    skipped = lib().oracle_fused(
        _DT[dtype], _ptr(xa), C, T, C, _ptr(wa), W, 1, W,
        _ptr(ca), _ptr(cache_out), _ptr(strides), nb, H, N, D,
        _ptr(pos), _ptr(sid), _ptr(slot), _ptr(qs),
        _ptr(bt), bt.shape[1], bt.shape[0], bt.shape[1],
        off_s, ws, int(activation in ("silu", "swish")), int(bool(use_residual)),
        t0, t1, _ptr(out_ref), _ptr(state), _ptr(widx))
    if skipped < 0:
        raise ValueError("oracle_fused: malformed arguments")
    if write_index:
        return out_ref, state, cache_out, int(skipped), widx
    return out_ref, state, cache_out, int(skipped)


def fused_streams(*, dtype, streams, cache, positions, block_table, seq_idx, slot_mapping,
                  query_start, block_size):
    """Several conv streams of one layer over one cache: by definition one
    fused_sconv per stream, every stream reading the cache as it was before
    the call (their lane ranges are disjoint, so no stream sees another's
    inserts).  ``streams``: dicts with x, weight, off_s, ws, activation,
    use_residual.  Returns (outs, states, cache_out, skipped)."""
    pre = _float_array(cache, dtype)
    cache_out = pre.copy()
    outs, states, skipped = [], [], 0
    for sd in streams:
        out, st, co, sk = fused(
            dtype=dtype, x=sd["x"], weight=sd["weight"], cache=pre, positions=positions,
            block_table=block_table, seq_idx=seq_idx, slot_mapping=slot_mapping,
            query_start=query_start, off_s=sd["off_s"], ws=sd["ws"], block_size=block_size,
            activation=sd.get("activation"), use_residual=sd.get("use_residual", True))
        changed = co.view(np.uint8).reshape(co.shape + (-1,)) != pre.view(np.uint8).reshape(
            pre.shape + (-1,))
        mask = changed.any(axis=-1)
        cache_out[mask] = co[mask]
        outs.append(out)
        states.append(st)
        skipped += sk
    return outs, states, cache_out, skipped


def update(*, dtype, x, weight, cache, positions, block_table, slot_mapping,
           off_s, ws, block_size, activation=None, use_residual=True,
           write_cache=True):
    """Oracle of the single-token decode form (causal_conv1d_update in
    "Implementation:Sgl project Sglang Mamba Ops"): token b is request b,
    so the fused definition applies with seq_idx[b] = query_start[b] = b."""
    B = _np(positions).shape[0]
    ar = np.arange(B, dtype=np.int32)
    return fused(dtype=dtype, x=x, weight=weight, cache=cache, positions=positions,
                 block_table=block_table, seq_idx=ar, slot_mapping=slot_mapping,
                 query_start=ar, off_s=off_s, ws=ws, block_size=block_size,
                 activation=activation, use_residual=use_residual,
                 write_cache=write_cache)


def seq_metadata(query_start_loc, num_reqs, num_actual_tokens, num_padded_tokens=None):
    """Oracle of sconv_seq_metadata; returns (seq_idx, query_start) int32."""
    qsl = _np(query_start_loc, np.int32)
    if num_padded_tokens is None:
        num_padded_tokens = num_actual_tokens
    si = np.zeros(num_padded_tokens, np.int32)
    qs = np.zeros(num_padded_tokens, np.int32)
    lib().oracle_seq_metadata(_ptr(qsl), num_reqs, num_actual_tokens,
                              num_padded_tokens, _ptr(si), _ptr(qs))
    return si, qs


# Entries of the resolved tap table (see oracle_resolve_taps).
SRC_X, SRC_ZERO = -2, -1


def resolve_taps(*, query_start_loc, num_reqs, num_actual_tokens, positions, slot_mapping,
                 block_table, num_blocks, block_size, W, num_padded_tokens=None):
    """Oracle of the per-step tap resolution: returns (seq_idx, query_start,
    taps) with taps int64 [num_padded, W-1] (lag d in column d-1): -2 for a
    same-forward x row, -1 for a zero tap, the flat cache slot of a
    pre-forward tap, or -(flags*256) when the token cannot be resolved.
    ``query_start_loc`` None is the decode form (token t is request t)."""
    if num_padded_tokens is None:
        num_padded_tokens = num_actual_tokens
    qsl = None if query_start_loc is None else _np(query_start_loc, np.int32)
    pos = _np(positions, np.int64)
    slot = _np(slot_mapping, np.int64)
    bt = _np(block_table, np.int32)
    if bt.ndim != 2:
        raise ValueError("block_table must be [num_reqs, max_blocks]")
    si = np.zeros(num_padded_tokens, np.int32)
    qs = np.zeros(num_padded_tokens, np.int32)
    taps = np.zeros((num_padded_tokens, max(W - 1, 0)), np.int64)
    lib().oracle_resolve_taps(_ptr(qsl), num_reqs, num_actual_tokens, num_padded_tokens,
                              _ptr(pos), _ptr(slot), _ptr(bt), bt.shape[1], bt.shape[1],
                              num_blocks, block_size, W, _ptr(si), _ptr(qs), _ptr(taps))
    return si, qs, taps


def extract_windows(*, dtype, src, abs_positions, real_count, out, d_conv):
    """Oracle of scatter_intermediate_conv ("core.ssm.ops.intermediate_extraction").

    ``src`` is [seq_len, conv_dim]; ``out`` [max_count, conv_dim, d_conv]
    holds the prior bytes.  Returns a new array with the gathered windows.
    """
    sa = _float_array(src, dtype)
    ap = _np(abs_positions, np.int32)
    oa = _float_array(out, dtype).copy()
    seq_len, conv_dim = sa.shape
    max_count = oa.shape[0]
    lib().oracle_extract_windows(
        _DT[dtype], _ptr(sa), seq_len, conv_dim, conv_dim, 1, _ptr(ap),
        int(real_count), max_count, _ptr(oa), conv_dim * d_conv, d_conv)
    return oa


def scatter_ssm(*, dtype, states, chunk_indices, real_count, out):
    """Oracle of scatter_intermediate_ssm ("core.ssm.ops.intermediate_extraction").
    ``states`` [num_chunks, ...] and ``out`` [max_count, ...] (same trailing
    shape); returns (a new out array, slots skipped for a bad index)."""
    sa = _float_array(states, dtype)
    oa = _float_array(out, dtype).copy()
    idx = _np(chunk_indices, np.int64)
    num_chunks = sa.shape[0]
    flat = int(np.prod(sa.shape[1:])) if sa.ndim > 1 else 1
    skipped = lib().oracle_scatter_ssm(_DT[dtype], _ptr(sa), num_chunks, flat, flat, _ptr(idx),
                                       int(real_count), oa.shape[0], _ptr(oa), flat)
    return oa, int(skipped)


def extract_windows_paged(*, dtype, cache, block_table, request, abs_positions, real_count,
                          out, d_conv, off_s, ws):
    """Window gather from the paged cache (sconv_extract_windows_paged):
    out [max_count, H*ws, d_conv] holds the prior bytes.  Returns (a new
    out array, slots skipped)."""
    ca = _float_array(cache, dtype)
    nb, H, N, D = ca.shape
    strides = np.array([st // ca.itemsize for st in ca.strides], np.int64)
    bt = _np(block_table, np.int32)
    rq = _np(request, np.int32)
    ap = _np(abs_positions, np.int32)
    oa = _float_array(out, dtype).copy()
    max_count = oa.shape[0]
    skipped = lib().oracle_extract_windows_paged(
        _DT[dtype], _ptr(ca), _ptr(strides), nb, H, N, off_s, ws, _ptr(bt), bt.shape[1],
        bt.shape[0], bt.shape[1], _ptr(rq), _ptr(ap), int(real_count), max_count, _ptr(oa),
        H * ws * d_conv, d_conv)
    if skipped < 0:
        raise ValueError("oracle_extract_windows_paged: malformed arguments")
    return oa, int(skipped)


def _dense_states(conv_states, dtype):
    """(states_in, states_out copy, L, num_lines) of a [num_lines, dim, L]
    state buffer, contiguous; (None, None, 0, 0) for no states."""
    if conv_states is None:
        return None, None, 0, 0
    sa = _float_array(conv_states, dtype)
    if sa.ndim != 3:
        raise ValueError("conv_states must be [num_lines, dim, state_len]")
    return sa, sa.copy(), sa.shape[2], sa.shape[0]


def conv1d_fwd(*, dtype, x, weight, bias=None, conv_states=None, query_start_loc,
               cache_indices=None, has_initial_state=None, activation=None,
               pad_slot_id=-1):
    """Oracle of causal_conv1d_fwd ("Implementation:Sgl project Sglang Mamba
    Ops") over x [total_tokens, dim] (token-major values; the layout the
    kernel reads is immaterial here).  Returns ``(out_ref, row_state,
    states_out, skipped)``: out_ref float64 [total_tokens, dim] (rows with
    row_state != 1 are zero), row_state uint8 [total_tokens], states_out the
    new [num_lines, dim, L] lines (None without conv_states)."""
    xa = _float_array(x, dtype)
    wa = _float_array(weight, dtype)
    if xa.ndim != 2 or wa.ndim != 2:
        raise ValueError("x [total_tokens, dim] and weight [dim, W] expected")
    T, dim = xa.shape
    W = wa.shape[1]
    ba = None if bias is None else _float_array(bias, dtype)
    s_in, s_out, L, lines = _dense_states(conv_states, dtype)
    qsl = _np(query_start_loc, np.int32)
    ci = None if cache_indices is None else _np(cache_indices, np.int32)
    hi = None if has_initial_state is None else _np(has_initial_state).astype(np.uint8)
    out_ref = np.zeros((T, dim), np.float64)
    state = np.zeros(T, np.uint8)
    skipped = lib().oracle_conv1d_fwd(
        _DT[dtype], _ptr(xa), dim, 1, T, dim, _ptr(wa), W, 1, W, _ptr(ba),
        _ptr(s_in), _ptr(s_out), dim * L, L, 1, L, lines,
        _ptr(qsl), qsl.shape[0] - 1, _ptr(ci), _ptr(hi),
        int(activation in ("silu", "swish")), int(pad_slot_id), _ptr(out_ref), _ptr(state))
    if skipped < 0:
        raise ValueError("oracle_conv1d_fwd: malformed arguments")
    return out_ref, state, s_out, int(skipped)


def conv1d_update(*, dtype, x, conv_state, weight, bias=None, activation=None,
                  cache_seqlens=None, conv_state_indices=None, pad_slot_id=-1):
    """Oracle of causal_conv1d_update ("Implementation:Sgl project Sglang
    Mamba Ops"): x [batch, dim], one token per sequence.  Returns
    ``(out_ref, row_state, states_out, skipped)``."""
    xa = _float_array(x, dtype)
    wa = _float_array(weight, dtype)
    B, dim = xa.shape
    W = wa.shape[1]
    ba = None if bias is None else _float_array(bias, dtype)
    s_in, s_out, L, lines = _dense_states(conv_state, dtype)
    if s_in is None:
        raise ValueError("conv_state is required")
    cs = None if cache_seqlens is None else _np(cache_seqlens, np.int32)
    ci = None if conv_state_indices is None else _np(conv_state_indices, np.int32)
    out_ref = np.zeros((B, dim), np.float64)
    state = np.zeros(B, np.uint8)
    skipped = lib().oracle_conv1d_update(
        _DT[dtype], _ptr(xa), dim, 1, B, dim, _ptr(wa), W, 1, W, _ptr(ba),
        _ptr(s_in), _ptr(s_out), dim * L, L, 1, L, lines, _ptr(cs), _ptr(ci),
        int(activation in ("silu", "swish")), int(pad_slot_id), _ptr(out_ref), _ptr(state))
    if skipped < 0:
        raise ValueError("oracle_conv1d_update: malformed arguments")
    return out_ref, state, s_out, int(skipped)


def check_preconditions(*, W, block_size, positions, seq_idx, slot_mapping,
                        query_start, block_table) -> int:
    """0 if one launch is well defined on these metadata, else 1..3
    (1 request rows not contiguous, 2 duplicate slots, 3 written slot read)."""
    pos = _np(positions, np.int64)
    sid = _np(seq_idx, np.int32)
    slot = _np(slot_mapping, np.int64)
    qs = _np(query_start, np.int32)
    bt = _np(block_table, np.int32)
    return int(lib().oracle_check_preconditions(
        pos.shape[0], W, block_size, _ptr(pos), _ptr(sid), _ptr(slot), _ptr(qs),
        _ptr(bt), bt.shape[1], bt.shape[1]))
