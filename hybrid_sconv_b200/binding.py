"""Thin Python binding of ``libsconv.so`` (the C ABI in include/sconv.h).

Argument marshalling only: each function checks tensor ranks and dtypes,
passes raw device pointers, element strides and the current CUDA stream to
the C entry point of the same name, and turns a non-zero status into an
exception.  Every step of the computation runs in the library's kernels; if
the library is missing the import fails loudly -- there is no fallback.
PyTorch provides device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsconv.so")

SCONV_OK, SCONV_ERR_INVALID, SCONV_ERR_UNSUPPORTED, SCONV_ERR_LAUNCH = 0, 1, 2, 3
SCONV_F32, SCONV_BF16 = 0, 1
SCONV_ACT_NONE, SCONV_ACT_SILU = 0, 1

# err_flag bits (SCONV_EFLAG_* in sconv.h)
EFLAG_SLOT, EFLAG_REQUEST, EFLAG_LOGICAL = 0x01, 0x02, 0x04
EFLAG_BLOCK, EFLAG_QUERY_START, EFLAG_POSITION = 0x08, 0x10, 0x20
EFLAG_TIMEOUT = 0x40

_DTYPES = {torch.float32: SCONV_F32, torch.bfloat16: SCONV_BF16}


class SconvError(RuntimeError):
    """A libsconv entry point returned a non-zero status."""

    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


_P, _I64, _INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
_I64P = ctypes.POINTER(ctypes.c_int64)
MAX_STREAMS = 4


class StreamDesc(ctypes.Structure):
    """sconv_stream_desc of sconv.h."""
    _fields_ = [("x", _P), ("x_row_stride", _I64), ("weight", _P), ("w_stride_c", _I64),
                ("w_stride_k", _I64), ("out", _P), ("out_row_stride", _I64), ("off_s", _INT),
                ("ws", _INT), ("act", _INT), ("use_residual", _INT)]


class TapsBuild(ctypes.Structure):
    """sconv_taps_build of sconv.h (one step's tap resolution)."""
    _fields_ = [("query_start_loc", _P), ("num_reqs", _INT), ("num_actual_tokens", _INT),
                ("num_padded_tokens", _INT), ("positions", _P), ("slot_mapping", _P),
                ("block_table", _P), ("bt_row_stride", _I64), ("max_blocks", _INT),
                ("seq_idx_out", _P), ("seq_idx_cap", _I64), ("query_start_out", _P),
                ("query_start_cap", _I64), ("taps_out", _P), ("taps_cap", _I64)]


_SIGNATURES = {
    "sconv_fused": [
        _P, _I64, _INT, _INT, _P, _I64, _I64, _INT,
        _P, _I64P, _I64, _INT, _INT, _INT,
        _P, _P, _P, _P,
        _P, _I64, _INT, _INT,
        _INT, _INT, _INT, _INT, _INT,
        _P, _I64, _P, _P],
    "sconv_fused_streams": [
        ctypes.POINTER(StreamDesc), _INT, _INT, _INT,
        _P, _I64P, _I64, _INT, _INT, _INT,
        _P, _P, _P, _P,
        _P, _I64, _INT, _INT,
        _INT, _P, _P],
    "sconv_update": [
        _P, _I64, _INT, _INT, _P, _I64, _I64, _INT,
        _P, _I64P, _I64, _INT, _INT, _INT,
        _P, _P,
        _P, _I64, _INT,
        _INT, _INT, _INT, _INT, _INT,
        _P, _I64, _P, _P],
    "sconv_extract_windows": [
        _P, _I64, _INT, _I64, _I64, _P, _P, _INT, _P, _I64, _INT, _INT, _P],
    "sconv_seq_metadata": [_P, _INT, _INT, _INT, _P, _I64, _P, _I64, _P],
    "sconv_seq_metadata_taps": [
        _P, _INT, _INT, _INT, _P, _P, _P, _I64, _INT, _I64, _INT, _INT,
        _P, _I64, _P, _I64, _P, _I64, _P],
    "sconv_seq_metadata_taps_ahead": [
        _P, _INT, _INT, _INT, _P, _P, _P, _I64, _INT, _I64, _INT, _INT,
        _P, _I64, _P, _I64, _P, _I64, _P],
    "sconv_fused_taps": [
        ctypes.POINTER(StreamDesc), _INT, _INT, _INT,
        _P, _I64P, _I64, _INT, _INT, _INT,
        _P, _P, _INT, _INT, _P, _P],
    "sconv_fused_taps_next": [
        ctypes.POINTER(StreamDesc), _INT, _INT, _INT,
        _P, _I64P, _I64, _INT, _INT, _INT,
        _P, _P, _INT, _P, ctypes.POINTER(TapsBuild), _P],
    "sconv_seq_metadata_ahead": [_P, _INT, _INT, _INT, _P, _I64, _P, _I64, _P],
    "sconv_scatter_intermediate_ssm": [
        _P, _I64, _I64, _I64, _P, _P, _INT, _P, _I64, _INT, _P, _P],
    "sconv_causal_conv1d_fwd": [
        _P, _I64, _I64, _INT, _INT, _P, _I64, _I64, _INT, _P,
        _P, _I64, _I64, _I64, _INT, _INT, _P, _INT, _P, _P, _INT, _INT, _P, _INT, _P, _P],
    "sconv_causal_conv1d_update": [
        _P, _I64, _I64, _INT, _INT, _P, _I64, _I64, _INT, _P,
        _P, _I64, _I64, _I64, _INT, _INT, _P, _P, _INT, _INT, _P, _INT, _P, _P],
    "sconv_extract_windows_paged": [
        _P, _I64P, _I64, _INT, _INT, _INT, _INT, _INT, _P, _I64, _INT, _INT, _P, _P, _P, _INT,
        _P, _I64, _INT, _INT, _P, _P],
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is not built; run `python -m hybrid_sconv_b200.build` "
            "(the sconv ops have no fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, args in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = _INT
    lib.sconv_status_string.argtypes = [_INT]
    lib.sconv_status_string.restype = ctypes.c_char_p
    lib.sconv_abi_version.argtypes = []
    lib.sconv_abi_version.restype = _INT
    if lib.sconv_abi_version() != 1:
        raise ImportError("libsconv.so ABI version mismatch; rebuild it")
    return lib


LIB = _load()
LIB_PATH = _LIB_PATH


def _check(fn: str, status: int, value_error: bool = False) -> None:
    if status != SCONV_OK:
        msg = LIB.sconv_status_string(status).decode()
        if value_error and status == SCONV_ERR_INVALID:
            raise ValueError(f"{fn}: {msg}")
        raise SconvError(fn, status, msg)


def _dev(*tensors: torch.Tensor) -> torch.device:
    d = tensors[0].device
    if d.type != "cuda":
        raise ValueError("sconv ops take CUDA tensors")
    for t in tensors[1:]:
        if t is not None and t.device != d:
            raise ValueError("all tensors must be on the same CUDA device")
    return d


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.data_ptr()


def _want(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _vector(t: torch.Tensor, dtype: torch.dtype, name: str, n: int) -> None:
    _want(t, dtype, name)
    if t.dim() != 1 or t.shape[0] < n or (n > 0 and t.stride(0) != 1):
        raise ValueError(f"{name} must be a contiguous 1-D tensor of at least {n} elements")


def _act(activation) -> int:
    # As in fused_sconv: "silu" and "swish" select SiLU, anything else none.
    return SCONV_ACT_SILU if activation in ("silu", "swish") else SCONV_ACT_NONE


def _stream(device, stream) -> int:
    s = torch.cuda.current_stream(device) if stream is None else stream
    return s.cuda_stream


def _float_common(x, weight, cache):
    dt = _DTYPES.get(x.dtype)
    if dt is None:
        raise TypeError("x must be float32 or bfloat16")
    if weight.dtype != x.dtype or cache.dtype != x.dtype:
        raise TypeError("x, weight and cache must share one dtype")
    if x.dim() != 2 or weight.dim() != 2 or cache.dim() != 4:
        raise ValueError("x [T, C], weight [C, W] and cache [num_blocks, H, N, D] expected")
    if x.shape[0] > 0 and x.stride(1) != 1:
        raise ValueError("x must have unit channel stride")
    if weight.shape[0] != x.shape[1]:
        raise ValueError("weight must be [C, W]")
    return dt


def sconv_fused(x, weight, cache, positions, block_table, seq_idx, slot_mapping,
                query_start, off_s, ws, block_size, activation=None, use_residual=True, *,
                out=None, err_flag=None, stream=None):
    """Insert + depthwise causal conv1d over the paged cache in one launch
    (fused_sconv, "vllm.models.inkling.nvidia.ops.sconv").  Returns ``out``
    ([T, C], allocated like x when not given).  See sconv.h for layouts."""
    dt = _float_common(x, weight, cache)
    T, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    if T == 0:
        return out
    d = _dev(x, weight, cache, positions, block_table, seq_idx, slot_mapping, query_start,
             out, err_flag)
    _vector(positions, torch.int64, "positions", T)
    _vector(seq_idx, torch.int32, "seq_idx", T)
    _vector(slot_mapping, torch.int64, "slot_mapping", T)
    _vector(query_start, torch.int32, "query_start", T)
    _want(block_table, torch.int32, "block_table")
    if block_table.dim() != 2 or block_table.stride(1) != 1:
        raise ValueError("block_table must be [num_reqs, max_blocks] with unit inner stride")
    if out.dtype != x.dtype or out.dim() != 2 or tuple(out.shape) != (T, C) or out.stride(1) != 1:
        raise ValueError("out must be [T, C] like x with unit channel stride")
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    if cache.shape[2] != block_size:
        raise ValueError("cache.shape[2] must equal block_size")
    nb, H, N, D = cache.shape
    cs = (ctypes.c_int64 * 4)(*cache.stride())
    with torch.cuda.device(d):
        st = LIB.sconv_fused(
            _ptr(x), x.stride(0), T, C, _ptr(weight), weight.stride(0), weight.stride(1),
            weight.shape[1], _ptr(cache), cs, nb, H, N, D,
            _ptr(positions), _ptr(seq_idx), _ptr(slot_mapping), _ptr(query_start),
            _ptr(block_table), block_table.stride(0), block_table.shape[0],
            block_table.shape[1], off_s, ws, _act(activation), int(bool(use_residual)), dt,
            _ptr(out), out.stride(0), _ptr(err_flag), _stream(d, stream))
    _check("sconv_fused", st)
    return out


def sconv_fused_streams(streams, cache, positions, block_table, seq_idx, slot_mapping,
                        query_start, block_size, *, err_flag=None, stream=None):
    """Several conv streams of one layer in one call (sconv_fused_streams in
    sconv.h): the same tokens, metadata and cache, disjoint lane ranges.
    ``streams`` is a sequence of dicts with keys ``x``, ``weight``,
    ``off_s``, ``ws`` and optionally ``activation``, ``use_residual``
    (default True, as in fused_sconv) and ``out``.  Returns the outputs."""
    if not 1 <= len(streams) <= MAX_STREAMS:
        raise ValueError(f"1..{MAX_STREAMS} streams per call")
    x0 = streams[0]["x"]
    dt = _float_common(x0, streams[0]["weight"], cache)
    T = x0.shape[0]
    outs = []
    descs = (StreamDesc * len(streams))()
    for i, sd in enumerate(streams):
        x, w = sd["x"], sd["weight"]
        _float_common(x, w, cache)
        if x.shape[0] != T or w.shape[1] != streams[0]["weight"].shape[1]:
            raise ValueError("all streams share T and W")
        out = sd.get("out")
        if out is None:
            out = torch.empty_like(x)
        if out.dtype != x.dtype or tuple(out.shape) != tuple(x.shape) or (T and out.stride(1) != 1):
            raise ValueError("out must be [T, C] like x with unit channel stride")
        outs.append(out)
        descs[i] = StreamDesc(_ptr(x), x.stride(0), _ptr(w), w.stride(0), w.stride(1), _ptr(out),
                              out.stride(0), sd["off_s"], sd["ws"], _act(sd.get("activation")),
                              int(bool(sd.get("use_residual", True))))
    if T == 0:
        return outs
    d = _dev(x0, cache, positions, block_table, seq_idx, slot_mapping, query_start, err_flag,
             *[sd["x"] for sd in streams], *[sd["weight"] for sd in streams], *outs)
    _vector(positions, torch.int64, "positions", T)
    _vector(seq_idx, torch.int32, "seq_idx", T)
    _vector(slot_mapping, torch.int64, "slot_mapping", T)
    _vector(query_start, torch.int32, "query_start", T)
    _want(block_table, torch.int32, "block_table")
    if block_table.dim() != 2 or block_table.stride(1) != 1:
        raise ValueError("block_table must be [num_reqs, max_blocks] with unit inner stride")
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    if cache.shape[2] != block_size:
        raise ValueError("cache.shape[2] must equal block_size")
    nb, H, N, D = cache.shape
    cs = (ctypes.c_int64 * 4)(*cache.stride())
    with torch.cuda.device(d):
        st = LIB.sconv_fused_streams(
            descs, len(streams), T, streams[0]["weight"].shape[1], _ptr(cache), cs, nb, H, N, D,
            _ptr(positions), _ptr(seq_idx), _ptr(slot_mapping), _ptr(query_start),
            _ptr(block_table), block_table.stride(0), block_table.shape[0],
            block_table.shape[1], dt, _ptr(err_flag), _stream(d, stream))
    _check("sconv_fused_streams", st)
    return outs


def sconv_update(x, weight, cache, positions, block_table, slot_mapping, off_s, ws,
                 block_size, activation=None, use_residual=True, *, out=None,
                 err_flag=None, stream=None):
    """Single-token decode: token b is request b (block_table row b).  Same
    result as sconv_fused with seq_idx = query_start = arange(B)."""
    dt = _float_common(x, weight, cache)
    B, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    if B == 0:
        return out
    d = _dev(x, weight, cache, positions, block_table, slot_mapping, out, err_flag)
    _vector(positions, torch.int64, "positions", B)
    _vector(slot_mapping, torch.int64, "slot_mapping", B)
    _want(block_table, torch.int32, "block_table")
    if block_table.dim() != 2 or block_table.shape[0] < B or block_table.stride(1) != 1:
        raise ValueError("block_table must be [>= B, max_blocks] with unit inner stride")
    if out.dtype != x.dtype or tuple(out.shape) != (B, C) or out.stride(1) != 1:
        raise ValueError("out must be [B, C] like x with unit channel stride")
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    if cache.shape[2] != block_size:
        raise ValueError("cache.shape[2] must equal block_size")
    nb, H, N, D = cache.shape
    cs = (ctypes.c_int64 * 4)(*cache.stride())
    with torch.cuda.device(d):
        st = LIB.sconv_update(
            _ptr(x), x.stride(0), B, C, _ptr(weight), weight.stride(0), weight.stride(1),
            weight.shape[1], _ptr(cache), cs, nb, H, N, D, _ptr(positions),
            _ptr(slot_mapping), _ptr(block_table), block_table.stride(0),
            block_table.shape[1], off_s, ws, _act(activation), int(bool(use_residual)), dt,
            _ptr(out), out.stride(0), _ptr(err_flag), _stream(d, stream))
    _check("sconv_update", st)
    return out


def sconv_extract_windows(src, abs_positions, real_count, out, d_conv, *, stream=None):
    """Gather the d_conv-long windows [pos - d_conv, pos) of ``src`` for the
    first ``real_count[0]`` slots into ``out[slot, conv_dim, d_conv]``
    (scatter_intermediate_conv, "core.ssm.ops.intermediate_extraction").
    ``src`` is [seq_len, conv_dim] or [batch, seq_len, conv_dim] (batch 0 is
    read); ``real_count`` is a device int32[1]."""
    if src.dim() == 3:
        src = src[0]
    if src.dim() != 2:
        raise ValueError("src must be [seq_len, conv_dim] or [batch, seq_len, conv_dim]")
    dt = _DTYPES.get(src.dtype)
    if dt is None or out.dtype != src.dtype:
        raise TypeError("src and out must share one dtype, float32 or bfloat16")
    max_count = out.shape[0]
    if max_count == 0:
        return out
    d = _dev(src, abs_positions, real_count, out)
    _vector(abs_positions, torch.int32, "abs_positions", max_count)
    _vector(real_count, torch.int32, "real_count", 1)
    seq_len, conv_dim = src.shape
    if out.dim() != 3 or out.shape[1] != conv_dim or out.shape[2] != d_conv or \
            out.stride(2) != 1 or out.stride(1) != d_conv:
        raise ValueError("out must be [max_count, conv_dim, d_conv] with dense inner dims")
    with torch.cuda.device(d):
        st = LIB.sconv_extract_windows(
            _ptr(src), seq_len, conv_dim, src.stride(0), src.stride(1),
            _ptr(abs_positions), _ptr(real_count), max_count, _ptr(out), out.stride(0),
            d_conv, dt, _stream(d, stream))
    _check("sconv_extract_windows", st)
    return out


def sconv_scatter_intermediate_ssm(states, chunk_indices, real_count, out, *, err_flag=None,
                                   stream=None):
    """Gather rows of ``states`` [num_chunks, *state_shape] at
    ``chunk_indices`` (int64 [max_count]) into ``out`` [max_count,
    *state_shape] for the first ``real_count[0]`` slots only
    (scatter_intermediate_ssm, "core.ssm.ops.intermediate_extraction")."""
    dt = _DTYPES.get(states.dtype)
    if dt is None or out.dtype != states.dtype:
        raise TypeError("states and out must share one dtype, float32 or bfloat16")
    max_count = out.shape[0]
    if max_count == 0:
        return out
    if tuple(out.shape[1:]) != tuple(states.shape[1:]):
        raise ValueError("out must be [max_count, *states.shape[1:]]")
    st2 = states.reshape(states.shape[0], -1)
    out2 = out.view(max_count, -1)
    if st2.shape[0] and st2.stride(1) != 1 or out2.stride(1) != 1:
        raise ValueError("state rows must be contiguous")
    d = _dev(states, chunk_indices, real_count, out, err_flag)
    _vector(chunk_indices, torch.int64, "chunk_indices", max_count)
    _vector(real_count, torch.int32, "real_count", 1)
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    with torch.cuda.device(d):
        st = LIB.sconv_scatter_intermediate_ssm(
            _ptr(st2), st2.shape[0], st2.shape[1], st2.stride(0) if st2.shape[0] else st2.shape[1],
            _ptr(chunk_indices), _ptr(real_count), max_count, _ptr(out2), out2.stride(0), dt,
            _ptr(err_flag), _stream(d, stream))
    _check("sconv_scatter_intermediate_ssm", st)
    return out


def sconv_extract_windows_paged(cache, block_table, request, abs_positions, real_count, out,
                                d_conv, off_s, ws, *, err_flag=None, stream=None):
    """Windows [pos - d_conv, pos) of each slot's request read from the
    paged cache [num_blocks, H, N, D] through ``block_table`` into ``out``
    [max_count, H*ws, d_conv], for the first ``real_count[0]`` slots."""
    dt = _DTYPES.get(cache.dtype)
    if dt is None or out.dtype != cache.dtype:
        raise TypeError("cache and out must share one dtype, float32 or bfloat16")
    max_count = out.shape[0]
    if max_count == 0:
        return out
    nb, H, N, D = cache.shape
    if out.dim() != 3 or out.shape[1] != H * ws or out.shape[2] != d_conv or             out.stride(2) != 1 or out.stride(1) != d_conv:
        raise ValueError("out must be [max_count, H*ws, d_conv] with dense inner dims")
    d = _dev(cache, block_table, request, abs_positions, real_count, out, err_flag)
    _vector(request, torch.int32, "request", max_count)
    _vector(abs_positions, torch.int32, "abs_positions", max_count)
    _vector(real_count, torch.int32, "real_count", 1)
    _want(block_table, torch.int32, "block_table")
    if block_table.dim() != 2 or block_table.stride(1) != 1:
        raise ValueError("block_table must be [num_reqs, max_blocks] with unit inner stride")
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    cs = (ctypes.c_int64 * 4)(*cache.stride())
    with torch.cuda.device(d):
        st = LIB.sconv_extract_windows_paged(
            _ptr(cache), cs, nb, H, N, D, off_s, ws, _ptr(block_table), block_table.stride(0),
            block_table.shape[0], block_table.shape[1], _ptr(request), _ptr(abs_positions),
            _ptr(real_count), max_count, _ptr(out), out.stride(0), d_conv, dt, _ptr(err_flag),
            _stream(d, stream))
    _check("sconv_extract_windows_paged", st)
    return out


def _seq_metadata(name, query_start_loc, num_reqs, num_actual_tokens, seq_idx_out,
                  query_start_out, num_padded_tokens, stream):
    if num_padded_tokens is None:
        num_padded_tokens = num_actual_tokens
    if num_padded_tokens < num_actual_tokens:
        raise ValueError("num_padded_tokens must cover all actual tokens")
    if num_padded_tokens > seq_idx_out.shape[0]:
        raise ValueError("seq_idx_out is too small for the padded token count")
    if num_padded_tokens > query_start_out.shape[0]:
        raise ValueError("query_start_out is too small for the padded token count")
    if num_padded_tokens == 0:
        return
    d = _dev(query_start_loc, seq_idx_out, query_start_out)
    _vector(query_start_loc, torch.int32, "query_start_loc", num_reqs + 1)
    _vector(seq_idx_out, torch.int32, "seq_idx_out", num_padded_tokens)
    _vector(query_start_out, torch.int32, "query_start_out", num_padded_tokens)
    with torch.cuda.device(d):
        st = getattr(LIB, name)(
            _ptr(query_start_loc), num_reqs, num_actual_tokens, num_padded_tokens,
            _ptr(seq_idx_out), seq_idx_out.shape[0], _ptr(query_start_out),
            query_start_out.shape[0], _stream(d, stream))
    _check(name, st, value_error=True)


def sconv_seq_metadata(query_start_loc, num_reqs, num_actual_tokens, seq_idx_out,
                       query_start_out, num_padded_tokens=None, *, stream=None):
    """Fill seq_idx_out / query_start_out for every token row in one launch
    (sconv_seq_metadata, "vllm.models.inkling.nvidia.ops.sconv").  Raises
    ValueError on the size errors the page names."""
    _seq_metadata("sconv_seq_metadata", query_start_loc, num_reqs, num_actual_tokens,
                  seq_idx_out, query_start_out, num_padded_tokens, stream)


def sconv_seq_metadata_ahead(query_start_loc, num_reqs, num_actual_tokens, seq_idx_out,
                             query_start_out, num_padded_tokens=None, *, stream=None):
    """sconv_seq_metadata with the lookup done before the launch waits for
    the kernels ahead of it on the stream (it still completes after them).
    The caller guarantees that no kernel enqueued since the stream was last
    fully ordered writes query_start_loc or touches the two outputs, e.g.
    one metadata buffer set per step in flight."""
    _seq_metadata("sconv_seq_metadata_ahead", query_start_loc, num_reqs, num_actual_tokens,
                  seq_idx_out, query_start_out, num_padded_tokens, stream)


# Entries of the resolved tap table (SCONV_TAP_* in sconv.h).
TAP_ZERO, TAP_X = -1, -2


def _seq_metadata_taps(name, query_start_loc, num_reqs, num_actual_tokens, positions,
                       slot_mapping, block_table, num_blocks, block_size, W, seq_idx_out,
                       query_start_out, taps_out, num_padded_tokens, stream):
    if num_padded_tokens is None:
        num_padded_tokens = num_actual_tokens
    if taps_out is None:
        taps_out = torch.empty((num_padded_tokens, max(W - 1, 0)), dtype=torch.int64,
                               device=positions.device)
    d = _dev(positions, slot_mapping, block_table, query_start_loc, seq_idx_out,
             query_start_out, taps_out)
    _vector(positions, torch.int64, "positions", num_actual_tokens)
    _vector(slot_mapping, torch.int64, "slot_mapping", num_actual_tokens)
    _want(block_table, torch.int32, "block_table")
    if block_table.dim() != 2 or block_table.stride(1) != 1:
        raise ValueError("block_table must be [rows, max_blocks] with unit inner stride")
    if query_start_loc is not None:
        _vector(query_start_loc, torch.int32, "query_start_loc", num_reqs + 1)
    for t, nm in ((seq_idx_out, "seq_idx_out"), (query_start_out, "query_start_out")):
        if t is not None:
            _vector(t, torch.int32, nm, num_padded_tokens)
    _want(taps_out, torch.int64, "taps_out")
    if not taps_out.is_contiguous():
        raise ValueError("taps_out must be contiguous")
    with torch.cuda.device(d):
        st = getattr(LIB, name)(
            _ptr(query_start_loc), num_reqs, num_actual_tokens, num_padded_tokens,
            _ptr(positions), _ptr(slot_mapping), _ptr(block_table), block_table.stride(0),
            block_table.shape[1], num_blocks, block_size, W,
            _ptr(seq_idx_out), seq_idx_out.numel() if seq_idx_out is not None else 0,
            _ptr(query_start_out), query_start_out.numel() if query_start_out is not None else 0,
            _ptr(taps_out), taps_out.numel(), _stream(d, stream))
    _check(name, st, value_error=True)
    return taps_out


def sconv_seq_metadata_taps(query_start_loc, num_reqs, num_actual_tokens, positions,
                            slot_mapping, block_table, num_blocks, block_size, W, *,
                            seq_idx_out=None, query_start_out=None, taps_out=None,
                            num_padded_tokens=None, stream=None):
    """sconv_seq_metadata plus every token's pre-forward taps resolved into
    a [num_padded, W-1] int64 table (sconv_seq_metadata_taps in sconv.h):
    TAP_X for a same-forward x row, TAP_ZERO before position 0, the flat
    cache slot of a pre-forward tap, or -(flags << 8) for a token that cannot
    be resolved.  ``query_start_loc`` None is the decode form (token t is
    request t, ``num_reqs`` the block-table rows).  seq_idx_out /
    query_start_out are written when given.  Returns the table."""
    return _seq_metadata_taps("sconv_seq_metadata_taps", query_start_loc, num_reqs,
                              num_actual_tokens, positions, slot_mapping, block_table,
                              num_blocks, block_size, W, seq_idx_out, query_start_out, taps_out,
                              num_padded_tokens, stream)


def sconv_seq_metadata_taps_ahead(query_start_loc, num_reqs, num_actual_tokens, positions,
                                  slot_mapping, block_table, num_blocks, block_size, W, *,
                                  seq_idx_out=None, query_start_out=None, taps_out=None,
                                  num_padded_tokens=None, stream=None):
    """sconv_seq_metadata_taps with its work done before the launch waits
    for the kernels ahead of it on the stream (same precondition as
    sconv_seq_metadata_ahead, extended to positions, slot_mapping, the block
    table and the table)."""
    return _seq_metadata_taps("sconv_seq_metadata_taps_ahead", query_start_loc, num_reqs,
                              num_actual_tokens, positions, slot_mapping, block_table,
                              num_blocks, block_size, W, seq_idx_out, query_start_out, taps_out,
                              num_padded_tokens, stream)


def sconv_fused_streams_taps(streams, cache, slot_mapping, taps, block_size, *,
                             metadata_ready=False, err_flag=None, stream=None):
    """The fused step of sconv_fused_streams with every token's taps read
    from a table of sconv_seq_metadata_taps (sconv_fused_taps in sconv.h).
    ``streams`` as in sconv_fused_streams.  metadata_ready=True lets the
    launch read slot_mapping and the table before waiting for the kernels
    it depends on; the caller guarantees the precondition sconv.h states
    (e.g. another call of this library, not an *_ahead builder, between
    the builder and this call on one stream; an event join from another
    stream does not suffice under graph capture).  Returns the outputs."""
    if not 1 <= len(streams) <= MAX_STREAMS:
        raise ValueError(f"1..{MAX_STREAMS} streams per call")
    x0 = streams[0]["x"]
    dt = _float_common(x0, streams[0]["weight"], cache)
    T = x0.shape[0]
    W = streams[0]["weight"].shape[1]
    outs = []
    descs = (StreamDesc * len(streams))()
    for i, sd in enumerate(streams):
        x, w = sd["x"], sd["weight"]
        _float_common(x, w, cache)
        if x.shape[0] != T or w.shape[1] != W:
            raise ValueError("all streams share T and W")
        out = sd.get("out")
        if out is None:
            out = torch.empty_like(x)
        if out.dtype != x.dtype or tuple(out.shape) != tuple(x.shape) or (T and out.stride(1) != 1):
            raise ValueError("out must be [T, C] like x with unit channel stride")
        outs.append(out)
        descs[i] = StreamDesc(_ptr(x), x.stride(0), _ptr(w), w.stride(0), w.stride(1), _ptr(out),
                              out.stride(0), sd["off_s"], sd["ws"], _act(sd.get("activation")),
                              int(bool(sd.get("use_residual", True))))
    if T == 0:
        return outs
    d = _dev(x0, cache, slot_mapping, taps, err_flag, *[sd["x"] for sd in streams],
             *[sd["weight"] for sd in streams], *outs)
    _vector(slot_mapping, torch.int64, "slot_mapping", T)
    if W > 1:
        _want(taps, torch.int64, "taps")
        if taps.dim() != 2 or taps.shape[0] < T or taps.shape[1] != W - 1 or \
                not taps.is_contiguous():
            raise ValueError("taps must be a contiguous [>= T, W-1] int64 table")
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    if cache.shape[2] != block_size:
        raise ValueError("cache.shape[2] must equal block_size")
    nb, H, N, D = cache.shape
    cs = (ctypes.c_int64 * 4)(*cache.stride())
    with torch.cuda.device(d):
        st = LIB.sconv_fused_taps(
            descs, len(streams), T, W, _ptr(cache), cs, nb, H, N, D, _ptr(slot_mapping),
            _ptr(taps) if W > 1 else 0, int(bool(metadata_ready)), dt, _ptr(err_flag),
            _stream(d, stream))
    _check("sconv_fused_taps", st)
    return outs


def sconv_fused_taps_next(x, weight, cache, slot_mapping, taps, off_s, ws, block_size,
                          activation=None, use_residual=True, *, next_step, out=None,
                          err_flag=None, stream=None):
    """One decode-loop step in one launch (sconv_fused_taps_next in
    sconv.h): this step's fused convolution reading ``taps`` (after the
    launch's wait), and the next step's tap table built by extra blocks of
    the same launch.  ``next_step`` is a dict with the arguments of
    sconv_seq_metadata_taps for that step: query_start_loc (or None),
    num_reqs, num_actual_tokens, positions, slot_mapping, block_table,
    taps_out, and optionally seq_idx_out, query_start_out,
    num_padded_tokens.  Returns ``out``."""
    dt = _float_common(x, weight, cache)
    T, C = x.shape
    W = weight.shape[1]
    if out is None:
        out = torch.empty_like(x)
    n = next_step
    npad = n.get("num_padded_tokens")
    npad = n["num_actual_tokens"] if npad is None else npad
    bt = n["block_table"]
    _want(bt, torch.int32, "next block_table")
    if bt.dim() != 2 or bt.stride(1) != 1:
        raise ValueError("next block_table must be [rows, max_blocks] with unit inner stride")
    _vector(n["positions"], torch.int64, "next positions", n["num_actual_tokens"])
    _vector(n["slot_mapping"], torch.int64, "next slot_mapping", n["num_actual_tokens"])
    if n.get("query_start_loc") is not None:
        _vector(n["query_start_loc"], torch.int32, "next query_start_loc", n["num_reqs"] + 1)
    for k in ("seq_idx_out", "query_start_out"):
        if n.get(k) is not None:
            _vector(n[k], torch.int32, k, npad)
    tout = n["taps_out"]
    _want(tout, torch.int64, "taps_out")
    if not tout.is_contiguous():
        raise ValueError("taps_out must be contiguous")
    d = _dev(x, weight, cache, slot_mapping, taps, out, err_flag, bt, n["positions"],
             n["slot_mapping"], tout)
    if T:
        _vector(slot_mapping, torch.int64, "slot_mapping", T)
        if out.dtype != x.dtype or tuple(out.shape) != (T, C) or out.stride(1) != 1:
            raise ValueError("out must be [T, C] like x with unit channel stride")
    if W > 1 and T:
        _want(taps, torch.int64, "taps")
        if taps.dim() != 2 or taps.shape[0] < T or taps.shape[1] != W - 1 or \
                not taps.is_contiguous():
            raise ValueError("taps must be a contiguous [>= T, W-1] int64 table")
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    if cache.shape[2] != block_size:
        raise ValueError("cache.shape[2] must equal block_size")
    nb, H, N, D = cache.shape
    cs = (ctypes.c_int64 * 4)(*cache.stride())
    desc = (StreamDesc * 1)(StreamDesc(_ptr(x), x.stride(0), _ptr(weight), weight.stride(0),
                                       weight.stride(1), _ptr(out), out.stride(0), off_s, ws,
                                       _act(activation), int(bool(use_residual))))
    si, qs = n.get("seq_idx_out"), n.get("query_start_out")
    build = TapsBuild(_ptr(n.get("query_start_loc")), n["num_reqs"], n["num_actual_tokens"],
                      npad, _ptr(n["positions"]), _ptr(n["slot_mapping"]), _ptr(bt),
                      bt.stride(0), bt.shape[1], _ptr(si), si.numel() if si is not None else 0,
                      _ptr(qs), qs.numel() if qs is not None else 0, _ptr(tout), tout.numel())
    with torch.cuda.device(d):
        st = LIB.sconv_fused_taps_next(
            desc, 1, T, W, _ptr(cache), cs, nb, H, N, D, _ptr(slot_mapping),
            _ptr(taps) if (W > 1 and T) else 0, dt, _ptr(err_flag), ctypes.byref(build),
            _stream(d, stream))
    _check("sconv_fused_taps_next", st)
    return out


def sconv_fused_taps(x, weight, cache, slot_mapping, taps, off_s, ws, block_size,
                     activation=None, use_residual=True, *, out=None, metadata_ready=False,
                     err_flag=None, stream=None):
    """sconv_fused with the tap sources read from a table built by
    sconv_seq_metadata_taps for the same step (one conv stream).  Same
    result as sconv_fused on the metadata the table was built from."""
    return sconv_fused_streams_taps(
        [dict(x=x, weight=weight, off_s=off_s, ws=ws, activation=activation,
              use_residual=use_residual, out=out)], cache, slot_mapping, taps, block_size,
        metadata_ready=metadata_ready, err_flag=err_flag, stream=stream)[0]


def _dense_common(x, weight, bias, states, out, err_flag, states_name):
    dt = _DTYPES.get(x.dtype)
    if dt is None:
        raise TypeError("x must be float32 or bfloat16")
    for t, name in ((weight, "weight"), (bias, "bias"), (states, states_name), (out, "out")):
        if t is not None and t.dtype != x.dtype:
            raise TypeError(f"{name} must have x's dtype")
    if x.dim() != 2 or weight.dim() != 2 or weight.shape[0] != x.shape[1]:
        raise ValueError("x [rows, dim] and weight [dim, W] expected")
    dim = x.shape[1]
    if bias is not None and (bias.dim() != 1 or bias.shape[0] != dim or bias.stride(0) != 1):
        raise ValueError("bias must be a contiguous [dim] tensor")
    if states is not None and (states.dim() != 3 or states.shape[1] != dim):
        raise ValueError(f"{states_name} must be [num_lines, dim, state_len]")
    if out.shape != x.shape or out.stride() != x.stride():
        raise ValueError("out must have x's shape and strides")
    if err_flag is not None:
        _vector(err_flag, torch.int32, "err_flag", 1)
    return dt


def sconv_causal_conv1d_fwd(x, weight, bias, conv_states, query_start_loc, cache_indices,
                            has_initial_state, silu_activation, pad_slot_id=-1, *, out=None,
                            err_flag=None, stream=None):
    """Varlen prefill over dense state lines (causal_conv1d_fwd,
    "Implementation:Sgl project Sglang Mamba Ops"), in place by default.

    x [total_tokens, dim] with any strides (a channel-major [dim, T] buffer
    is passed as its transpose view); weight [dim, W]; bias [dim] or None;
    conv_states [num_lines, dim, state_len] (any strides) or None;
    query_start_loc int32 [batch+1]; cache_indices int32 [batch] or None;
    has_initial_state bool/uint8 [batch] or None.  Writes the outputs into
    ``out`` (default: x itself) and the new lines into conv_states; returns
    ``out``."""
    if out is None:
        out = x
    dt = _dense_common(x, weight, bias, conv_states, out, err_flag, "conv_states")
    batch = query_start_loc.shape[0] - 1
    d = _dev(x, weight, bias, conv_states, query_start_loc, cache_indices, has_initial_state,
             out, err_flag)
    _vector(query_start_loc, torch.int32, "query_start_loc", batch + 1)
    if cache_indices is not None:
        _vector(cache_indices, torch.int32, "cache_indices", batch)
    if has_initial_state is not None:
        if has_initial_state.dtype not in (torch.bool, torch.uint8):
            raise TypeError("has_initial_state must be bool or uint8")
        if has_initial_state.dim() != 1 or has_initial_state.shape[0] < batch or (
                batch > 0 and has_initial_state.stride(0) != 1):
            raise ValueError("has_initial_state must be a contiguous [batch] tensor")
    cs = conv_states
    s_strides = cs.stride() if cs is not None else (0, 0, 0)
    with torch.cuda.device(d):
        st = LIB.sconv_causal_conv1d_fwd(
            _ptr(x), x.stride(0), x.stride(1), x.shape[0], x.shape[1], _ptr(weight),
            weight.stride(0), weight.stride(1), weight.shape[1], _ptr(bias), _ptr(cs),
            s_strides[0], s_strides[1], s_strides[2], cs.shape[2] if cs is not None else 0,
            cs.shape[0] if cs is not None else 0, _ptr(query_start_loc), batch,
            _ptr(cache_indices), _ptr(has_initial_state),
            SCONV_ACT_SILU if silu_activation else SCONV_ACT_NONE, int(pad_slot_id), _ptr(out),
            dt, _ptr(err_flag), _stream(d, stream))
    _check("sconv_causal_conv1d_fwd", st)
    return out


def sconv_causal_conv1d_update(x, conv_state, weight, bias, silu_activation, cache_seqlens=None,
                               conv_state_indices=None, pad_slot_id=-1, *, out=None,
                               err_flag=None, stream=None):
    """One decode token per sequence over dense state lines
    (causal_conv1d_update, "Implementation:Sgl project Sglang Mamba Ops"),
    in place by default.  x [batch, dim]; conv_state [num_lines, dim,
    state_len]; cache_seqlens int32 [batch] makes the lines circular;
    conv_state_indices int32 [batch] or None.  Returns ``out`` (default x)."""
    if out is None:
        out = x
    dt = _dense_common(x, weight, bias, conv_state, out, err_flag, "conv_state")
    if conv_state is None:
        raise ValueError("conv_state is required")
    batch = x.shape[0]
    d = _dev(x, conv_state, weight, bias, cache_seqlens, conv_state_indices, out, err_flag)
    if cache_seqlens is not None:
        _vector(cache_seqlens, torch.int32, "cache_seqlens", batch)
    if conv_state_indices is not None:
        _vector(conv_state_indices, torch.int32, "conv_state_indices", batch)
    cs = conv_state
    with torch.cuda.device(d):
        st = LIB.sconv_causal_conv1d_update(
            _ptr(x), x.stride(0), x.stride(1), batch, x.shape[1], _ptr(weight),
            weight.stride(0), weight.stride(1), weight.shape[1], _ptr(bias), _ptr(cs),
            cs.stride(0), cs.stride(1), cs.stride(2), cs.shape[2], cs.shape[0],
            _ptr(cache_seqlens), _ptr(conv_state_indices),
            SCONV_ACT_SILU if silu_activation else SCONV_ACT_NONE, int(pad_slot_id), _ptr(out),
            dt, _ptr(err_flag), _stream(d, stream))
    _check("sconv_causal_conv1d_update", st)
    return out


# Names used on the pages, for callers coming from them.
fused_sconv = sconv_fused
scatter_intermediate_conv = sconv_extract_windows
scatter_intermediate_ssm = sconv_scatter_intermediate_ssm
causal_conv1d_fwd = sconv_causal_conv1d_fwd
causal_conv1d_update = sconv_causal_conv1d_update
