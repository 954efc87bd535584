"""The C ABI library loads, exports every entry point include/sconv.h
declares, and rejects malformed arguments on the host (CPU only: no call
here reaches a kernel launch)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sconv.h")


@pytest.fixture(scope="module")
def lib():
    from hybrid_sconv_b200 import build
    build.build()
    from hybrid_sconv_b200 import binding
    return binding.LIB


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sconv_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("sconv_fused", "sconv_update", "sconv_extract_windows", "sconv_seq_metadata"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.sconv_abi_version() == 1
    assert lib.sconv_status_string(0) == b"ok"


FAKE = 1 << 20  # a non-null address; validation fails before anything is dereferenced


def _strides(*s):
    return (ctypes.c_int64 * 4)(*s)


def _fused(lib, **over):
    a = dict(x=FAKE, x_rs=8, T=4, C=8, w=FAKE + 4096, w_sc=4, w_sk=1, W=4,
             cache=FAKE * 64, cs=_strides(512, 256, 16, 1), nb=8, H=2, N=16, D=16,
             pos=FAKE, sid=FAKE, slot=FAKE, qs=FAKE, bt=FAKE, bt_rs=4, R=2, MB=4,
             off_s=0, ws=4, act=0, res=1, dt=1, out=FAKE * 512, out_rs=8, err=0, stream=0)
    a.update(over)
    return lib.sconv_fused(a["x"], a["x_rs"], a["T"], a["C"], a["w"], a["w_sc"], a["w_sk"],
                           a["W"], a["cache"], a["cs"], a["nb"], a["H"], a["N"], a["D"],
                           a["pos"], a["sid"], a["slot"], a["qs"], a["bt"], a["bt_rs"],
                           a["R"], a["MB"], a["off_s"], a["ws"], a["act"], a["res"], a["dt"],
                           a["out"], a["out_rs"], a["err"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(T=0), 0),
    (dict(T=-1), 1),
    (dict(W=0), 1),
    (dict(W=9), 2),
    (dict(dt=7), 2),
    (dict(act=5), 1),
    (dict(C=6), 1),                      # C != H*ws
    (dict(off_s=14), 1),                 # off_s + ws > D
    (dict(cs=_strides(512, 256, 16, 2)), 1),  # D stride must be 1
    (dict(x_rs=4), 1),                   # row stride < C
    (dict(out_rs=4), 1),
    (dict(bt_rs=2), 1),                  # block_table row stride < max_blocks
    (dict(out=FAKE), 1),                 # out aliases x
    (dict(out=FAKE * 64 + 64), 1),       # out inside the cache
    (dict(x=0), 1),
    (dict(sid=0), 1),
    (dict(R=0), 1),
    (dict(nb=0), 1),
])
def test_fused_host_validation(lib, over, status):
    assert _fused(lib, **over) == status


def test_update_host_validation(lib):
    def call(B=4, W=4, dt=1, x=FAKE, out=FAKE * 512):
        return lib.sconv_update(x, 8, B, 8, FAKE + 4096, 4, 1, W, FAKE * 64,
                                _strides(512, 256, 16, 1), 8, 2, 16, 16, FAKE, FAKE, FAKE,
                                4, 4, 0, 4, 0, 1, dt, out, 8, 0, 0)
    assert call(B=0) == 0
    assert call(B=-2) == 1
    assert call(W=12) == 2
    assert call(dt=3) == 2
    assert call(out=FAKE) == 1


def test_extract_host_validation(lib):
    def call(max_count=4, d_conv=4, sc=1, out=FAKE * 64, ss=16, dt=1, oss=64, rc=FAKE):
        return lib.sconv_extract_windows(FAKE, 100, 16, ss, sc, FAKE, rc, max_count, out,
                                         oss, d_conv, dt, 0)
    assert call(max_count=0) == 0
    assert call(max_count=-1) == 1
    assert call(d_conv=9) == 2
    assert call(d_conv=0) == 1
    assert call(sc=2) == 1
    assert call(ss=8) == 1            # row stride < conv_dim
    assert call(oss=32) == 1          # slot stride < conv_dim * d_conv
    assert call(out=FAKE + 64) == 1   # overlaps src
    assert call(dt=9) == 2
    assert call(rc=0) == 1


@pytest.mark.parametrize("name", ["sconv_seq_metadata", "sconv_seq_metadata_ahead"])
def test_seq_metadata_host_validation(lib, name):
    def call(R=3, na=7, npad=10, cap_s=10, cap_q=10):
        return getattr(lib, name)(FAKE, R, na, npad, FAKE * 2, cap_s, FAKE * 3, cap_q, 0)
    assert call(na=0, npad=0) == 0
    assert call(npad=5) == 1           # fewer padded than actual
    assert call(cap_s=9) == 1
    assert call(cap_q=9) == 1
    assert call(R=0) == 1
    assert call(na=-1) == 1


def test_python_binding_size_errors_match_the_page():
    """sconv_seq_metadata raises ValueError for the size errors the page
    names before touching a device."""
    import torch
    from hybrid_sconv_b200 import sconv_seq_metadata
    qsl = torch.zeros(4, dtype=torch.int32)
    small = torch.zeros(3, dtype=torch.int32)
    big = torch.zeros(10, dtype=torch.int32)
    with pytest.raises(ValueError, match="cover all actual"):
        sconv_seq_metadata(qsl, 3, 5, big, big, 4)
    with pytest.raises(ValueError, match="seq_idx_out is too small"):
        sconv_seq_metadata(qsl, 3, 5, small, big)
    with pytest.raises(ValueError, match="query_start_out is too small"):
        sconv_seq_metadata(qsl, 3, 5, big, small)


def test_product_path_does_not_import_the_oracle():
    """The package's sources never reference the CPU oracle."""
    pkg = os.path.join(ROOT, "hybrid_sconv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text, f


def test_streams_host_validation(lib):
    """sconv_fused_streams rejects overlapping lane ranges, too many streams
    and outputs that overlap another stream's buffers, before any launch."""
    from hybrid_sconv_b200.binding import StreamDesc

    def desc(x, out, off_s, ws=4, w=FAKE + 4096):
        return StreamDesc(x, 8, w, 4, 1, out, 8, off_s, ws, 0, 1)

    def call(descs, n=None, T=4):
        arr = (StreamDesc * len(descs))(*descs)
        return lib.sconv_fused_streams(arr, len(descs) if n is None else n, T, 4, FAKE * 64,
                                       _strides(512, 256, 16, 1), 8, 2, 16, 16, FAKE, FAKE,
                                       FAKE, FAKE, FAKE, 4, 2, 4, 1, 0, 0)
    ok_a = desc(FAKE, FAKE * 512, 0)
    ok_b = desc(FAKE * 2, FAKE * 1024, 8)
    assert call([ok_a, ok_b], T=0) == 0
    assert call([ok_a, desc(FAKE * 2, FAKE * 1024, 2)]) == 1          # lanes 0..3 and 2..5 overlap
    assert call([ok_a, desc(FAKE * 2, FAKE * 512 + 16, 8)]) == 1      # outputs overlap
    assert call([ok_a, desc(FAKE * 512, FAKE * 1024, 8)]) == 1        # output is another's x
    assert call([ok_a] * 5) == 2                                       # more than 4 streams
    assert call([ok_a], n=0) == 1


def test_gather_entry_points_host_validation(lib):
    """Malformed calls of the SSM state gather and the paged window
    extraction are rejected before any launch."""
    def ssm(max_count=4, flat=64, srs=64, ors=64, dt=0, out=FAKE * 64, nchunks=8, rc=FAKE):
        return lib.sconv_scatter_intermediate_ssm(FAKE, nchunks, flat, srs, FAKE * 2, rc,
                                                  max_count, out, ors, dt, 0, 0)
    assert ssm(max_count=0) == 0
    assert ssm(max_count=-1) == 1
    assert ssm(max_count=70000) == 2
    assert ssm(flat=0) == 1
    assert ssm(srs=32) == 1
    assert ssm(ors=32) == 1
    assert ssm(dt=4) == 2
    assert ssm(out=FAKE + 16) == 1       # overlaps the states
    assert ssm(rc=0) == 1

    def paged(max_count=4, d_conv=4, off_s=0, ws=4, D=16, cs=None, oss=32, out=FAKE * 512,
              bt_rs=4):
        cs = cs or _strides(512, 256, 16, 1)
        return lib.sconv_extract_windows_paged(FAKE * 64, cs, 8, 2, 16, D, off_s, ws, FAKE,
                                               bt_rs, 2, 4, FAKE, FAKE, FAKE, max_count, out,
                                               oss, d_conv, 1, 0, 0)
    assert paged(max_count=0) == 0
    assert paged(d_conv=9) == 2
    assert paged(d_conv=0) == 1
    assert paged(off_s=14) == 1          # off_s + ws > D
    assert paged(cs=_strides(512, 256, 16, 2)) == 1
    assert paged(oss=16) == 1            # slot stride < C * d_conv
    assert paged(out=FAKE * 64 + 32) == 1  # inside the cache
    assert paged(bt_rs=2) == 1


def test_dense_entry_points_host_validation(lib):
    """Malformed calls of sconv_causal_conv1d_fwd / _update are rejected
    before any launch (every call here either fails validation or has an
    empty batch)."""
    def fwd(batch=2, W=4, dt=1, act=1, L=3, x_st=16, x_sc=1, T=8, dim=16, out=FAKE,
            states=FAKE * 64, s_c=3, s_k=1, lines=4, qsl=FAKE * 3, w=FAKE * 2):
        return lib.sconv_causal_conv1d_fwd(
            FAKE, x_st, x_sc, T, dim, w, 4, 1, W, 0, states, 48, s_c, s_k, L, lines, qsl,
            batch, 0, 0, act, -1, out, dt, 0, 0)
    assert fwd(batch=0) == 0
    assert fwd(batch=0, x_st=1, x_sc=8) == 0       # channel-major x
    assert fwd(batch=0, states=0) == 0              # no state lines
    assert fwd(batch=-1) == 1
    assert fwd(W=1) == 1
    assert fwd(W=9) == 2
    assert fwd(dt=5) == 2
    assert fwd(act=3) == 1
    assert fwd(L=2) == 1                            # state_len < W-1
    assert fwd(L=17) == 2
    assert fwd(x_st=8) == 1                         # rows of x overlap
    assert fwd(out=FAKE + 2) == 1                   # out overlaps x without being x
    assert fwd(states=FAKE + 4) == 1                # lines overlap x
    assert fwd(s_c=2) == 1                          # line entries overlap
    assert fwd(lines=0) == 1
    assert fwd(qsl=0) == 1
    assert fwd(dim=0) == 1
    assert fwd(w=FAKE + 32) == 1                    # weight inside x (written in place)

    def upd(batch=2, W=4, L=3, st=FAKE * 64, dt=1):
        return lib.sconv_causal_conv1d_update(
            FAKE, 16, 1, batch, 16, FAKE * 2, 4, 1, W, 0, st, 48, 3, 1, L, 4, 0, 0, 1, -1,
            FAKE, dt, 0, 0)
    assert upd(batch=0) == 0
    assert upd(st=0) == 1
    assert upd(batch=-3) == 1
    assert upd(L=17) == 2
    assert upd(W=9) == 2
    assert upd(dt=9) == 2


@pytest.mark.parametrize("name", ["sconv_seq_metadata_taps", "sconv_seq_metadata_taps_ahead"])
def test_seq_metadata_taps_host_validation(lib, name):
    """Size, capacity and pointer errors of the tap resolution are rejected
    before any launch."""
    def call(qsl=FAKE, R=3, na=7, npad=10, pos=FAKE * 4, slot=FAKE * 5, bt=FAKE * 6, bt_rs=4,
             MB=4, nb=8, N=16, W=4, si=FAKE * 2, cap_s=10, qs=FAKE * 3, cap_q=10, taps=FAKE * 7,
             cap_t=30):
        return getattr(lib, name)(qsl, R, na, npad, pos, slot, bt, bt_rs, MB, nb, N, W, si,
                                  cap_s, qs, cap_q, taps, cap_t, 0)
    assert call(na=0, npad=0) == 0
    assert call(npad=5) == 1            # fewer padded than actual rows
    assert call(cap_s=9) == 1
    assert call(cap_q=9) == 1
    assert call(cap_t=29) == 1          # 10 rows x 3 lags do not fit
    assert call(W=0) == 1
    assert call(W=9) == 2
    assert call(R=0) == 1
    assert call(bt_rs=3) == 1
    assert call(N=0) == 1
    assert call(taps=0) == 1            # a table is needed for W > 1
    assert call(pos=0) == 1
    assert call(W=1, taps=0, cap_t=0, si=0, qs=0) == 0   # nothing to write


def test_fused_taps_host_validation(lib):
    """sconv_fused_taps needs a table for W > 1, rejects an output that
    overlaps it, and applies the stream checks of sconv_fused_streams."""
    from hybrid_sconv_b200.binding import StreamDesc

    def desc(x, out, off_s, ws=4):
        return StreamDesc(x, 8, FAKE + 4096, 4, 1, out, 8, off_s, ws, 0, 1)

    def call(descs, T=4, W=4, taps=FAKE * 2048, slot=FAKE, ready=1, cs=None, dt=1):
        arr = (StreamDesc * len(descs))(*descs)
        return lib.sconv_fused_taps(arr, len(descs), T, W, FAKE * 64,
                                    cs or _strides(512, 256, 16, 1), 8, 2, 16, 16, slot, taps,
                                    ready, dt, 0, 0)
    ok = desc(FAKE, FAKE * 512, 0)
    assert call([ok], T=0) == 0
    assert call([ok], taps=0) == 1                      # W > 1 without a table
    assert call([ok], slot=0) == 1
    assert call([ok], taps=FAKE * 512 + 8) == 1         # table inside the output
    assert call([ok, desc(FAKE * 2, FAKE * 1024, 2)]) == 1   # lane ranges overlap
    assert call([ok], W=9) == 2
    assert call([ok], cs=_strides(512, 256, 16, 2)) == 1    # D stride must be 1
    assert call([ok], dt=7) == 2


def test_fused_taps_next_host_validation(lib):
    """The combined step checks both its convolution arguments and the next
    step's resolution, and rejects a next table that overlaps this step's
    table or output, before any launch."""
    from hybrid_sconv_b200.binding import StreamDesc, TapsBuild

    def call(T=4, W=4, taps=FAKE * 2048, next_taps=FAKE * 4096, npad=8, nq=FAKE * 8,
             nnull=False):
        d = (StreamDesc * 1)(StreamDesc(FAKE, 8, FAKE + 4096, 4, 1, FAKE * 512, 8, 0, 4, 0, 1))
        b = TapsBuild(nq, 2, npad, npad, FAKE * 16, FAKE * 24, FAKE * 32, 4, 4, 0, 0, 0, 0,
                      next_taps, npad * (W - 1))
        return lib.sconv_fused_taps_next(d, 1, T, W, FAKE * 64, _strides(512, 256, 16, 1), 8,
                                         2, 16, 16, FAKE, taps, 1, 0,
                                         None if nnull else ctypes.byref(b), 0)
    assert call(nnull=True) == 1                      # next is required
    assert call(T=0, npad=0) == 0                     # nothing to do
    assert call(taps=0) == 1                          # this step's table is needed
    assert call(next_taps=FAKE * 2048 + 8) == 1       # next table overlaps this one
    assert call(next_taps=FAKE * 512 + 8) == 1        # next table inside the output
    assert call(W=9) == 2
