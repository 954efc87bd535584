"""GPU parity of sconv_seq_metadata and sconv_seq_metadata_ahead against
the CPU oracle (bit-exact) ("vllm.models.inkling.nvidia.ops.sconv",
sconv_seq_metadata)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests._gpu import hs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(qsl_np, R, n_actual, n_padded, cap=None):
    cap = cap or n_padded
    qsl = torch.from_numpy(qsl_np).to(DEV)
    rsi, rqs = oracle.seq_metadata(qsl_np, R, n_actual, n_padded)
    for name in ("sconv_seq_metadata", "sconv_seq_metadata_ahead"):
        si = torch.full((cap,), -7, dtype=torch.int32, device=DEV)
        qs = torch.full((cap,), -7, dtype=torch.int32, device=DEV)
        getattr(hs(), name)(qsl, R, n_actual, si, qs, n_padded)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(si.cpu().numpy()[:n_padded], rsi, err_msg=name)
        np.testing.assert_array_equal(qs.cpu().numpy()[:n_padded], rqs, err_msg=name)
        assert bool((si[n_padded:] == -7).all() and (qs[n_padded:] == -7).all()), name


def _qsl(rng, R, max_len, empty_frac=0.2):
    lens = rng.integers(1, max_len + 1, size=R)
    lens[rng.random(R) < empty_frac] = 0
    if lens.sum() == 0:
        lens[0] = 1
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


@pytest.mark.parametrize("seed,R,max_len", [
    (0, 1, 1000), (1, 7, 50), (2, 256, 1), (3, 16, 2048), (4, 128, 4),
    (5, 4096, 3), (6, 4097, 3), (7, 20000, 2)])  # the last two search global memory
def test_against_oracle(seed, R, max_len):
    rng = np.random.default_rng(seed)
    qsl = _qsl(rng, R, max_len)
    T = int(qsl[-1])
    _run(qsl, R, T, T + int(rng.integers(0, 300)), cap=T + 400)


def test_no_padding_argument():
    qsl = np.array([0, 2, 2, 5], np.int32)
    _run(qsl, 3, 5, 5)


def test_only_padded_rows():
    _run(np.zeros(2, np.int32), 1, 0, 33)
