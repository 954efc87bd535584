"""Test-side helpers: build paged inputs from dense per-request sequences,
and the textbook references the oracle is pinned against.

The dense route is independent of the oracle: a request's whole sequence
(cached history followed by this step's tokens) is written out densely, its
history is placed into the paged cache by plain 4-D indexing
cache[block_table[r, p // N], h, p % N, off_s + j] (the page's cache layout,
"vllm.models.inkling.nvidia.ops.sconv" module docstring), and the expected
output is a library depthwise conv1d over the dense sequence.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

import workloads


def bf16_round(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def as_storage(values: np.ndarray, dtype: str) -> torch.Tensor:
    """float64 values already representable in ``dtype`` -> a torch tensor."""
    t = torch.from_numpy(np.asarray(values, np.float32))
    return t.to(workloads.TORCH_DTYPE[dtype])


def dense_case(seqs, hist, *, dtype="f32", H=1, ws=1, off_s=0, D=None, W=4, N=4,
               weight=None, act=None, residual=False, seed=0, pad_rows=None,
               extra_blocks=2):
    """Paged inputs for requests whose full sequences are ``seqs[r]``
    ([L_r, C] float arrays, values representable in ``dtype``) with the first
    ``hist[r]`` rows already cached.  Returns (workload, tensors)."""
    C = H * ws
    D = off_s + ws if D is None else D
    new = [len(s) - h for s, h in zip(seqs, hist)]
    need = sum(-(-len(s) // N) for s in seqs)
    wl = workloads.build("dense", dtype=dtype, H=H, D=D, ws=ws, off_s=off_s, W=W, N=N,
                         hist=hist, new=new, act=act, residual=residual, seed=seed,
                         pad_rows=pad_rows, num_blocks=need + extra_blocks)
    t = wl.tensors("cpu")
    if weight is not None:
        t["weight"] = as_storage(np.asarray(weight, np.float64).reshape(C, W), dtype)
    x_rows = [np.asarray(s, np.float64)[h:] for s, h in zip(seqs, hist)]
    t["x"] = as_storage(np.concatenate(x_rows, 0).reshape(-1, C), dtype)
    cache = t["cache"].clone()
    for r, (s, h) in enumerate(zip(seqs, hist)):
        s = np.asarray(s, np.float64).reshape(-1, C)
        for p in range(h):
            b = int(wl.block_table[r, p // N])
            for hh in range(H):
                cache[b, hh, p % N, off_s: off_s + ws] = as_storage(
                    s[p, hh * ws:(hh + 1) * ws], dtype)
    t["cache"] = cache
    return wl, t


def textbook_conv(seq: np.ndarray, weight: np.ndarray, act, residual) -> np.ndarray:
    """Depthwise causal conv1d of a dense sequence [L, C] with weight [C, W]
    by torch's conv1d (cross-correlation, W-1 zeros of left padding), then the
    SiLU and residual epilogue by torch's own silu."""
    L, C = seq.shape
    W = weight.shape[1]
    inp = torch.from_numpy(np.ascontiguousarray(seq.T, np.float64))[None]
    w = torch.from_numpy(np.ascontiguousarray(weight, np.float64))[:, None, :]
    y = F.conv1d(inp, w, padding=W - 1, groups=C)[0, :, :L].T
    if act in ("silu", "swish"):
        y = F.silu(y)
    if residual:
        y = y + torch.from_numpy(np.asarray(seq, np.float64))
    return y.numpy()


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()
