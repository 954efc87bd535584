"""B200-native (sm_100a) fused short-convolution step of hybrid/SSM inference.

One launch per call: paged sliding-window cache insert, depthwise causal
conv1d over the window ending at each token's absolute position, optional
SiLU and residual ("vllm.models.inkling.nvidia.ops.sconv"), plus the decode
update, several streams of a layer in one call, prefix-caching window
extraction ("core.ssm.ops.intermediate_extraction") and the per-token
metadata builder.

The kernels live in ``libsconv.so`` (C ABI: include/sconv.h), built by
``python -m hybrid_sconv_b200.build``.  The ops are loaded on first use;
using one without the library raises ImportError (there is no fallback).
"""

_EXPORTS = (
    "EFLAG_BLOCK", "EFLAG_LOGICAL", "EFLAG_POSITION", "EFLAG_QUERY_START", "EFLAG_REQUEST",
    "EFLAG_SLOT", "EFLAG_TIMEOUT", "LIB_PATH", "SconvError", "causal_conv1d_fwd",
    "causal_conv1d_update", "fused_sconv", "scatter_intermediate_conv",
    "scatter_intermediate_ssm", "sconv_causal_conv1d_fwd", "sconv_causal_conv1d_update",
    "sconv_extract_windows",
    "sconv_extract_windows_paged", "sconv_fused", "sconv_fused_streams",
    "sconv_scatter_intermediate_ssm", "sconv_seq_metadata", "sconv_seq_metadata_ahead",
    "sconv_update", "sconv_seq_metadata_taps", "sconv_seq_metadata_taps_ahead",
    "sconv_fused_taps", "sconv_fused_streams_taps", "sconv_fused_taps_next", "TAP_X",
    "TAP_ZERO",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import binding  # loads libsconv.so, or raises ImportError
        return getattr(binding, name)
    raise AttributeError(f"module 'hybrid_sconv_b200' has no attribute {name!r}")
