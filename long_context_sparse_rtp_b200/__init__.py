"""RTPurbo sparse-attention layer for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``librtp.so`` (``include/rtp.h``); this package
holds its CUDA sources (``csrc/``), the build step (``build.py``), a thin ctypes
binding with the same entry-point names (``rtp.py``), a layer-level convenience
wrapper (``layer.py``) and the seeded synthetic-input generator (``synth.py``).
Importing the package does not load the library; the first call does, and fails
loudly if it is not built.
"""
from .rtp import (  # noqa: F401
    RtpError,
    local_ring_alloc,
    rtp_check_device,
    rtp_dense_attn,
    rtp_get_device_status,
    rtp_index_scores,
    rtp_local_attn,
    rtp_local_attn_decode_ring,
    rtp_local_ring_write,
    rtp_sparse_attn_decode,
    rtp_sparse_attn_decode_select,
    rtp_sparse_attn_prefill,
    rtp_status_string,
    rtp_topp_select,
    rtp_version,
    rtp_workspace_size,
)
from .layer import DecodeGraph, rtp_layer_decode, rtp_layer_prefill  # noqa: F401
