"""chunked_gated_delta_12_b200: chunk-KDA forward for B200 (sm_100a).

The compute lives in libkda.so (CUDA, C ABI in include/kda.h); this package
only marshals torch tensors into that ABI.
"""
from ._lib import KdaError, bwd_workspace_bytes, device_status, kda_chunk_bwd, kda_chunk_fwd, lib, wait_selftest

__all__ = ["kda_chunk_fwd", "kda_chunk_bwd", "bwd_workspace_bytes", "device_status", "wait_selftest", "KdaError",
           "lib"]
