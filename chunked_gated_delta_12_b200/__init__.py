"""chunked_gated_delta_12_b200: chunk-KDA forward (and its recurrent and backward companions) for B200.

The compute lives in libkda.so (CUDA, C ABI in include/kda.h); this package
only marshals torch tensors into that ABI.
"""
from ._lib import (NOALLOC_SCRATCH_BYTES, RECURRENT_MAX_LEN, KdaError, bwd_workspace_bytes, device_status,
                   host_workspace_bytes, kda_chunk_bwd, kda_chunk_bwd_noalloc, kda_chunk_fwd, kda_chunk_fwd_host,
                   kda_chunk_fwd_long, kda_recurrent_fwd, lib,
                   long_segments, long_workspace_bytes, resolve_mode, split_workspace_bytes, use_split,
                   wait_selftest)

__all__ = ["kda_chunk_fwd", "kda_chunk_fwd_host", "host_workspace_bytes", "use_split", "split_workspace_bytes", "kda_chunk_fwd_long", "long_segments", "long_workspace_bytes", "kda_recurrent_fwd", "resolve_mode", "RECURRENT_MAX_LEN", "kda_chunk_bwd",
           "kda_chunk_bwd_noalloc", "NOALLOC_SCRATCH_BYTES", "bwd_workspace_bytes", "device_status", "wait_selftest", "KdaError", "lib"]
