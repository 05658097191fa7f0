"""B200-native (sm_100a) Gated Delta Rule chunked forward.

The compute path is the C-ABI library ``libgdn.so`` (CUDA kernels for
sm_100a, include/gdn.h); this package only marshals arguments to it.
Importing the package does not load the library; the first call does, and
raises if the library has not been built.
"""
from ._binding import (CHUNK, HEAD_DIM, SHORT_MAX, Stages, check_values, chunk_fwd, chunk_fwd_host,
                       chunk_fwd_noalloc, decode_status, host_buffer_bytes, host_plan, lib, noalloc_status,
                       pipeline_ranges, read_status, recurrent_fwd, recurrent_window_fwd, set_value_checks, short_fwd,
                       status_string, workspace_bytes, workspace_layout)

__all__ = ["chunk_fwd", "chunk_fwd_host", "chunk_fwd_noalloc", "recurrent_fwd", "recurrent_window_fwd", "short_fwd",
           "pipeline_ranges", "Stages", "workspace_bytes", "workspace_layout", "lib", "status_string", "read_status",
           "noalloc_status", "decode_status", "check_values", "set_value_checks", "host_buffer_bytes", "host_plan",
           "HEAD_DIM", "CHUNK", "SHORT_MAX"]
