"""B200-native KDA (Kimi Delta Attention) forward pass, decode step and backward pass.

The compute path is the C-ABI library ``libkda.so`` built from ``csrc/``
(hand-written sm_100a CUDA kernels); ``kda.py`` is a thin ctypes binding with
the same entry-point names.  PyTorch is used only for device memory and
streams.  Importing this package does not load the CUDA library; the first
call does, and it raises if the library is missing.
"""
from .kda import (KdaError, kda_forward, kda_decode_step, kda_status_string,  # noqa: F401
                  kda_forward_workspace_bytes, kda_forward_kernel_name, kda_launch_count,
                  kda_device_status, kda_forward_noalloc, kda_selftest_timeout,
                  kda_noalloc_status, kda_noalloc_selftest_timeout, kda_forward_segments, kda_release_workspace, kda_segment_maps, kda_segment_scan,
                  kda_forward_indexed, kda_decode_step_indexed, kda_forward_fused,
                  kda_decode_step_fused, kda_backward, kda_backward_workspace_bytes,
                  library_path, load_library)

__all__ = ["KdaError", "kda_forward", "kda_decode_step", "kda_status_string",
           "kda_forward_workspace_bytes", "kda_forward_kernel_name", "kda_launch_count",
           "kda_device_status", "kda_forward_noalloc", "kda_selftest_timeout",
           "kda_noalloc_status", "kda_noalloc_selftest_timeout",
           "kda_forward_segments", "kda_release_workspace", "kda_segment_maps", "kda_segment_scan",
           "kda_forward_indexed", "kda_decode_step_indexed", "kda_forward_fused",
           "kda_decode_step_fused", "kda_backward", "kda_backward_workspace_bytes",
           "library_path", "load_library"]
