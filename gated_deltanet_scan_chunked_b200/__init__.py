"""Gated DeltaNet chunked scan for NVIDIA B200 (sm_100a).

The computation lives in libgdn.so (CUDA kernels behind the C ABI in
include/gdn.h).  ``gdn`` is a thin ctypes binding; ``inputs`` holds the
seeded synthetic workloads; ``build`` compiles the library.
"""
from .gdn import (GdnError, bwd_workspace_size, conv_workspace_size,  # noqa: F401
                  gdn_check_device_error, gdn_chunk_bwd, gdn_chunk_fwd, gdn_chunk_fwd_conv,
                  gdn_conv_frontend, gdn_decode_conv, gdn_decode_multi, gdn_decode_step,
                  gdn_gr_read, gdn_gr_write, load, workspace_size)

__all__ = ["gdn_chunk_fwd", "gdn_chunk_bwd", "gdn_decode_step", "gdn_decode_multi",
           "gdn_check_device_error", "gdn_conv_frontend", "gdn_chunk_fwd_conv", "gdn_decode_conv", "gdn_gr_read",
           "gdn_gr_write", "GdnError", "load",
           "workspace_size", "bwd_workspace_size", "conv_workspace_size"]
