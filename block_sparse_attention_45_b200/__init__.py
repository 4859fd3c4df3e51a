"""B200-native dynamic block-sparse attention for video diffusion transformers.

The compute path is libbsa.so (hand-written sm_100a CUDA behind the C ABI in
include/bsa.h); this package is its ctypes binding plus the seeded synthetic
workload generator.  Importing it does not load the library; the first call
does, and raises if the library was not built.
"""
from .binding import (BSA_OK, BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED, BSA_ERR_LAUNCH,
                      BSA_ERR_DRIVER, TEXT_KEEP, FRAME0_DENSE, DEVERR_BAD_INDEX,
                      DEVERR_BAD_COUNT, DEVERR_TIMEOUT, BsaError, BsaLayout, attention_fwd,
                      attention_workspace_bytes,
                      block_scores, build_mask, dense_fwd, make_layout, sparse_attention,
                      status_string, workspace_bytes)

__all__ = ["BSA_OK", "BSA_ERR_INVALID_ARG", "BSA_ERR_UNSUPPORTED", "BSA_ERR_LAUNCH",
           "BSA_ERR_DRIVER", "TEXT_KEEP", "FRAME0_DENSE", "DEVERR_BAD_INDEX", "DEVERR_BAD_COUNT",
           "DEVERR_TIMEOUT", "BsaError", "BsaLayout", "attention_fwd", "attention_workspace_bytes",
           "block_scores",
           "build_mask", "dense_fwd", "make_layout", "sparse_attention", "status_string",
           "workspace_bytes"]
