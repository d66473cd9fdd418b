"""B200 (sm_100a) lightning attention: causal linear attention with the
right-product kernel trick, tiled into blocks (MiniMax-01, "Scaling Foundation
Models with Lightning Attention").

The computation lives in ``liblightning.so`` (C ABI in
``include/lightning_attention.h``); ``api`` is its thin binding.  Importing
this package does not load the library; the first call does, and fails loudly
if it is missing.
"""
from .api import (LA_BF16, LA_FP32, LA_OUT_RMSNORM, LA_WRITE_STATE, LightningError,
                  LightningLibraryError, decode_step, device_status, lib, prefill, state_out,
                  status_string, version)

__all__ = ["prefill", "decode_step", "state_out", "device_status", "lib", "status_string",
           "version", "LightningError", "LightningLibraryError", "LA_BF16", "LA_FP32",
           "LA_OUT_RMSNORM", "LA_WRITE_STATE"]
