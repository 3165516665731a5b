"""B200 (sm_100a) gated delta rule: chunked WY/UT prefill and recurrent decode step.

The compute lives in ``libgdn.so`` (C ABI, ``include/gdn.h``); ``gdn`` is its ctypes binding.
Importing this package does not load the library; the first call does, and raises if it is absent.
"""
from .gdn import (CHUNK, GDN_BF16, GDN_F32, GDN_QK_L2NORM, GdnError, gdn_chunk_prefill, gdn_chunk_prefill_cuts,  # noqa: F401
                  gdn_decode_step, gdn_decode_verify, gdn_decode_verify_tree, gdn_get_device_status, lib,
                  status_string,
                  workspace_bytes)

__all__ = ["gdn_chunk_prefill", "gdn_chunk_prefill_cuts", "gdn_decode_step", "gdn_decode_verify",
           "gdn_decode_verify_tree",
           "gdn_get_device_status", "workspace_bytes", "lib", "status_string", "GdnError", "CHUNK", "GDN_F32",
           "GDN_BF16", "GDN_QK_L2NORM"]
