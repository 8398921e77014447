"""B200 (sm_100a) WKV6 recurrence: chunked prefill and decode step behind a C ABI.

The compute lives in ``libgoldwkv.so`` (see ``include/goldwkv.h``); ``binding`` marshals
torch tensors into it.  Importing this package does not load the library; the first call
does, and raises if it was not built.
"""
from .binding import (WkvError, backward_workspace_bytes, decode_workspace_bytes, gold_compress,
                      gold_decompress, load,
                      new_workspace, prefill_workspace_bytes, wkv6_backward, wkv6_decode_step,
                      wkv6_decode_step_gn, wkv6_prefill, wkv6_prefill_gn, wkv6_prefill_static,
                      prefill_static_status,
                      wkv6c2_backward, wkv6c2_decode_step, wkv6c2_prefill, workspace_status)

__all__ = ["WkvError", "backward_workspace_bytes", "decode_workspace_bytes", "gold_compress",
           "gold_decompress", "load",
           "new_workspace", "prefill_workspace_bytes", "wkv6_backward", "wkv6_decode_step",
           "wkv6_decode_step_gn", "wkv6_prefill", "wkv6_prefill_gn", "wkv6_prefill_static",
           "prefill_static_status",
           "wkv6c2_backward", "wkv6c2_decode_step", "wkv6c2_prefill", "workspace_status"]
