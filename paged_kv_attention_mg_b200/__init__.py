"""B200-native paged KV attention (the mini-sglang attention hot path).

``store_kv``, ``decode_attn`` and ``extend_attn`` call the CUDA library
``libmg.so`` (C ABI in ``include/mg.h``) through ``paged_kv_attention_mg_b200.mg``.
``workload`` draws seeded synthetic inputs; ``roofline`` holds the sizing and
algorithmic byte / FLOP formulas.
"""
from .mg import (MgError, decode_attn, decode_plan, decode_workspace_bytes, extend_attn, load,
                 read_device_error, store_decode_attn, store_kv)

__all__ = ["MgError", "decode_attn", "decode_plan", "decode_workspace_bytes", "extend_attn", "load",
           "read_device_error", "store_decode_attn", "store_kv"]
