"""B200 (sm_100a) hot path of one FreeToken-style MoE layer with FP4 experts
offloaded to pinned host memory: router, LRU expert-slot pool in HBM, copy-engine
miss streaming, FP4 SwiGLU expert FFN, router-weighted combine, and the q*
bandwidth split.  The work is in libmoe_fp4.so (include/moe_fp4.h); this package
is its Python binding."""
from . import _lib  # noqa: F401
from .api import (BandwidthEstimate, Lookup, Pool, combine, decode_layer, decode_resident,  # noqa: F401
                  dequant_slot, expert_ffn, ffn_launch_info, nvfp4_gemm,
                  nvfp4_quantize, prefill_ffn, prefill_workspace_bytes, qstar_split,
                  route, route_noalloc, route_workspace_bytes, set_wait_limits, slot_lookup,
                  slot_lookup_launch, slot_lookup_result, stream_misses)
from .layer import DecodeLayer  # noqa: F401
