"""ctypes declarations of libmoe_fp4.so (see include/moe_fp4.h).

Loading fails loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_fp4.so")

MOE_OK, MOE_EINVAL, MOE_ENOMEM, MOE_ECUDA, MOE_ETIMEOUT, MOE_EBOUNDS, MOE_ESTATE = range(7)
ERR_NAMES = {1: "MOE_EINVAL", 2: "MOE_ENOMEM", 3: "MOE_ECUDA", 4: "MOE_ETIMEOUT",
             5: "MOE_EBOUNDS", 6: "MOE_ESTATE"}
MOE_MXFP4, MOE_NVFP4 = 0, 1
MOE_COPY_SM, MOE_COPY_DMA = 0, 1
MOE_BW_PCIE, MOE_BW_HOST = 0, 1
STATUS_READY_TIMEOUT, STATUS_DEP_TIMEOUT, STATUS_BAD_SLOT, STATUS_BAD_EXPERT, STATUS_PIPE_TIMEOUT = 1, 2, 4, 8, 16
STATUS_NOT_RESIDENT = 32


class MoeConfig(C.Structure):
    _fields_ = [("H", C.c_int), ("I", C.c_int), ("E", C.c_int), ("k", C.c_int), ("L", C.c_int),
                ("fmt", C.c_int), ("n_slots", C.c_int), ("max_tokens", C.c_int),
                ("host_layers", C.c_int), ("reserved", C.c_int * 3)]


class ExpertSrc(C.Structure):
    _fields_ = [("codes_h", C.c_void_p * 3), ("scales_h", C.c_void_p * 3),
                ("tensor_scale", C.c_float * 3)]


class Miss(C.Structure):
    _fields_ = [("expert", C.c_int32), ("slot", C.c_int32), ("ticket", C.c_uint32),
                ("evicted_key", C.c_int32)]


class LookupResult(C.Structure):
    _fields_ = [("n_uniq", C.c_int), ("n_miss", C.c_int), ("uniq_h", C.POINTER(C.c_int32)),
                ("is_hit_h", C.POINTER(C.c_int32)), ("miss_h", C.POINTER(Miss))]


class BwEstimate(C.Structure):
    _fields_ = [("alpha", C.c_double), ("b_pcie", C.c_double), ("b_host", C.c_double),
                ("n_pcie", C.c_longlong), ("n_host", C.c_longlong)]


class Stats(C.Structure):
    _fields_ = [("lookups", C.c_longlong), ("unique", C.c_longlong), ("hits", C.c_longlong),
                ("misses", C.c_longlong), ("evictions", C.c_longlong),
                ("h2d_bytes", C.c_longlong), ("h2d_copies", C.c_longlong)]


class MoeError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn}: {ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


# name -> (restype, argtypes); every entry point of include/moe_fp4.h
vp, i32, f64, sz = C.c_void_p, C.c_int, C.c_double, C.c_size_t
SIGNATURES = {
    "moe_last_error": (C.c_char_p, []),
    "moe_pool_create": (i32, [C.POINTER(MoeConfig), C.POINTER(vp)]),
    "moe_pool_destroy": (i32, [vp]),
    "moe_expert_block_bytes": (sz, [C.POINTER(MoeConfig)]),
    "moe_pool_load_expert": (i32, [vp, i32, i32, C.POINTER(ExpertSrc)]),
    "moe_pool_read_state": (i32, [vp, vp, vp, vp, vp]),
    "moe_pool_reset": (i32, [vp, i32]),
    "moe_pool_stats": (i32, [vp, C.POINTER(Stats)]),
    "moe_pool_slot_ptr": (i32, [vp, i32, C.POINTER(vp), C.POINTER(sz)]),
    "moe_route_workspace_bytes": (sz, [i32, i32]),
    "moe_route": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp]),
    "moe_slot_lookup": (i32, [vp, i32, vp, i32, i32, vp, C.POINTER(LookupResult), vp]),
    "moe_slot_lookup_launch": (i32, [vp, i32, vp, i32, i32, vp, vp]),
    "moe_slot_lookup_result": (i32, [vp, C.POINTER(LookupResult)]),
    "moe_stream_misses": (i32, [vp, i32, C.POINTER(Miss), i32, vp]),
    "moe_pool_set_copy_mode": (i32, [vp, i32]),
    "moe_pool_resize": (i32, [vp, i32]),
    "moe_lru_plan_resize": (i32, [vp, vp, i32, i32, vp, C.POINTER(i32), vp, vp, C.POINTER(i32)]),
    "moe_set_ffn_trace": (i32, [vp]),
    "moe_ffn_launch_info": (i32, [vp, i32, vp, vp, vp, vp]),
    "moe_expert_ffn": (i32, [vp, i32, vp, i32, vp, vp, vp, vp, vp, vp, vp]),
    "moe_combine": (i32, [vp, i32, i32, i32, vp, vp]),
    "moe_decode_layer": (i32, [vp, i32, vp, i32, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, C.c_size_t,
                               C.POINTER(LookupResult), vp, vp, i32, vp, vp]),
    "moe_decode_resident": (i32, [vp, i32, i32, vp, i32, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]),
    "qstar_split": (i32, [i32, f64, f64, C.POINTER(i32), C.POINTER(i32), C.POINTER(f64)]),
    "moe_bw_init": (i32, [C.POINTER(BwEstimate), f64, f64, f64]),
    "moe_bw_observe": (i32, [C.POINTER(BwEstimate), i32, f64, f64]),
    "moe_bw_qstar": (i32, [C.POINTER(BwEstimate), i32, C.POINTER(i32), C.POINTER(i32), C.POINTER(f64)]),
    "moe_dequant_slot": (i32, [vp, i32, i32, i32, vp, vp]),
    "moe_set_wait_limits": (i32, [f64, f64, f64]),
    "moe_nvfp4_gemm": (i32, [vp, vp, vp, vp, i32, i32, i32, vp, vp, vp]),
    "moe_nvfp4_quantize": (i32, [vp, i32, i32, vp, vp, vp, vp]),
    "moe_prefill_workspace_bytes": (sz, [vp, i32]),
    "moe_prefill_ffn": (i32, [vp, i32, vp, i32, vp, vp, vp, vp, vp, sz, vp, vp]),
    "moe_route_noalloc": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]),
}

_lib = None


def load():
    """Load libmoe_fp4.so (raises if it was never built: no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m expert_offload_fp4_b200.build` (nvcc, sm_100a)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(fn_name, rc):
    if rc != MOE_OK:
        msg = load().moe_last_error()
        raise MoeError(fn_name, rc, msg.decode() if msg else "")
    return rc
