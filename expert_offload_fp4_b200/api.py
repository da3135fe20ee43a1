"""Thin Python binding of libmoe_fp4.so: argument marshalling only.

Device buffers are torch tensors (their data_ptr is passed); streams are
torch.cuda.Stream objects (their cuda_stream handle is passed).  Every step of
the MoE layer runs in the library's kernels.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import _lib as L

FMT = {"mxfp4": L.MOE_MXFP4, "nvfp4": L.MOE_NVFP4}


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _np(a, dt):
    a = np.ascontiguousarray(a, dtype=dt)
    return a, a.ctypes.data_as(C.c_void_p)


class Pool:
    """The library-owned expert store: pinned host blocks, HBM slots, LRU state."""

    def __init__(self, H, I, E, k, L_layers, fmt, n_slots, max_tokens=8, host_layers=0):
        self.lib = L.load()
        self.cfg = L.MoeConfig(H, I, E, k, L_layers, FMT[fmt], n_slots, max_tokens, host_layers)
        self.H, self.I, self.E, self.k, self.L = H, I, E, k, L_layers
        self.fmt, self.n_slots, self.max_tokens = fmt, n_slots, max_tokens
        self.n_active = n_slots
        self.host_layers = host_layers or L_layers
        h = C.c_void_p()
        L.check("moe_pool_create", self.lib.moe_pool_create(C.byref(self.cfg), C.byref(h)))
        self.handle = h
        self.block_bytes = self.lib.moe_expert_block_bytes(C.byref(self.cfg))

    def close(self):
        if getattr(self, "handle", None):
            self.lib.moe_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def load_expert(self, layer, expert, tensors):
        """tensors: {"gate"|"up"|"down": (codes uint8, scales uint8, tensor_scale)}"""
        src = L.ExpertSrc()
        keep = []
        for i, name in enumerate(("gate", "up", "down")):
            c, s, ts = tensors[name]
            c, cp = _np(c, np.uint8)
            s, sp = _np(s, np.uint8)
            keep += [c, s]
            src.codes_h[i] = cp.value
            src.scales_h[i] = sp.value
            src.tensor_scale[i] = float(ts)
        L.check("moe_pool_load_expert",
                self.lib.moe_pool_load_expert(self.handle, int(layer), int(expert), C.byref(src)))

    def reset(self, n_active_slots=None):
        """Empty the pool and use only the first n_active_slots slots from now on."""
        n = self.n_slots if n_active_slots is None else int(n_active_slots)
        L.check("moe_pool_reset", self.lib.moe_pool_reset(self.handle, n))
        self.n_active = n

    def resize(self, n_active_slots):
        """Resize the slot pool at run time, keeping the LRU state (moe_pool_resize)."""
        L.check("moe_pool_resize", self.lib.moe_pool_resize(self.handle, int(n_active_slots)))
        self.n_active = int(n_active_slots)

    def set_copy_mode(self, mode):
        """"sm" (a kernel reads the mapped host block over PCIe) or "dma" (copy engine)."""
        m = {"sm": L.MOE_COPY_SM, "dma": L.MOE_COPY_DMA}[mode]
        L.check("moe_pool_set_copy_mode", self.lib.moe_pool_set_copy_mode(self.handle, m))

    def read_state(self):
        sk = np.empty(self.n_slots, np.int32)
        sc = np.empty(self.n_slots, np.uint64)
        ks = np.empty(self.L * self.E, np.int32)
        g = np.zeros(1, np.uint64)
        L.check("moe_pool_read_state", self.lib.moe_pool_read_state(
            self.handle, sk.ctypes.data_as(C.c_void_p), sc.ctypes.data_as(C.c_void_p),
            ks.ctypes.data_as(C.c_void_p), g.ctypes.data_as(C.c_void_p)))
        return dict(slot_key=sk, slot_clock=sc, key_slot=ks, clock=int(g[0]))

    def stats(self):
        st = L.Stats()
        L.check("moe_pool_stats", self.lib.moe_pool_stats(self.handle, C.byref(st)))
        return {f: getattr(st, f) for f, _ in L.Stats._fields_}

    def slot_ptr(self, slot):
        p, n = C.c_void_p(), C.c_size_t()
        L.check("moe_pool_slot_ptr", self.lib.moe_pool_slot_ptr(self.handle, int(slot), C.byref(p), C.byref(n)))
        return p.value, n.value


def route_workspace_bytes(T, E):
    return L.load().moe_route_workspace_bytes(int(T), int(E))


def route(x, wr, bias, k, renormalize, idx, w, workspace, stream=None):
    T, H = x.shape
    E = wr.shape[0]
    L.check("moe_route", L.load().moe_route(
        _p(x), _p(wr), _p(bias), T, H, E, int(k), int(renormalize), _p(idx), _p(w),
        _p(workspace), workspace.numel() * workspace.element_size(), _s(stream)))


def route_noalloc(x, wr, bias, k, renormalize, idx, w, stream=None):
    """moe_route_noalloc: the router with its scratch in a static device array of
    the library (for callers that cannot allocate device memory)."""
    T, H = x.shape
    E = wr.shape[0]
    L.check("moe_route_noalloc", L.load().moe_route_noalloc(
        _p(x), _p(wr), _p(bias), T, H, E, int(k), int(renormalize), _p(idx), _p(w), _s(stream)))


class Lookup:
    """Host-side result of one slot lookup (arrays sized for the call)."""

    def __init__(self, cap):
        self.uniq = np.zeros(cap, np.int32)
        self.is_hit = np.zeros(cap, np.int32)
        self.misses = (L.Miss * cap)()
        self.res = L.LookupResult(0, 0, self.uniq.ctypes.data_as(C.POINTER(C.c_int32)),
                                  self.is_hit.ctypes.data_as(C.POINTER(C.c_int32)), self.misses)

    @property
    def n_uniq(self):
        return self.res.n_uniq

    @property
    def n_miss(self):
        return self.res.n_miss

    def miss_list(self):
        return [(m.expert, m.slot, m.ticket, m.evicted_key) for m in self.misses[:self.res.n_miss]]


def slot_lookup(pool, layer, idx, slot_of, result=None, stream=None):
    T, k = idx.shape
    if result is None:
        result = Lookup(min(T * k, pool.E))
    L.check("moe_slot_lookup", pool.lib.moe_slot_lookup(
        pool.handle, int(layer), _p(idx), T, k, _p(slot_of), C.byref(result.res), _s(stream)))
    return result


def slot_lookup_launch(pool, layer, idx, slot_of, stream=None):
    T, k = idx.shape
    L.check("moe_slot_lookup_launch", pool.lib.moe_slot_lookup_launch(
        pool.handle, int(layer), _p(idx), T, k, _p(slot_of), _s(stream)))


def slot_lookup_result(pool, result):
    L.check("moe_slot_lookup_result", pool.lib.moe_slot_lookup_result(pool.handle, C.byref(result.res)))
    return result


def stream_misses(pool, layer, lookup, copy_stream):
    L.check("moe_stream_misses", pool.lib.moe_stream_misses(
        pool.handle, int(layer), lookup.misses, lookup.res.n_miss, _s(copy_stream)))


def expert_ffn(pool, layer, x, idx, w, slot_of, y_part, status, y=None, stream=None):
    """moe_expert_ffn: y_part [T, k, H] fp32; with y [T, H] bf16 also the fused combine."""
    T = x.shape[0]
    L.check("moe_expert_ffn", pool.lib.moe_expert_ffn(
        pool.handle, int(layer), _p(x), T, _p(idx), _p(w), _p(slot_of), _p(y_part), _p(y), _p(status),
        _s(stream)))


def ffn_launch_info(pool, T):
    """moe_ffn_launch_info: the decode FFN's launch shape for T tokens on this pool."""
    c, st, sb, sm = C.c_int(), C.c_int(), C.c_int(), C.c_int()
    L.check("moe_ffn_launch_info", pool.lib.moe_ffn_launch_info(
        pool.handle, int(T), C.byref(c), C.byref(st), C.byref(sb), C.byref(sm)))
    return dict(ctas=c.value, stages=st.value, stage_bytes=sb.value, smem_bytes=sm.value)


def decode_layer(pool, layer, x, wr, bias, renormalize, idx, w, slot_of, y_part, y, status, ws,
                 lookup=None, copy_events=None, overlap=True, stream=None, copy_stream=None):
    """moe_decode_layer: route, lookup, FFN, miss copies and combine of one layer."""
    T = x.shape[0]
    if copy_stream is None:
        raise ValueError("decode_layer needs a copy_stream of its own (torch.cuda.Stream())")
    cs = copy_stream
    ev0, ev1 = (None, None) if copy_events is None else (C.c_void_p(copy_events[0].cuda_event),
                                                        C.c_void_p(copy_events[1].cuda_event))
    L.check("moe_decode_layer", pool.lib.moe_decode_layer(
        pool.handle, int(layer), _p(x), T, _p(wr), _p(bias), int(renormalize), _p(idx), _p(w),
        _p(slot_of), _p(y_part), _p(y), _p(status), _p(ws), ws.numel(),
        C.byref(lookup.res) if lookup is not None else None, ev0, ev1, 1 if overlap else 0,
        _s(stream), _s(cs)))


def decode_resident(pool, layer0, x, wr, bias, renormalize, idx, w, slot_of, y_part, y, status, stream=None):
    """moe_decode_resident: one FFN launch per layer with the router, the resident
    lookup and the combine fused in, for x.shape[0] consecutive layers from
    layer0, with no host wait (capturable in a CUDA graph).  x, y: [n_layers, T, H]
    bf16; wr: list of n_layers [E, H] bf16; bias: list of n_layers [E] fp32
    (entries may be None) or None."""
    n, T = x.shape[0], x.shape[1]
    if len(wr) != n or (bias is not None and len(bias) != n):
        raise ValueError("decode_resident: one router weight (and bias) per layer")
    wr_arr = (C.c_void_p * n)(*[t.data_ptr() for t in wr])
    b_arr = None if bias is None else (C.c_void_p * n)(*[None if b is None else b.data_ptr() for b in bias])
    L.check("moe_decode_resident", pool.lib.moe_decode_resident(
        pool.handle, int(layer0), n, _p(x), T, wr_arr, b_arr, int(renormalize), _p(idx), _p(w), _p(slot_of),
        _p(y_part), _p(y), _p(status), _s(stream)))


def combine(y_part, y, stream=None):
    T, k, H = y_part.shape
    L.check("moe_combine", L.load().moe_combine(_p(y_part), T, k, H, _p(y), _s(stream)))


def lru_plan_resize(slot_key, slot_clock, n_new):
    """moe_lru_plan_resize on host arrays: (evicted slots, [(from, to) moves])."""
    sk = np.ascontiguousarray(slot_key, np.int32)
    sc = np.ascontiguousarray(slot_clock, np.uint64)
    n_old = len(sk)
    ev, mf, mt = (np.zeros(n_old, np.int32) for _ in range(3))
    ne, nm = C.c_int(), C.c_int()
    L.check("moe_lru_plan_resize", L.load().moe_lru_plan_resize(
        sk.ctypes.data_as(C.c_void_p), sc.ctypes.data_as(C.c_void_p), n_old, int(n_new),
        ev.ctypes.data_as(C.c_void_p), C.byref(ne), mf.ctypes.data_as(C.c_void_p),
        mt.ctypes.data_as(C.c_void_p), C.byref(nm)))
    return ev[:ne.value].tolist(), list(zip(mf[:nm.value].tolist(), mt[:nm.value].tolist()))


class BandwidthEstimate:
    """Moving estimates of PCIe and host-memory bandwidth (GB/s) and the q* split
    recomputed from them (moe_bw_init / moe_bw_observe / moe_bw_qstar)."""

    def __init__(self, alpha=0.25, b_pcie=0.0, b_host=0.0):
        self.est = L.BwEstimate()
        L.check("moe_bw_init", L.load().moe_bw_init(C.byref(self.est), float(alpha), float(b_pcie),
                                                     float(b_host)))

    def observe(self, link, nbytes, seconds):
        """link: "pcie" or "host"."""
        which = {"pcie": L.MOE_BW_PCIE, "host": L.MOE_BW_HOST}[link]
        L.check("moe_bw_observe", L.load().moe_bw_observe(C.byref(self.est), which, float(nbytes),
                                                           float(seconds)))

    @property
    def b_pcie(self):
        return self.est.b_pcie

    @property
    def b_host(self):
        return self.est.b_host

    def qstar(self, m):
        qg, qc, r = C.c_int(), C.c_int(), C.c_double()
        L.check("moe_bw_qstar", L.load().moe_bw_qstar(C.byref(self.est), int(m), C.byref(qg), C.byref(qc),
                                                       C.byref(r)))
        return qg.value, qc.value, r.value


def qstar_split(m, b_pcie, b_host):
    qg, qc, r = C.c_int(), C.c_int(), C.c_double()
    L.check("qstar_split", L.load().qstar_split(int(m), float(b_pcie), float(b_host),
                                                C.byref(qg), C.byref(qc), C.byref(r)))
    return qg.value, qc.value, r.value


def dequant_slot(pool, slot, key, which, out, stream=None):
    L.check("moe_dequant_slot", pool.lib.moe_dequant_slot(
        pool.handle, int(slot), int(key), int(which), _p(out), _s(stream)))


def nvfp4_gemm(a_codes, a_scales, b_codes, b_scales, D, status, stream=None):
    """D [M, N] fp32 = dq(A) dq(B)^T for NVFP4 A [M, K] and B [N, K] (codes uint8
    [rows, K/2], E4M3 scales uint8 [rows, K/16]), on the tcgen05 tensor cores."""
    M, N, K = a_codes.shape[0], b_codes.shape[0], a_codes.shape[1] * 2
    L.check("moe_nvfp4_gemm", L.load().moe_nvfp4_gemm(
        _p(a_codes), _p(a_scales), _p(b_codes), _p(b_scales), M, N, K, _p(D), _p(status), _s(stream)))


def nvfp4_quantize(x, codes, scales, sx, stream=None):
    """Per-token NVFP4 quantisation of x [T, H] bf16 (the prefill A operand)."""
    T, H = x.shape
    L.check("moe_nvfp4_quantize", L.load().moe_nvfp4_quantize(
        _p(x), T, H, _p(codes), _p(scales), _p(sx), _s(stream)))


def prefill_workspace_bytes(pool, T):
    return pool.lib.moe_prefill_workspace_bytes(pool.handle, int(T))


def prefill_ffn(pool, layer, x, idx, w, slot_of, y, workspace, status, stream=None):
    """y: y_part [T, k, H] fp32, every row written: the routed experts' FFN outputs
    times their routing weights, one row per (token, rank); sum and round them in
    rank order with combine(y, y_bf16)."""
    T = x.shape[0]
    L.check("moe_prefill_ffn", pool.lib.moe_prefill_ffn(
        pool.handle, int(layer), _p(x), T, _p(idx), _p(w), _p(slot_of), _p(y), _p(workspace),
        workspace.numel() * workspace.element_size(), _p(status), _s(stream)))


def set_wait_limits(ready_ms, dep_ms, pipe_ms):
    L.check("moe_set_wait_limits", L.load().moe_set_wait_limits(float(ready_ms), float(dep_ms),
                                                                 float(pipe_ms)))
