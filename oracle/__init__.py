"""ctypes front of the C oracle (oracle.c).

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg import this package.  It never touches the CUDA library.
Functions here only marshal numpy arrays into the C calls; all arithmetic is in
oracle.c, except in prefill_batch.py, which runs the prefill path's per-token
dot products of oracle.c as float64 matrix products (a library matmul as one
step) so that a whole 2048-token prompt can be checked in seconds.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                               "-fPIC", "-shared", "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


class Expert(C.Structure):
    _fields_ = [("codes", C.c_void_p * 3), ("scales", C.c_void_p * 3), ("tscale", C.c_float * 3)]


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        vp, i32, f32, f64 = C.c_void_p, C.c_int, C.c_float, C.c_double
        sig = {
            "or_e2m1_value": (f64, [i32]), "or_e8m0_value": (f64, [i32]),
            "or_e4m3_value": (f64, [i32]), "or_e2m1_quantize": (i32, [f32]),
            "or_e4m3_quantize": (i32, [f32]), "or_f32_to_bf16": (C.c_uint16, [f32]),
            "or_dequant": (None, [i32, vp, vp, f32, i32, i32, vp]),
            "or_nvfp4_quantize_row": (None, [vp, i32, f32, vp, vp]),
            "or_token_scale": (f32, [vp, i32]),
            "or_prefill_quantize_x": (f32, [vp, i32, vp, vp]),
            "or_router_logits": (None, [vp, vp, vp, i32, i32, i32, vp]),
            "or_topk": (None, [vp, i32, i32, i32, vp]),
            "or_route_weights": (None, [vp, vp, i32, i32, i32, i32, vp]),
            "or_route": (None, [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]),
            "or_lru_create": (vp, [i32, i32]), "or_lru_destroy": (None, [vp]),
            "or_lru_state": (None, [vp, vp, vp, vp, vp]),
            "or_lru_step": (i32, [vp, i32, i32, vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]),
            "or_lru_resize": (i32, [vp, i32]),
            "or_expert_ffn": (None, [i32, i32, i32, vp, vp, vp]),
            "or_moe_decode": (None, [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
            "or_moe_dense": (None, [i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
            "or_moe_prefill_token": (None, [i32, i32, i32, vp, vp, vp, vp, vp, vp]),
            "or_prefill_h_rows": (None, [vp, vp, i32, i32, vp, vp]),
            "or_qstar_split": (i32, [i32, f64, f64, vp, vp, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


FMT = {"mxfp4": 0, "nvfp4": 1}


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ------------------------------------------------------------------------- codecs

def e2m1_value(c): return lib().or_e2m1_value(int(c))
def e8m0_value(b): return lib().or_e8m0_value(int(b))
def e4m3_value(b): return lib().or_e4m3_value(int(b))
def e2m1_quantize(v): return lib().or_e2m1_quantize(float(v))
def e4m3_quantize(v): return lib().or_e4m3_quantize(float(v))
def f32_to_bf16(v): return lib().or_f32_to_bf16(float(v))


def dequant(fmt, codes, scales, tscale):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, K), np.float32)
    lib().or_dequant(FMT[fmt], _p(codes), _p(scales), float(tscale), rows, K, _p(out))
    return out


def nvfp4_quantize_row(v, S):
    v = _c(v, np.float32)
    K = v.shape[0]
    codes = np.empty(K // 2, np.uint8)
    scales = np.empty(K // 16, np.uint8)
    lib().or_nvfp4_quantize_row(_p(v), K, float(S), _p(codes), _p(scales))
    return codes, scales


def prefill_quantize_x(x_bf16):
    x = _c(x_bf16, np.uint16)
    H = x.shape[0]
    codes = np.empty(H // 2, np.uint8)
    scales = np.empty(H // 16, np.uint8)
    S = lib().or_prefill_quantize_x(_p(x), H, _p(codes), _p(scales))
    return codes, scales, S


def token_scale(v):
    v = _c(v, np.float32)
    return lib().or_token_scale(_p(v), v.shape[0])


# -------------------------------------------------------------------------- router

def router_logits(x, wr, bias):
    x, wr = _c(x, np.uint16), _c(wr, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), np.float32)
    lib().or_router_logits(_p(x), _p(wr), None if b is None else _p(b), T, H, E, _p(out))
    return out


def topk(logits, k):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    lib().or_topk(_p(logits), T, E, k, _p(idx))
    return idx


def route(x, wr, bias, k, renormalize=1):
    x, wr = _c(x, np.uint16), _c(wr, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    logits = np.empty((T, E), np.float32)
    lib().or_route(_p(x), _p(wr), None if b is None else _p(b), T, H, E, k, int(renormalize),
                   _p(idx), _p(w), _p(logits))
    return idx, w, logits


# ----------------------------------------------------------------------------- LRU

class LRU:
    """The oracle's global LRU slot pool over L*E (layer, expert) keys."""

    def __init__(self, n_slots, L, E):
        self.n_slots, self.L, self.E = n_slots, L, E
        self._h = lib().or_lru_create(n_slots, L * E)

    def __del__(self):
        if getattr(self, "_h", None):
            lib().or_lru_destroy(self._h)
            self._h = None

    def step(self, layer, idx):
        idx = _c(idx, np.int32)
        T, k = idx.shape
        n = T * k
        slot_of = np.empty((T, k), np.int32)
        uniq, hit = np.empty(n, np.int32), np.empty(n, np.int32)
        me, ms, ev = np.empty(n, np.int32), np.empty(n, np.int32), np.empty(n, np.int32)
        nu, nm = C.c_int(0), C.c_int(0)
        rc = lib().or_lru_step(self._h, layer, self.E, _p(idx), T, k, _p(slot_of), _p(uniq),
                               _p(hit), C.byref(nu), _p(me), _p(ms), _p(ev), C.byref(nm))
        if rc != 0:
            raise ValueError("slot pool smaller than the unique experts of one step")
        u, m = nu.value, nm.value
        return dict(slot_of=slot_of, uniq=uniq[:u].copy(), hit=hit[:u].astype(bool),
                    miss_expert=me[:m].copy(), miss_slot=ms[:m].copy(), evicted=ev[:m].copy())

    def resize(self, n_new):
        """Resize to n_new slots; returns the number of evicted entries."""
        rc = lib().or_lru_resize(self._h, int(n_new))
        if rc < 0:
            raise ValueError("n_new must be >= 1")
        self.n_slots = int(n_new)
        return rc

    def state(self):
        sk = np.empty(self.n_slots, np.int32)
        sc = np.empty(self.n_slots, np.uint64)
        ks = np.empty(self.L * self.E, np.int32)
        g = C.c_uint64(0)
        lib().or_lru_state(self._h, _p(sk), _p(sc), _p(ks), C.byref(g))
        return dict(slot_key=sk, slot_clock=sc, key_slot=ks, clock=g.value)


# ------------------------------------------------------------------------------ FFN

def make_expert(tensors, keep):
    """tensors: {"gate": (codes, scales, ts), "up": ..., "down": ...} -> Expert struct.
    Arrays are appended to `keep` so they outlive the call."""
    ex = Expert()
    for i, name in enumerate(("gate", "up", "down")):
        c, s, ts = tensors[name]
        c, s = _c(c, np.uint8), _c(s, np.uint8)
        keep += [c, s]
        ex.codes[i] = c.ctypes.data
        ex.scales[i] = s.ctypes.data
        ex.tscale[i] = float(ts)
    return ex


def _expert_array(experts: dict, E, keep):
    arr = (Expert * E)()
    for e, t in experts.items():
        arr[e] = make_expert(t, keep)
    return arr


def expert_ffn(fmt, H, I, tensors, x_f32):
    keep = []
    ex = make_expert(tensors, keep)
    x = _c(x_f32, np.float32)
    y = np.empty(H, np.float64)
    lib().or_expert_ffn(FMT[fmt], H, I, C.byref(ex), _p(x), _p(y))
    return y


def moe_decode(fmt, H, I, E, x, idx, w, experts: dict):
    """experts: {e: tensors} for at least every chosen e.  Returns (y_f32, y_bf16)."""
    keep = []
    arr = _expert_array(experts, E, keep)
    x, idx, w = _c(x, np.uint16), _c(idx, np.int32), _c(w, np.float32)
    T, k = idx.shape
    yf = np.empty((T, H), np.float32)
    yb = np.empty((T, H), np.uint16)
    lib().or_moe_decode(FMT[fmt], H, I, T, k, _p(x), _p(idx), _p(w), arr, _p(yf), _p(yb))
    return yf, yb


def moe_dense(fmt, H, I, E, k, renormalize, x, wr, bias, experts: dict):
    keep = []
    arr = _expert_array(experts, E, keep)
    x, wr = _c(x, np.uint16), _c(wr, np.uint16)
    b = None if bias is None else _c(bias, np.float32)
    T = x.shape[0]
    y = np.empty((T, H), np.float64)
    mask = np.empty((T, E), np.int32)
    lib().or_moe_dense(FMT[fmt], H, I, E, T, k, int(renormalize), _p(x), _p(wr),
                       None if b is None else _p(b), arr, _p(y), _p(mask))
    return y, mask.astype(bool)


def moe_prefill_token(H, I, E, x_t, idx_t, w_t, experts: dict):
    keep = []
    arr = _expert_array(experts, E, keep)
    x_t, idx_t, w_t = _c(x_t, np.uint16), _c(idx_t, np.int32), _c(w_t, np.float32)
    yf = np.empty(H, np.float32)
    yb = np.empty(H, np.uint16)
    lib().or_moe_prefill_token(H, I, idx_t.shape[0], _p(x_t), _p(idx_t), _p(w_t), arr,
                               _p(yf), _p(yb))
    return yf, yb


def prefill_h_rows(g, u):
    """h = fp32(silu(g) * u) of [rows, I] double dot products, quantised to NVFP4
    with tensor scale 1: (codes [rows, I/2], scales [rows, I/16])."""
    g, u = _c(g, np.float64), _c(u, np.float64)
    rows, I = g.shape
    codes = np.empty((rows, I // 2), np.uint8)
    scales = np.empty((rows, I // 16), np.uint8)
    lib().or_prefill_h_rows(_p(g), _p(u), rows, I, _p(codes), _p(scales))
    return codes, scales


# ------------------------------------------------------------------------------- q*

def qstar_split(m, b_pcie, b_host):
    qg, qc, r = C.c_int(0), C.c_int(0), C.c_double(0)
    rc = lib().or_qstar_split(int(m), float(b_pcie), float(b_host), C.byref(qg), C.byref(qc),
                              C.byref(r))
    if rc != 0:
        raise ValueError("bad q* arguments")
    return qg.value, qc.value, r.value
