"""Seeded synthetic inputs for the MoE-layer tests, smoke check and benchmark.

Everything is drawn from a counter-based generator so that any tensor of any
(layer, step) can be regenerated alone:

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): output i of a stream with key K is
  mix64(K + (i + 1) * GAMMA).  Stream keys chain mix64 over
  (seed, tensor id, a, b).
* Normals: Box-Muller in float64 on two consecutive outputs, then rounded
  (round-to-nearest-even) to float32 and, for activations and router weights,
  to bfloat16.

This module holds input preparation only.  The FP4 expert weights it returns
are synthetic *inputs* of the MoE layer: for the "normal" recipe a N(0, sigma)
float32 tensor is quantised offline to NVFP4 here (per-tensor FP32 scale
amax/(6*448), per-16 E4M3 scale, E2M1 codes, round-to-nearest-even with
saturation), the way a checkpoint would be prepared before serving.  The layer
itself (routing, caching, dequantisation, FFN, combine) lives elsewhere.

Canonical tensor layout returned here (shared by the oracle and the library
loader): codes uint8 [rows, K/2] with element c of a row in byte c//2, the lower
element index in the low nibble; scales uint8 [rows, K/bs] (E8M0 for MXFP4,
E4M3 for NVFP4); one float32 tensor scale (1.0 for MXFP4).
"""
from __future__ import annotations

import math

import numpy as np

from .workloads import MXFP4, NVFP4, Workload, block_elems

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor ids of the generator streams
T_X, T_WR, T_PERM, T_GATE, T_UP, T_DOWN, T_GATE_S, T_UP_S, T_DOWN_S = range(1, 10)


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser; works in place on z (a fresh uint64 array)."""
    t = np.empty_like(z)
    for sh, mul in ((30, _M1), (27, _M2)):
        np.right_shift(z, np.uint64(sh), out=t)
        np.bitwise_xor(z, t, out=z)
        np.multiply(z, mul, out=z)
    np.right_shift(z, np.uint64(31), out=t)
    np.bitwise_xor(z, t, out=z)
    return z


def stream_key(seed: int, tensor: int, a: int = 0, b: int = 0) -> np.uint64:
    with np.errstate(over="ignore"):
        k = _mix64(np.array([seed], np.uint64) + GAMMA)
        for v in (tensor, a, b):
            k = _mix64(k ^ np.array([v], np.uint64))
    return k[0]


def uint64s(key: np.uint64, n: int, start: int = 0) -> np.ndarray:
    """Outputs start .. start+n-1 of the SplitMix64 stream with this key."""
    with np.errstate(over="ignore"):
        z = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        np.multiply(z, GAMMA, out=z)
        np.add(z, key, out=z)
        return _mix64(z)


def normals(key: np.uint64, n: int, start: int = 0) -> np.ndarray:
    """n standard normals (float64); normal j uses stream outputs 2j and 2j+1."""
    u = uint64s(key, 2 * n, 2 * start)
    scale = 2.0 ** -53
    u1 = ((u[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * scale
    u2 = ((u[1::2] >> np.uint64(11)).astype(np.float64) + 1.0) * scale
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------- inputs

def router_weight(w: Workload, layer: int) -> np.ndarray:
    """W_r [E, H] bf16 bits, N(0, 0.02)."""
    lk = 0 if w.shared_layer else layer
    z = normals(stream_key(w.seed, T_WR, lk), w.E * w.H) * 0.02
    return f32_to_bf16_bits(z.astype(np.float32)).reshape(w.E, w.H)


def router_bias(w: Workload, layer: int, zipf_s: float | None = None) -> np.ndarray:
    """Zipf skew as a logit bias: b_e = -s * ln(rank_e), rank from a seeded permutation."""
    s = w.zipf_s if zipf_s is None else zipf_s
    lk = 0 if w.shared_layer else layer
    order = np.argsort(uint64s(stream_key(w.seed, T_PERM, lk), w.E), kind="stable")
    rank = np.empty(w.E, np.int64)
    rank[order] = np.arange(1, w.E + 1)
    return (-s * np.log(rank.astype(np.float64))).astype(np.float32)


def activations(w: Workload, layer: int, step: int, T: int) -> np.ndarray:
    """x [T, H] bf16 bits, N(0, 1), fresh for every (layer, step)."""
    z = normals(stream_key(w.seed, T_X, layer, step), T * w.H)
    return f32_to_bf16_bits(z.astype(np.float32)).reshape(T, w.H)


# ------------------------------------------------------------- FP4 weight synthesis

def _e4m3_table() -> np.ndarray:
    v = np.zeros(127, np.float64)
    for c in range(127):
        e, m = c >> 3, c & 7
        v[c] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return v


E4M3_POS = _e4m3_table()                       # codes 0..126, ascending
E2M1_POS = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _nearest_even(v: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest table entry to v >= 0, ties to the even index, saturating."""
    n = len(table)
    i = np.clip(np.searchsorted(table, v, side="left"), 1, n - 1)
    lo, hi = table[i - 1], table[i]
    dlo, dhi = v - lo, hi - v
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (i % 2 == 0))
    idx = np.where(pick_hi, i, i - 1)
    return np.where(v >= table[-1], n - 1, idx).astype(np.uint8)


def _pack_nibbles(codes: np.ndarray) -> np.ndarray:
    c = codes.reshape(codes.shape[0], -1, 2)
    return (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8)


def _normal_nvfp4(key: np.uint64, rows: int, K: int, sigma: float):
    w = (normals(key, rows * K) * sigma).astype(np.float32).reshape(rows, K)
    amax = np.float32(np.abs(w).max())
    S = np.float32(amax / np.float32(2688.0))
    blocks = w.reshape(rows, K // 16, 16)
    bmax = np.abs(blocks).max(axis=2)
    ratio = (bmax / (np.float32(6.0) * S)).astype(np.float32)
    sc = _nearest_even(ratio.astype(np.float64), E4M3_POS)
    q = (E4M3_POS[sc].astype(np.float32) * S).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(q[..., None] > 0, blocks / q[..., None], np.float32(0)).astype(np.float32)
    mag = _nearest_even(np.abs(r).astype(np.float64), E2M1_POS)
    codes = mag | (np.signbit(r).astype(np.uint8) << 3)
    return _pack_nibbles(codes.reshape(rows, K)), sc.reshape(rows, K // 16), float(S)


def _uniform_mxfp4(key_c: np.uint64, key_s: np.uint64, rows: int, K: int, exp_range):
    nbytes = rows * K // 2
    codes = uint64s(key_c, (nbytes + 7) // 8).view(np.uint8)[:nbytes].reshape(rows, K // 2)
    lo, hi = exp_range
    ns = rows * K // 32
    e = (uint64s(key_s, ns) % np.uint64(hi - lo + 1)).astype(np.int64) + lo + 127
    return codes.copy(), e.astype(np.uint8).reshape(rows, K // 32), 1.0


def expert_weights(w: Workload, layer: int, expert: int) -> dict:
    """Canonical FP4 tensors of one expert: gate [I,H], up [I,H], down [H,I].

    Returns {"gate": (codes, scales, tensor_scale), "up": ..., "down": ...}.
    """
    lk = 0 if w.shared_layer else layer
    out = {}
    for name, tid, tid_s, rows, K in (("gate", T_GATE, T_GATE_S, w.I, w.H),
                                      ("up", T_UP, T_UP_S, w.I, w.H),
                                      ("down", T_DOWN, T_DOWN_S, w.H, w.I)):
        kc = stream_key(w.seed, tid, lk, expert)
        if w.weight_recipe == "normal":
            assert w.fmt == NVFP4
            out[name] = _normal_nvfp4(kc, rows, K, w.sigma)
        else:
            assert w.fmt == MXFP4
            ks = stream_key(w.seed, tid_s, lk, expert)
            out[name] = _uniform_mxfp4(kc, ks, rows, K, w.exp_range)
    assert all(s.shape[1] == (K // block_elems(w.fmt)) for (_, s, _), K in
               zip(out.values(), (w.H, w.H, w.I)))
    return out


def _expert_job(args):
    w, layer, expert = args
    return expert, expert_weights(w, layer, expert)


def expert_weights_many(w: Workload, layer: int, experts, workers: int | None = None) -> dict:
    """expert_weights for many experts, fanned out over a spawn-started process pool
    (safe to call after CUDA is initialised in the parent)."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    experts = list(experts)
    if workers is None:
        workers = min(len(experts), os.cpu_count() or 1, 32)
    if workers <= 1 or len(experts) <= 2:
        return {e: expert_weights(w, layer, e) for e in experts}
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        return dict(ex.map(_expert_job, [(w, layer, e) for e in experts], chunksize=1))
