"""The prefill expert FFN of the oracle for a whole prompt at once.

TEST INFRASTRUCTURE (see the package docstring).  Same steps as
or_moe_prefill_token in oracle.c (post.smzdm.com/p/aomxznrn, "FreeToken干的事":
prefill is compute-bound and scheduled apart from decode; the activation and h
quantisation are the readings stated in oracle.c's header), but the per-token
dot products of all tokens routed to one expert are taken together as float64
matrix products (numpy matmul: a library primitive standing in for the
sums).  Every other step calls oracle.c: the per-token NVFP4 quantisation of x
and its dequantisation, the exact fp32 dequantisation of the weights, the
silu(g)*u rounding and NVFP4 quantisation of h.  The routing-weighted sum runs
over the ranks in order, in double, and is rounded to fp32 once.

Only the order of the float64 additions inside a dot product differs from the
per-token C function, so the two agree to float64 rounding.
"""
from __future__ import annotations

import numpy as np

from . import dequant, prefill_h_rows, prefill_quantize_x


def moe_prefill(H, I, E, x, idx, w, experts):
    """x [T, H] bf16 bits, idx/w [T, k] (routing), experts {e: tensors} for every
    routed e.  Returns y [T, H] float32 (before the output's bf16 rounding)."""
    x = np.ascontiguousarray(x, np.uint16)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    T, k = idx.shape
    # quantised-then-dequantised activations, token by token (C)
    xq = np.empty((T, H), np.float64)
    for t in range(T):
        c, s, S = prefill_quantize_x(x[t])
        xq[t] = dequant("nvfp4", c[None, :], s[None, :], S)[0]
    # per-(token, rank) expert outputs, grouped by expert
    ye = np.zeros((T, k, H), np.float64)
    for e in sorted(set(idx.ravel().tolist())):
        tok, rank = np.nonzero(idx == e)
        t = experts[e]
        wg = dequant("nvfp4", *t["gate"]).astype(np.float64)      # [I, H]
        wu = dequant("nvfp4", *t["up"]).astype(np.float64)
        wd = dequant("nvfp4", *t["down"]).astype(np.float64)      # [H, I]
        X = xq[tok]
        g = X @ wg.T
        u = X @ wu.T
        hc, hs = prefill_h_rows(g, u)
        hq = dequant("nvfp4", hc, hs, 1.0).astype(np.float64)     # [M_e, I]
        ye[tok, rank] = hq @ wd.T
    acc = np.zeros((T, H), np.float64)
    for j in range(k):
        acc += w[:, j:j + 1].astype(np.float64) * ye[:, j]
    return acc.astype(np.float32)
