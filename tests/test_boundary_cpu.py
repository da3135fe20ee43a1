"""The C-ABI library on a machine without a GPU: it loads, exports every entry
point that include/moe_fp4.h declares, and its host-only calls and argument
checks behave (nothing here launches a kernel)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from conftest import ROOT, read_golden
from synthetic import workloads as W

HEADER = os.path.join(ROOT, "include", "moe_fp4.h")


@pytest.fixture(scope="module")
def lib():
    from expert_offload_fp4_b200 import build, _lib
    build.build()
    return _lib


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "moe_route" in names and "qstar_split" in names and len(names) >= 17
    L = lib.load()
    for n in names:
        assert hasattr(L, n), n
        assert n in lib.SIGNATURES, f"{n} has no binding signature"


def declared_arities():
    """{name: number of parameters} of every function the header declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(([^;]*?)\)\s*;", src,
                         flags=re.M | re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(lib):
    """Every ctypes signature has as many arguments as the header's declaration."""
    ar = declared_arities()
    assert set(ar) == set(declared_functions())
    for name, n in ar.items():
        assert len(lib.SIGNATURES[name][1]) == n, (name, n, len(lib.SIGNATURES[name][1]))


def test_qstar_split_through_the_abi_matches_table(lib):
    import expert_offload_fp4_b200 as m
    for _, bp, bh, pct in read_golden("qstar_table.txt"):
        qg, qc, r = m.qstar_split(256, float(bp), float(bh))
        assert f"{100 * r:.1f}" == pct and qg + qc == 256
    assert m.qstar_split(6, 49.0, 53.8)[:2] == (5, 1)
    assert m.qstar_split(7, 60, 50)[:2] == (7, 0)
    with pytest.raises(lib.MoeError) as e:
        m.qstar_split(3, 0.0, 1.0)
    assert e.value.code == lib.MOE_EINVAL


def _cfg(lib, w, n_slots=8, max_tokens=4, host_layers=0):
    return lib.MoeConfig(w.H, w.I, w.E, w.k, w.L, 0 if w.fmt == "mxfp4" else 1, n_slots,
                         max_tokens, host_layers)


@pytest.mark.parametrize("w", [W.TINY, W.DECODE_35B, W.DECODE_284B])
def test_block_layout_matches_workload(lib, w):
    cfg = _cfg(lib, w)
    assert lib.load().moe_expert_block_bytes(C.byref(cfg)) == W.expert_block_bytes(w)


def test_config_validation(lib):
    L = lib.load()
    bad = [dict(H=200), dict(I=0), dict(E=2000), dict(k=0), dict(k=33), dict(max_tokens=17),
           dict(n_slots=0), dict(fmt=5)]
    for b in bad:
        d = dict(H=256, I=256, E=16, k=2, L=1, fmt=0, n_slots=8, max_tokens=4, host_layers=0)
        d.update(b)
        cfg = lib.MoeConfig(d["H"], d["I"], d["E"], d["k"], d["L"], d["fmt"], d["n_slots"],
                            d["max_tokens"], d["host_layers"])
        assert L.moe_expert_block_bytes(C.byref(cfg)) == 0, b
        h = C.c_void_p()
        assert L.moe_pool_create(C.byref(cfg), C.byref(h)) == lib.MOE_EINVAL, b
        assert h.value is None


def test_route_argument_checks_need_no_gpu(lib):
    L = lib.load()
    ws = L.moe_route_workspace_bytes(4, 16)
    assert ws >= 4 * 16 * 4 and L.moe_route_workspace_bytes(0, 16) == 0
    buf = (C.c_uint8 * 64)()
    p = C.cast(buf, C.c_void_p)
    # H not a multiple of 256, T = 0, k > E, workspace too small
    assert L.moe_route(p, p, None, 4, 200, 16, 2, 1, p, p, p, ws, None) == lib.MOE_EINVAL
    assert L.moe_route(p, p, None, 0, 256, 16, 2, 1, p, p, p, ws, None) == lib.MOE_EINVAL
    assert L.moe_route(p, p, None, 4, 256, 16, 17, 1, p, p, p, ws, None) == lib.MOE_EINVAL
    assert L.moe_route(p, p, None, 4, 256, 16, 2, 1, p, p, p, 8, None) == lib.MOE_EINVAL
    assert b"workspace" in L.moe_last_error()
    odd = C.c_void_p(p.value | 1)   # x and W_r are read 16 bytes at a time
    assert L.moe_route(odd, p, None, 4, 256, 16, 2, 1, p, p, p, ws, None) == lib.MOE_EINVAL
    assert b"aligned" in L.moe_last_error()
    assert L.moe_combine(p, 4, 2, 254, p, None) == lib.MOE_EINVAL
    # the per-layer call and the copy-mode setter need a pool
    assert L.moe_decode_layer(None, 0, p, 1, p, None, 1, p, p, p, p, p, p, p, 64, None, None, None, 1,
                              None, None) == lib.MOE_EINVAL
    assert L.moe_pool_set_copy_mode(None, lib.MOE_COPY_DMA) == lib.MOE_EINVAL
    # with overlap, a copy stream equal to the compute stream would deadlock: refused
    fake_pool = C.c_void_p(p.value)
    s1 = C.c_void_p(0x1000)
    assert L.moe_decode_layer(fake_pool, 0, p, 1, p, None, 1, p, p, p, p, p, p, p, 64, None, None, None, 1,
                              s1, s1) == lib.MOE_EINVAL
    assert b"copy_stream" in L.moe_last_error()
    assert L.moe_set_wait_limits(-1.0, 1.0, 1.0) == lib.MOE_EINVAL
