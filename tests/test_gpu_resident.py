"""The all-resident multi-layer decode (moe_decode_resident) on the GPU.

* On a pool that already holds every expert, its outputs equal those of the
  per-layer call (moe_decode_layer) bit for bit, layer by layer, and the oracle's
  within the output tolerance; the LRU state moves the same way (hits only).
* Captured into a CUDA graph and replayed, it gives the same bits again.
* An expert that is not resident sets MOE_STATUS_NOT_RESIDENT and leaves the
  pool's keys untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import gen, workloads as W

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def m():
    from expert_offload_fp4_b200 import build
    build.build()
    import expert_offload_fp4_b200 as mod
    return mod


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16(bits):
    return dev(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def resident_pool(m, w, L, T, experts):
    """A pool of L * E slots with every (layer, expert) loaded and resident."""
    pool = m.Pool(w.H, w.I, w.E, w.k, L, w.fmt, L * w.E, max_tokens=T, host_layers=1)
    for e in range(w.E):
        pool.load_expert(0, e, experts[e])
    rows = (w.E + w.k - 1) // w.k
    idx = (torch.arange(rows * w.k, dtype=torch.int32, device="cuda") % w.E).view(rows, w.k)
    slot_of = torch.empty_like(idx)
    cs = torch.cuda.Stream()
    for layer in range(L):
        res = m.slot_lookup(pool, layer, idx, slot_of)
        m.stream_misses(pool, layer, res, cs)
    cs.synchronize()
    return pool


class Buffers:
    def __init__(self, m, w, T, L):
        self.idx = torch.empty((T, w.k), dtype=torch.int32, device="cuda")
        self.w = torch.empty((T, w.k), dtype=torch.float32, device="cuda")
        self.slot_of = torch.empty((T, w.k), dtype=torch.int32, device="cuda")
        self.y_part = torch.empty((T, w.k, w.H), dtype=torch.float32, device="cuda")
        self.y = torch.empty((L, T, w.H), dtype=torch.bfloat16, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.ws = torch.zeros(m.route_workspace_bytes(T, w.E), dtype=torch.uint8, device="cuda")

    def run(self, m, pool, x, wr, bias, stream=None):
        m.decode_resident(pool, 0, x, wr, bias, 1, self.idx, self.w, self.slot_of, self.y_part, self.y,
                          self.status, stream=stream)


CASES = [("35b_t1", W.DECODE_35B, 1), ("35b_t8", W.DECODE_35B, 8), ("tiny_t4", W.TINY, 4)]


@pytest.mark.parametrize("name,w,T", CASES, ids=[c[0] for c in CASES])
def test_resident_equals_per_layer_and_oracle(m, name, w, T):
    """Two pools built the same way: one runs the layers through moe_decode_layer
    (router, lookup kernel, FFN), the other through moe_decode_resident (the
    lookup folded into the FFN).  Outputs and the whole LRU state must agree bit
    for bit; outputs are also checked against the oracle."""
    L = 3
    experts = gen.expert_weights_many(w, 0, range(w.E))
    pool_a = resident_pool(m, w, L, T, experts)
    pool_b = resident_pool(m, w, L, T, experts)
    xs = np.stack([gen.activations(w, l, 5, T) for l in range(L)])
    x = bf16(xs)
    wr_h = [gen.router_weight(w, l) for l in range(L)]
    b_h = [gen.router_bias(w, l) for l in range(L)]
    wr = [bf16(a) for a in wr_h]
    bias = [dev(b) for b in b_h]
    lo = m.DecodeLayer(pool_a, T)
    y_ref = []
    for layer in range(L):
        y_ref.append(lo(layer, x[layer], wr[layer], bias[layer]).clone())
        assert lo.lookup.n_miss == 0
    torch.cuda.synchronize()
    assert int(lo.status.item()) == 0
    b = Buffers(m, w, T, L)
    b.run(m, pool_b, x, wr, bias)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    # the last layer's choices, weights and slots
    assert np.array_equal(b.idx.cpu().numpy(), lo.idx.cpu().numpy())
    assert np.array_equal(b.w.cpu().numpy().view(np.uint32), lo.w.cpu().numpy().view(np.uint32))
    assert np.array_equal(b.slot_of.cpu().numpy(), lo.slot_of.cpu().numpy())
    for layer in range(L):
        got = b.y[layer].view(torch.int16).cpu().numpy()
        assert np.array_equal(got, y_ref[layer].view(torch.int16).cpu().numpy()), layer
        idx_r, w_r, _ = oracle.route(xs[layer], wr_h[layer], b_h[layer], w.k, 1)
        yf, _ = oracle.moe_decode(w.fmt, w.H, w.I, w.E, xs[layer], idx_r, w_r,
                                  {e: experts[e] for e in set(idx_r.ravel().tolist())})
        rms = float(np.sqrt(np.mean(yf.astype(np.float64) ** 2)))
        assert float(np.max(np.abs(b.y[layer].float().cpu().numpy() - yf))) <= TOL * rms, layer
    sa, sb = pool_a.read_state(), pool_b.read_state()
    for key in ("slot_key", "slot_clock", "key_slot"):
        assert np.array_equal(sa[key], sb[key]), key
    assert sa["clock"] == sb["clock"]
    pool_a.close()
    pool_b.close()


def test_resident_graph_replay_is_bit_identical(m):
    w, T, L = W.DECODE_35B, 1, 4
    experts = gen.expert_weights_many(w, 0, range(w.E))
    pool = resident_pool(m, w, L, T, experts)
    x = bf16(np.stack([gen.activations(w, l, 2, T) for l in range(L)]))
    wr = [bf16(gen.router_weight(w, 0))] * L
    bias = [dev(gen.router_bias(w, 0))] * L
    b = Buffers(m, w, T, L)
    b.run(m, pool, x, wr, bias)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    eager = b.y.view(torch.int16).cpu().numpy().copy()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b.run(m, pool, x, wr, bias, stream=s)     # warm on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        b.run(m, pool, x, wr, bias, stream=torch.cuda.current_stream())
    for _ in range(3):
        b.y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert int(b.status.item()) == 0
        assert np.array_equal(b.y.view(torch.int16).cpu().numpy(), eager)
    del g
    pool.close()


def test_not_resident_sets_status_and_keeps_keys(m):
    w, T, L = W.TINY, 4, 1
    experts = gen.expert_weights_many(w, 0, range(w.E))
    # a pool of E slots with only half the experts resident
    pool = m.Pool(w.H, w.I, w.E, w.k, L, w.fmt, w.E, max_tokens=T, host_layers=1)
    for e in range(w.E):
        pool.load_expert(0, e, experts[e])
    half = torch.arange(w.E // 2, dtype=torch.int32, device="cuda").view(-1, w.k)
    slot_of = torch.empty_like(half)
    res = m.slot_lookup(pool, 0, half, slot_of)
    cs = torch.cuda.Stream()
    m.stream_misses(pool, 0, res, cs)
    cs.synchronize()
    st0 = pool.read_state()
    b = Buffers(m, w, T, L)
    x = bf16(gen.activations(w, 0, 0, T)[None])
    # route towards the upper half of the experts (not resident)
    bias_h = np.zeros(w.E, np.float32)
    bias_h[w.E // 2:] = 1000.0
    b.run(m, pool, x, [bf16(gen.router_weight(w, 0))], [dev(bias_h)])
    torch.cuda.synchronize()
    st = int(b.status.item())
    assert st & m._lib.STATUS_NOT_RESIDENT
    assert st & m._lib.STATUS_BAD_SLOT
    st1 = pool.read_state()
    assert np.array_equal(st1["slot_key"], st0["slot_key"])
    assert np.array_equal(st1["key_slot"], st0["key_slot"])
    pool.close()
