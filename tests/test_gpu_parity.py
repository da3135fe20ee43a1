"""GPU parity of every C-ABI call against the oracle, on the same seeded inputs.

Bit-exact: router logits and expert indices, LRU slot state and miss lists,
dequantised slot contents, the combine's bf16 rounding.  Tolerance (the decode
layer's output): max |y - y_ref| <= 2e-2 * rms(y_ref) per (step, layer) bf16
tensor, with y_ref the oracle's double-accumulated SwiGLU layer.
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


def host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def small(name, fmt, H=256, I=256, E=16, k=2, L=1, seed=11, zipf=0.0):
    return W.Workload(name=name, H=H, I=I, E=E, k=k, L=L, fmt=fmt, seed=seed, batches=(1,),
                      steps=4, zipf_s=zipf,
                      weight_recipe="normal" if fmt == W.NVFP4 else "uniform",
                      exp_range=(-6, -2))


_weights = {}


def prefetch(w, layer, experts):
    """Generate the experts' weights not yet cached, in parallel (spawned workers)."""
    lk = 0 if w.shared_layer else layer
    todo = [e for e in experts if (w, lk, e) not in _weights]
    if todo:
        for e, t in gen.expert_weights_many(w, lk, todo).items():
            _weights[(w, lk, e)] = t


def weights(w, layer, e):
    lk = 0 if w.shared_layer else layer
    if (w, lk, e) not in _weights:
        _weights[(w, lk, e)] = gen.expert_weights(w, lk, e)
    return _weights[(w, lk, e)]


# ------------------------------------------------------------------------- router

@pytest.mark.parametrize("wl,T,renorm", [
    (W.TINY, 4, 1), (W.TINY, 4, 0), (W.DECODE_35B, 1, 1), (W.DECODE_35B, 4, 1),
    (W.DECODE_35B, 8, 1), (W.DECODE_35B, 13, 1), (W.DECODE_284B, 1, 1), (W.DECODE_284B, 6, 0),
    (W.PREFILL_35B, 2048, 1)])
def test_route_bit_exact(m, wl, T, renorm):
    x = gen.activations(wl, 0, 5, T)
    wr = gen.router_weight(wl, 0)
    b = gen.router_bias(wl, 0)
    idx_r, w_r, l_r = oracle.route(x, wr, b, wl.k, renorm)
    idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(m.route_workspace_bytes(T, wl.E), dtype=torch.uint8, device="cuda")
    for rep in range(2):   # the second call checks that the tile counters were reset
        m.route(bf16(x), bf16(wr), dev(b), wl.k, renorm, idx, w, ws)
        torch.cuda.synchronize()
        logits = ws[:T * wl.E * 4].view(torch.float32).view(T, wl.E).cpu().numpy()
        assert np.array_equal(logits.view(np.uint32), l_r.view(np.uint32))
        assert np.array_equal(idx.cpu().numpy(), idx_r)
        np.testing.assert_allclose(w.cpu().numpy(), w_r, rtol=3e-6, atol=1e-7)


def test_route_ties_go_to_lower_index(m):
    wl = W.DECODE_35B
    x = gen.activations(wl, 0, 1, 3)
    xf = gen.bf16_bits_to_f32(x)
    wr = gen.router_weight(wl, 0).copy()
    b = np.zeros(wl.E, np.float32)
    wr[4] = gen.f32_to_bf16_bits((np.sign(xf[0]) * 0.05).astype(np.float32))  # top for token 0
    wr[9] = wr[4]        # exact ties: experts 4 and 9, 20 and 70
    wr[70] = wr[20]
    idx_r, w_r, l_r = oracle.route(x, wr, b, wl.k, 1)
    assert l_r[0, 4] == l_r[0, 9] and list(idx_r[0, :2]) == [4, 9]
    idx = torch.empty((3, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((3, wl.k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(m.route_workspace_bytes(3, wl.E), dtype=torch.uint8, device="cuda")
    m.route(bf16(x), bf16(wr), dev(b), wl.k, 1, idx, w, ws)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_r)


# ------------------------------------------------------------------------- lookup

@pytest.mark.parametrize("E,k,L,S,T,steps,skew", [(16, 2, 3, 8, 4, 60, 0.0), (128, 8, 4, 64, 8, 40, 1.0),
                                                  (256, 6, 5, 13, 1, 80, 0.5)])
def test_lookup_bit_exact_against_oracle_lru(m, E, k, L, S, T, steps, skew):
    pool = m.Pool(256, 256, E, k, L, "mxfp4", S, max_tokens=min(T, 16))
    ref = oracle.LRU(S, L, E)
    rng = np.random.default_rng(E + S)
    p = 1.0 / np.arange(1, E + 1) ** skew
    p /= p.sum()
    slot_of = torch.empty((T, k), dtype=torch.int32, device="cuda")
    for step in range(steps):
        layer = int(rng.integers(L))
        idx = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
        res = m.slot_lookup(pool, layer, dev(idx), slot_of)
        r = ref.step(layer, idx)
        assert res.uniq[:res.n_uniq].tolist() == r["uniq"].tolist()
        assert res.is_hit[:res.n_uniq].astype(bool).tolist() == r["hit"].tolist()
        ml = res.miss_list()
        assert [e for e, _, _, _ in ml] == r["miss_expert"].tolist()
        assert [s for _, s, _, _ in ml] == r["miss_slot"].tolist()
        assert [v for _, _, _, v in ml] == r["evicted"].tolist()
        assert np.array_equal(slot_of.cpu().numpy(), r["slot_of"])
        st, so = pool.read_state(), ref.state()
        assert np.array_equal(st["slot_key"], so["slot_key"])
        assert np.array_equal(st["slot_clock"], so["slot_clock"])
        assert np.array_equal(st["key_slot"], so["key_slot"])
        assert st["clock"] == so["clock"]
    s = pool.stats()
    assert s["lookups"] == steps and s["hits"] + s["misses"] == s["unique"]
    pool.close()


def test_lookup_rejects_bad_expert(m):
    pool = m.Pool(256, 256, 16, 2, 1, "mxfp4", 8, max_tokens=4)
    slot_of = torch.empty((1, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(m._lib.MoeError) as e:
        m.slot_lookup(pool, 0, dev(np.array([[3, 16]], np.int32)), slot_of)
    assert e.value.code == m._lib.MOE_EBOUNDS
    pool.close()


# ------------------------------------------------------------------- load + dequant

def make_resident(m, pool, w, layer, experts):
    """Load the experts' host blocks, look them up (k distinct per token) and
    stream them into slots; returns {(layer, expert): slot}."""
    experts = list(experts)
    assert len(experts) % pool.k == 0
    for e in experts:
        pool.load_expert(layer, e, weights(w, layer, e))
    idx = np.array(experts, np.int32).reshape(-1, pool.k)
    slot_of = torch.empty(idx.shape, dtype=torch.int32, device="cuda")
    res = m.slot_lookup(pool, layer, dev(idx), slot_of)
    cs = torch.cuda.Stream()
    m.stream_misses(pool, layer, res, cs)
    cs.synchronize()
    return {(layer, int(e)): int(s) for e, s in zip(idx.ravel(), slot_of.cpu().numpy().ravel())}


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_dequantised_slots_bit_exact(m, fmt):
    w = small("dq", fmt, H=512, I=256, E=6, k=2, L=2)
    pool = m.Pool(w.H, w.I, w.E, w.k, w.L, fmt, 12, max_tokens=4)
    res = {}
    for layer in range(2):
        res.update(make_resident(m, pool, w, layer, range(w.E)))
    for (layer, e), s in res.items():
        t = weights(w, layer, e)
        for which, name in enumerate(("gate", "up", "down")):
            c, sc, ts = t[name]
            rows, K = c.shape[0], c.shape[1] * 2
            out = torch.empty((rows, K), dtype=torch.float32, device="cuda")
            m.dequant_slot(pool, s, layer * w.E + e, which, out)
            ref = oracle.dequant(fmt, c, sc, ts)
            got = out.cpu().numpy()
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), (layer, e, name)
    pool.close()


# ------------------------------------------------------------------------ combine

def test_combine_rounds_rank_ordered_fp32_sum(m):
    rng = np.random.default_rng(4)
    yp = rng.standard_normal((5, 6, 512)).astype(np.float32)
    y = torch.empty((5, 512), dtype=torch.bfloat16, device="cuda")
    m.combine(dev(yp), y)
    torch.cuda.synchronize()
    s = np.zeros((5, 512), np.float32)
    for j in range(6):
        s = (s + yp[:, j]).astype(np.float32)
    assert np.array_equal(host_bits(y), gen.f32_to_bf16_bits(s))


# ------------------------------------------------------------------ decode layer

def run_layer(m, pool, w, layer, step, T, layer_obj, zipf=None, renorm=1):
    """One decode layer on the GPU, loading missed experts' host blocks on demand."""
    x = gen.activations(w, layer, step, T)
    wr = gen.router_weight(w, layer)
    b = gen.router_bias(w, layer, zipf)
    xd, wrd, bd = bf16(x), bf16(wr), dev(b)
    lo = layer_obj
    m.route(xd, wrd, bd, w.k, renorm, lo.idx, lo.w, lo.ws)
    m.slot_lookup(pool, layer, lo.idx, lo.slot_of, lo.lookup)
    misses = lo.lookup.miss_list()
    prefetch(w, layer, [e for e, _, _, _ in misses])
    for e, _, _, _ in misses:
        pool.load_expert(layer % pool.host_layers, e, weights(w, layer, e))
    m.stream_misses(pool, layer, lo.lookup, lo.copy_stream)
    lo.status.zero_()
    m.expert_ffn(pool, layer, xd, lo.idx, lo.w, lo.slot_of, lo.y_part, lo.status)
    m.combine(lo.y_part, lo.y)
    torch.cuda.synchronize()
    return x, wr, b


def check_layer(w, lo, x, wr, b, layer, renorm=1):
    idx_r, w_r, _ = oracle.route(x, wr, b, w.k, renorm)
    assert np.array_equal(lo.idx.cpu().numpy(), idx_r)
    assert int(lo.status.item()) == 0
    chosen = sorted(set(idx_r.ravel().tolist()))
    ex = {e: weights(w, layer, e) for e in chosen}
    yf, _ = oracle.moe_decode(w.fmt, w.H, w.I, w.E, x, idx_r, w_r, ex)
    y = lo.y.float().cpu().numpy()
    rms = float(np.sqrt(np.mean(yf.astype(np.float64) ** 2)))
    err = float(np.max(np.abs(y - yf)))
    assert err <= TOL * rms, (err, rms)
    return err / rms


@pytest.mark.parametrize("fmt,H,I,E,k,S,T", [
    ("mxfp4", 256, 256, 16, 2, 16, 4),     # the tiny workload's shape, all resident
    ("nvfp4", 512, 256, 8, 2, 6, 3),       # misses every step, ragged T
    ("nvfp4", 768, 512, 12, 3, 12, 16),    # max tokens: pool holds one layer, misses on switch
    ("mxfp4", 1024, 768, 10, 4, 8, 2),
    ("mxfp4", 512, 512, 16, 4, 16, 12)])   # MXFP4 past 8 tokens (two 8-column tiles)
def test_decode_layer_small(m, fmt, H, I, E, k, S, T):
    w = small(f"d{H}", fmt, H=H, I=I, E=E, k=k, L=2)
    pool = m.Pool(H, I, E, k, 2, fmt, S, max_tokens=T)
    lo = m.DecodeLayer(pool, T)
    for step in range(3):
        for layer in range(2):
            x, wr, b = run_layer(m, pool, w, layer, step, T, lo)
            check_layer(w, lo, x, wr, b, layer)
    st = pool.stats()
    assert st["misses"] > 0 and st["h2d_copies"] == st["misses"]
    pool.close()


def test_decode_tiny_workload(m):
    w = W.TINY
    pool = m.Pool(w.H, w.I, w.E, w.k, 1, w.fmt, 16, max_tokens=4)
    lo = m.DecodeLayer(pool, 4)
    for rep in range(2):
        x, wr, b = run_layer(m, pool, w, 0, 0, 4, lo)
        check_layer(w, lo, x, wr, b, 0)
    pool.close()


@pytest.mark.parametrize("T", [1, 4, 8])
def test_decode_35b_shapes_sampled(m, T):
    """Full decode_35b layer shape (H=2048, I=768, E=128, k=8, NVFP4), a 25% pool
    over 2 layer positions, outputs checked on every (step, layer) run."""
    w = W.DECODE_35B
    pool = m.Pool(w.H, w.I, w.E, w.k, 2, w.fmt, 64, max_tokens=T, host_layers=2)
    lo = m.DecodeLayer(pool, T)
    for step in range(2):
        for layer in range(2):
            x, wr, b = run_layer(m, pool, w, layer, step, T, lo)
            check_layer(w, lo, x, wr, b, layer)
    pool.close()


def test_decode_284b_shapes_sampled(m):
    """decode_284b layer shape (H=4096, I=2048, E=256, k=6, MXFP4), small pool."""
    w = W.DECODE_284B
    pool = m.Pool(w.H, w.I, w.E, w.k, 2, w.fmt, 8, max_tokens=1, host_layers=2)
    lo = m.DecodeLayer(pool, 1)
    for step in range(2):
        for layer in range(2):
            x, wr, b = run_layer(m, pool, w, layer, step, 1, lo)
            check_layer(w, lo, x, wr, b, layer)
    pool.close()


# ------------------------------------------------------------ bounded waits / faults

def test_missing_copy_times_out_with_status_and_recovers(m):
    """A missed expert whose copy is never issued: the FFN's bounded wait gives up,
    sets MOE_STATUS_READY_TIMEOUT and the kernel returns; after streaming the
    miss the same call succeeds."""
    w = small("to", "mxfp4", H=256, I=256, E=8, k=2, L=1)
    pool = m.Pool(w.H, w.I, w.E, w.k, 1, "mxfp4", 8, max_tokens=2)
    for e in range(w.E):
        pool.load_expert(0, e, weights(w, 0, e))
    lo = m.DecodeLayer(pool, 2)
    x = gen.activations(w, 0, 0, 2)
    wr = gen.router_weight(w, 0)
    b = gen.router_bias(w, 0)
    xd = bf16(x)
    m.route(xd, bf16(wr), dev(b), w.k, 1, lo.idx, lo.w, lo.ws)
    m.slot_lookup(pool, 0, lo.idx, lo.slot_of, lo.lookup)
    assert lo.lookup.n_miss > 0
    try:
        m.set_wait_limits(50, 50, 2000)
        lo.status.zero_()
        m.expert_ffn(pool, 0, xd, lo.idx, lo.w, lo.slot_of, lo.y_part, lo.status)
        torch.cuda.synchronize()
        assert int(lo.status.item()) & m._lib.STATUS_READY_TIMEOUT
    finally:
        m.set_wait_limits(5000, 5000, 10000)
    m.stream_misses(pool, 0, lo.lookup, lo.copy_stream)
    lo.status.zero_()
    m.expert_ffn(pool, 0, xd, lo.idx, lo.w, lo.slot_of, lo.y_part, lo.status)
    m.combine(lo.y_part, lo.y)
    torch.cuda.synchronize()
    check_layer(w, lo, x, wr, b, 0)
    pool.close()


def test_bad_slot_index_is_reported_not_used(m):
    w = small("bs", "mxfp4", H=256, I=256, E=8, k=2, L=1)
    pool = m.Pool(w.H, w.I, w.E, w.k, 1, "mxfp4", 8, max_tokens=1)
    lo = m.DecodeLayer(pool, 1)
    xd = bf16(gen.activations(w, 0, 0, 1))
    idx = dev(np.array([[1, 2]], np.int32))
    wt = dev(np.array([[0.5, 0.5]], np.float32))
    slot_of = dev(np.array([[0, 99]], np.int32))
    lo.status.zero_()
    m.set_wait_limits(50, 50, 2000)
    try:
        m.expert_ffn(pool, 0, xd, idx, wt, slot_of, lo.y_part, lo.status)
        torch.cuda.synchronize()
    finally:
        m.set_wait_limits(5000, 5000, 10000)
    assert int(lo.status.item()) & m._lib.STATUS_BAD_SLOT
    pool.close()


def test_decode_layer_call_with_misses_matches_oracle(m):
    """The public DecodeLayer call (FFN enqueued before the host drives the copy
    engine) over steps and layers with misses."""
    w = small("dl", "nvfp4", H=512, I=512, E=16, k=4, L=3, zipf=0.8)
    T = 4
    pool = m.Pool(w.H, w.I, w.E, w.k, w.L, w.fmt, 16, max_tokens=T)
    for layer in range(w.L):
        for e in range(w.E):
            pool.load_expert(layer, e, weights(w, layer, e))
    lo = m.DecodeLayer(pool, T)
    for step in range(3):
        for layer in range(w.L):
            x = gen.activations(w, layer, step, T)
            wr = gen.router_weight(w, layer)
            b = gen.router_bias(w, layer)
            lo(layer, bf16(x), bf16(wr), dev(b))
            torch.cuda.synchronize()
            check_layer(w, lo, x, wr, b, layer)
    assert pool.stats()["misses"] > 0
    pool.close()


def test_native_layer_call_matches_step_by_step_calls(m):
    """moe_decode_layer (one native call per layer, with and without overlap) and
    the same layer issued call by call from Python give bit-identical outputs,
    miss lists and LRU state; the copy-event hook records one pair per layer
    with misses."""
    w = small("nl", "mxfp4", H=256, I=256, E=16, k=4, L=2, zipf=0.5)
    T = 3
    pools, layers = [], []
    for mode in ("native", "native_serial", "python"):
        pool = m.Pool(w.H, w.I, w.E, w.k, w.L, w.fmt, 12, max_tokens=T)
        for layer in range(w.L):
            for e in range(w.E):
                pool.load_expert(layer, e, weights(w, layer, e))
        lo = m.DecodeLayer(pool, T, overlap=(mode != "native_serial"))
        if mode == "python":
            lo.ffn_events = []
        lo.copy_events = []
        pools.append(pool)
        layers.append(lo)
    for step in range(3):
        for layer in range(w.L):
            x = gen.activations(w, layer, step, T)
            wr = gen.router_weight(w, layer)
            b = gen.router_bias(w, layer)
            outs = []
            for lo in layers:
                y = lo(layer, bf16(x), bf16(wr), dev(b))
                torch.cuda.synchronize()
                assert int(lo.status.item()) == 0
                outs.append((host_bits(y), lo.lookup.miss_list()))
            for o in outs[1:]:
                assert np.array_equal(o[0], outs[0][0]) and o[1] == outs[0][1]
    states = [p.read_state() for p in pools]
    for st in states[1:]:
        for key in states[0]:
            assert np.array_equal(st[key], states[0][key]), key
    n_layers_with_misses = len(layers[0].copy_events)
    assert n_layers_with_misses > 0
    assert all(len(lo.copy_events) == n_layers_with_misses for lo in layers)
    assert all(ev[0].elapsed_time(ev[1]) >= 0.0 for ev, _ in layers[0].copy_events)
    for p in pools:
        p.close()


@pytest.mark.parametrize("mode", ["sm", "dma"])
def test_copy_modes_fill_slots_identically(m, mode):
    """Both miss-copy paths (SM loads of the mapped host store, copy engine) put
    the expert's exact host bytes into the slot and give oracle-exact outputs."""
    w = small("cm", "nvfp4", H=512, I=256, E=16, k=4, L=2, zipf=0.3)
    T = 2
    pool = m.Pool(w.H, w.I, w.E, w.k, w.L, w.fmt, 8, max_tokens=T)
    pool.set_copy_mode(mode)
    for layer in range(w.L):
        for e in range(w.E):
            pool.load_expert(layer, e, weights(w, layer, e))
    lo = m.DecodeLayer(pool, T)
    for step in range(2):
        for layer in range(w.L):
            x = gen.activations(w, layer, step, T)
            wr = gen.router_weight(w, layer)
            b = gen.router_bias(w, layer)
            lo(layer, bf16(x), bf16(wr), dev(b))
            torch.cuda.synchronize()
            check_layer(w, lo, x, wr, b, layer)
            for e, slot, _, _ in lo.lookup.miss_list():
                for which, name in enumerate(("gate", "up", "down")):
                    codes, scales, ts = weights(w, layer, e)[name]
                    rows, K = codes.shape[0], codes.shape[1] * 2
                    out = torch.empty((rows, K), dtype=torch.float32, device="cuda")
                    m.dequant_slot(pool, slot, layer * w.E + e, which, out)
                    ref = oracle.dequant(w.fmt, codes, scales, ts)
                    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert pool.stats()["misses"] > 0
    pool.close()


def test_pool_resize_keeps_lru_state_and_outputs(m):
    """Shrink and grow a live pool between steps: the slot table follows the
    oracle's resize bit for bit (moved blocks included) and later layers still
    match the oracle."""
    w = small("rs", "mxfp4", H=256, I=256, E=16, k=2, L=2, zipf=0.7)
    T = 2
    pool = m.Pool(w.H, w.I, w.E, w.k, w.L, w.fmt, 12, max_tokens=T)
    for layer in range(w.L):
        for e in range(w.E):
            pool.load_expert(layer, e, weights(w, layer, e))
    ref = oracle.LRU(12, w.L, w.E)
    lo = m.DecodeLayer(pool, T)

    def steps(s0, n):
        for step in range(s0, s0 + n):
            for layer in range(w.L):
                x = gen.activations(w, layer, step, T)
                wr = gen.router_weight(w, layer)
                b = gen.router_bias(w, layer)
                lo(layer, bf16(x), bf16(wr), dev(b))
                torch.cuda.synchronize()
                check_layer(w, lo, x, wr, b, layer)
                r = ref.step(layer, lo.idx.cpu().numpy())
                assert [s for _, s, _, _ in lo.lookup.miss_list()] == r["miss_slot"].tolist()

    def same_state(n_active):
        got, want = pool.read_state(), ref.state()
        assert got["slot_key"][:n_active].tolist() == want["slot_key"].tolist()
        assert (got["slot_key"][n_active:] < 0).all()
        assert got["slot_clock"][:n_active].tolist() == want["slot_clock"].tolist()
        assert np.array_equal(got["key_slot"], want["key_slot"]) and got["clock"] == want["clock"]

    steps(0, 4)
    same_state(12)
    pool.resize(5)
    ref.resize(5)
    same_state(5)
    steps(4, 3)
    same_state(5)
    pool.resize(12)
    ref.resize(12)
    same_state(12)
    steps(7, 2)
    same_state(12)
    pool.close()


def test_pool_reset_restricts_active_slots(m):
    """After a reset to n active slots the LRU behaves as a fresh n-slot pool."""
    E, k, L = 32, 4, 2
    pool = m.Pool(256, 256, E, k, L, "mxfp4", 24, max_tokens=2)
    rng = np.random.default_rng(3)
    slot_of = torch.empty((2, k), dtype=torch.int32, device="cuda")
    for _ in range(10):
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(2)]).astype(np.int32)
        m.slot_lookup(pool, 0, dev(idx), slot_of)
    pool.reset(8)
    ref = oracle.LRU(8, L, E)
    for step in range(30):
        layer = step % L
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(2)]).astype(np.int32)
        res = m.slot_lookup(pool, layer, dev(idx), slot_of)
        r = ref.step(layer, idx)
        assert [s for _, s, _, _ in res.miss_list()] == r["miss_slot"].tolist()
        assert np.array_equal(slot_of.cpu().numpy(), r["slot_of"])
        assert slot_of.cpu().numpy().max() < 8
    st = pool.stats()
    assert st["lookups"] == 30
    pool.close()
