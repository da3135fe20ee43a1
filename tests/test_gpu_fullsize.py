"""GPU parity at the workloads' full sizes.

* The LRU slot lookup against the oracle's LRU on the real pool sizes (1536
  slots of the 35B-A3B decode, 2570 of the 284B decode, 1024 / 2560 / 5120 of
  the cache-stress sweep), with Zipf-skewed routing traces long enough to evict
  many times: after every lookup the whole slot table, every clock, the key
  table, the miss list and the victims must agree bit for bit.
* Routing of every cache-stress variant (Zipf exponent 0, 0.6, 1.0, 1.4, its
  permutation re-drawn per layer) bit-exact against the oracle.
* The 284B layer on its 2570-slot (32 GiB) pool over several layer positions,
  outputs within 2e-2 * rms of the oracle.
* Every token of the 2048-token prefill prompt of the 35B-A3B layer against the
  oracle's batched prefill.
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


# ------------------------------------------------------------------ LRU, full pools

def zipf_trace(rng, E, k, T, s, perm):
    """k distinct experts per token, P(expert) proportional to rank^-s, ranks from a
    per-layer permutation."""
    rank = np.empty(E, np.int64)
    rank[perm] = np.arange(1, E + 1)
    p = 1.0 / rank.astype(np.float64) ** s
    p /= p.sum()
    return np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


LOOKUP_CASES = [
    # (name, E, k, L, S, T, zipf)
    ("decode_35b_pool", 128, 8, 48, 1536, 1, 1.1),
    ("decode_35b_pool_t8", 128, 8, 48, 1536, 8, 1.1),
    ("decode_284b_pool", 256, 6, 40, 2570, 1, 1.0),
] + [(f"stress_s{s:g}_p{int(f * 100)}", 256, 6, 40, int(round(f * 40 * 256)), 1, s)
     for s in W.STRESS_ZIPF for f in W.STRESS_POOL]


@pytest.mark.parametrize("name,E,k,L,S,T,zipf", LOOKUP_CASES, ids=[c[0] for c in LOOKUP_CASES])
def test_lookup_full_pool_bit_exact(m, name, E, k, L, S, T, zipf):
    # small expert blocks: the lookup never reads the weights
    pool = m.Pool(256, 256, E, k, L, "mxfp4", S, max_tokens=min(T, 16), host_layers=1)
    ref = oracle.LRU(S, L, E)
    rng = np.random.default_rng(S + 7 * E + int(zipf * 10) + T)
    perms = [rng.permutation(E) for _ in range(L)]
    # at least 300 lookups; past that, stop once 200 victims have been chosen, or
    # after enough lookups to fill the pool three times over
    cap = max(300, 3 * S // min(T * k, E) + 300)
    slot_of = torch.empty((T, k), dtype=torch.int32, device="cuda")
    evictions, seen, n = 0, set(), 0
    while n < cap and not (n >= 300 and evictions >= 200):
        layer = n % L                                       # layers in decode order
        idx = zipf_trace(rng, E, k, T, zipf, perms[layer])
        seen.update(layer * E + int(e) for e in idx.ravel())
        res = m.slot_lookup(pool, layer, dev(idx), slot_of)
        r = ref.step(layer, idx)
        assert res.uniq[:res.n_uniq].tolist() == r["uniq"].tolist(), n
        assert res.is_hit[:res.n_uniq].astype(bool).tolist() == r["hit"].tolist(), n
        ml = res.miss_list()
        assert [e for e, _, _, _ in ml] == r["miss_expert"].tolist(), n
        assert [s for _, s, _, _ in ml] == r["miss_slot"].tolist(), n
        assert [v for _, _, _, v in ml] == r["evicted"].tolist(), n
        evictions += sum(v >= 0 for _, _, _, v in ml)
        assert np.array_equal(slot_of.cpu().numpy(), r["slot_of"]), n
        st, so = pool.read_state(), ref.state()
        assert np.array_equal(st["slot_key"], so["slot_key"]), n
        assert np.array_equal(st["slot_clock"], so["slot_clock"]), n
        assert np.array_equal(st["key_slot"], so["key_slot"]), n
        assert st["clock"] == so["clock"], n
        n += 1
    # victims were searched whenever more keys were touched than the pool holds
    assert (evictions > 0) == (len(seen) > S), (evictions, len(seen))
    pool.close()


# --------------------------------------------------------------- stress routing

@pytest.mark.parametrize("zipf", W.STRESS_ZIPF)
def test_route_stress_variants_bit_exact(m, zipf):
    """Routing of the cache-stress sweep: 284B router weights and the Zipf bias of
    each exponent, on several layer positions (each has its own permutation)."""
    w = W.STRESS_284B
    idx = torch.empty((1, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((1, w.k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(m.route_workspace_bytes(1, w.E), dtype=torch.uint8, device="cuda")
    for layer in (0, 1, 17, 39):
        wr = gen.router_weight(w, layer)
        b = gen.router_bias(w, layer, zipf)
        wrd, bd = bf16(wr), dev(b)
        for step in range(3):
            x = gen.activations(w, layer, step, 1)
            idx_r, w_r, l_r = oracle.route(x, wr, b, w.k, 1)
            m.route(bf16(x), wrd, bd, w.k, 1, idx, wt, ws)
            torch.cuda.synchronize()
            logits = ws[:w.E * 4].view(torch.float32).cpu().numpy()
            assert np.array_equal(logits.view(np.uint32), l_r.ravel().view(np.uint32))
            assert np.array_equal(idx.cpu().numpy(), idx_r)
            np.testing.assert_allclose(wt.cpu().numpy(), w_r, rtol=3e-6, atol=1e-7)


# ------------------------------------------------------------ 284B on its full pool

def test_decode_284b_on_full_pool(m):
    """The 284B decode layer (H=4096, I=2048, E=256, k=6, MXFP4) on its 2570-slot
    32 GiB pool over 40 layer positions: layers 0..3 for two steps, every output
    within tolerance of the oracle; missed experts' host blocks are packed right
    before their copy (one host layer serves every position)."""
    w = W.DECODE_284B
    S = W.n_slots(w)
    assert S == 2570
    pool = m.Pool(w.H, w.I, w.E, w.k, w.L, w.fmt, S, max_tokens=1, host_layers=1)
    lo = m.DecodeLayer(pool, 1)
    cache = {}
    for step in range(2):
        for layer in range(4):
            x = gen.activations(w, layer, step, 1)
            wr = gen.router_weight(w, layer)
            b = gen.router_bias(w, layer)
            xd = bf16(x)
            m.route(xd, bf16(wr), dev(b), w.k, 1, lo.idx, lo.w, lo.ws)
            m.slot_lookup(pool, layer, lo.idx, lo.slot_of, lo.lookup)
            idx_r, w_r, _ = oracle.route(x, wr, b, w.k, 1)
            assert np.array_equal(lo.idx.cpu().numpy(), idx_r)
            for e in idx_r.ravel().tolist():
                if (layer, e) not in cache:
                    cache[(layer, e)] = gen.expert_weights(w, layer, e)
            for e, _, _, _ in lo.lookup.miss_list():
                pool.load_expert(0, e, cache[(layer, e)])
            m.stream_misses(pool, layer, lo.lookup, lo.copy_stream)
            lo.status.zero_()
            m.expert_ffn(pool, layer, xd, lo.idx, lo.w, lo.slot_of, lo.y_part, lo.status)
            m.combine(lo.y_part, lo.y)
            torch.cuda.synchronize()          # the copies have landed: the host block may change
            assert int(lo.status.item()) == 0
            yf, _ = oracle.moe_decode(w.fmt, w.H, w.I, w.E, x, idx_r, w_r,
                                      {e: cache[(layer, e)] for e in set(idx_r.ravel().tolist())})
            y = lo.y.float().cpu().numpy()
            rms = float(np.sqrt(np.mean(yf.astype(np.float64) ** 2)))
            assert float(np.max(np.abs(y - yf))) <= TOL * rms, (step, layer)
    st = pool.stats()
    assert st["misses"] == len(cache) and st["hits"] == st["unique"] - st["misses"]
    pool.close()


# ----------------------------------------------------- the whole 2048-token prompt

def test_prefill_35b_every_token(m):
    """Every token of the prefill_35b prompt (2048 tokens routed top-8 over 128
    experts, uneven groups) within 2e-2 * rms of the oracle's batched prefill."""
    from oracle import prefill_batch
    w = W.PREFILL_35B
    T = 2048
    experts = gen.expert_weights_many(w, 0, range(w.E))
    x = gen.activations(w, 0, 0, T)
    wr = gen.router_weight(w, 0)
    b = gen.router_bias(w, 0)
    pool = m.Pool(w.H, w.I, w.E, w.k, 1, w.fmt, w.E, max_tokens=1)
    for e in range(w.E):
        pool.load_expert(0, e, experts[e])
    idx = torch.empty((T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, w.k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(m.route_workspace_bytes(T, w.E), dtype=torch.uint8, device="cuda")
    xd = bf16(x)
    m.route(xd, bf16(wr), dev(b), w.k, 1, idx, wt, ws)
    slot_of = torch.empty_like(idx)
    res = m.slot_lookup(pool, 0, idx, slot_of)
    cs = torch.cuda.Stream()
    m.stream_misses(pool, 0, res, cs)
    cs.synchronize()
    y_part = torch.full((T, w.k, w.H), float("nan"), dtype=torch.float32, device="cuda")
    work = torch.zeros(m.prefill_workspace_bytes(pool, T), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.prefill_ffn(pool, 0, xd, idx, wt, slot_of, y_part, work, status)
    y = torch.empty((T, w.H), dtype=torch.bfloat16, device="cuda")
    m.combine(y_part, y)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    idx_r, w_r, _ = oracle.route(x, wr, b, w.k, 1)
    assert np.array_equal(idx.cpu().numpy(), idx_r)
    counts = np.bincount(idx_r.ravel(), minlength=w.E)
    assert counts.min() < counts.max()
    ref = prefill_batch.moe_prefill(w.H, w.I, w.E, x, idx_r, w_r, experts)
    got = y.float().cpu().numpy()
    rms = np.sqrt(np.mean(ref.astype(np.float64) ** 2, axis=1))
    err = np.max(np.abs(got - ref), axis=1)
    bad = np.nonzero(err > TOL * rms)[0]
    assert bad.size == 0, (bad[:10].tolist(), float((err / rms).max()))
    pool.close()
