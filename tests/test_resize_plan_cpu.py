"""The library's slot-pool resize decision (moe_lru_plan_resize, host code, no GPU)
against the oracle's resize on random LRU states."""
import numpy as np
import pytest

from expert_offload_fp4_b200.api import lru_plan_resize


def _random_state(orc, S, L, E, steps, seed):
    rng = np.random.default_rng(seed)
    pool = orc.LRU(S, L, E)
    p = 1.0 / np.arange(1, E + 1) ** 0.8
    p /= p.sum()
    for s in range(steps):
        idx = rng.choice(E, (1, 3), replace=False, p=p).astype(np.int32)
        pool.step(s % L, idx)
    return pool


def _apply(st, evicted, moves, n_new):
    sk, sc = st["slot_key"].copy(), st["slot_clock"].copy()
    for s in evicted:
        sk[s], sc[s] = -1, 0
    for a, b in moves:
        assert sk[b] < 0, "a move must land in a free slot"
        sk[b], sc[b] = sk[a], sc[a]
        sk[a], sc[a] = -1, 0
    assert (sk[n_new:] < 0).all() if n_new < len(sk) else True
    return sk[:n_new], sc[:n_new]


@pytest.mark.parametrize("S,n_new,steps,seed", [(16, 5, 40, 1), (16, 15, 40, 2), (32, 3, 200, 3),
                                                 (9, 9, 30, 4), (12, 20, 30, 5), (40, 1, 100, 6),
                                                 (24, 8, 3, 7)])
def test_plan_matches_oracle_resize(orc, S, n_new, steps, seed):
    pool = _random_state(orc, S, 3, 24, steps, seed)
    st = pool.state()
    evicted, moves = lru_plan_resize(st["slot_key"], st["slot_clock"], n_new)
    n_ev = pool.resize(n_new)
    ref = pool.state()
    assert len(evicted) == n_ev
    if n_new >= S:
        assert evicted == [] and moves == []
        return
    sk, sc = _apply(st, evicted, moves, n_new)
    assert sk.tolist() == ref["slot_key"].tolist()
    assert sc.tolist() == ref["slot_clock"].tolist()


def test_plan_rejects_bad_sizes():
    from expert_offload_fp4_b200._lib import MoeError
    with pytest.raises(MoeError):
        lru_plan_resize(np.array([-1, 3], np.int32), np.array([0, 1], np.uint64), 0)
