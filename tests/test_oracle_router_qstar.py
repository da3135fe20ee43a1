"""Pins of the oracle's router (logits, top-k, weights) and of q*."""
import math

import numpy as np
import pytest
import scipy.special

from conftest import read_golden
from synthetic import gen, workloads as W


# ---------------------------------------------------------------------------- q*

def test_qstar_reproduces_printed_table(orc):
    rows = read_golden("qstar_table.txt")
    assert len(rows) == 4
    for _, bp, bh, pct in rows:
        qg, qc, r = orc.qstar_split(256, float(bp), float(bh))
        assert f"{100 * r:.1f}" == pct
        assert qg + qc == 256


def test_qstar_ratio_form_of_second_page(orc):
    # pull : compute = pcie_bw : (cpu_bw - pcie_bw)  ->  pull share = B_p / B_h
    for _, bp, bh, _ in read_golden("qstar_table.txt"):
        bp, bh = float(bp), float(bh)
        share = bp / (bp + (bh - bp))
        assert orc.qstar_split(10, bp, bh)[2] == pytest.approx(share, rel=1e-15)


@pytest.mark.parametrize("m,bp,bh,qg", [
    (6, 49.0, 53.8, 5), (6, 11.8, 47.5, 1), (0, 10, 20, 0), (7, 60, 50, 7), (4, 1, 8, 1),
    (1, 1, 2, 1)])   # 0.5 rounds half up
def test_qstar_counts(orc, m, bp, bh, qg):
    g, c, _ = orc.qstar_split(m, bp, bh)
    assert (g, c) == (qg, m - qg)


def test_qstar_rejects_bad_args(orc):
    with pytest.raises(ValueError):
        orc.qstar_split(3, 0.0, 10.0)
    with pytest.raises(ValueError):
        orc.qstar_split(-1, 1.0, 10.0)


# ------------------------------------------------------------------------- router

def _inputs(w, T, layer=0, step=0):
    x = gen.activations(w, layer, step, T)
    wr = gen.router_weight(w, layer)
    b = gen.router_bias(w, layer)
    return x, wr, b


@pytest.mark.parametrize("wl,T", [(W.TINY, 4), (W.DECODE_35B, 8), (W.DECODE_284B, 2)])
def test_logits_within_fp32_error_bound_of_exact_dot(orc, wl, T):
    x, wr, b = _inputs(wl, T)
    got = orc.router_logits(x, wr, b).astype(np.float64)
    xf = gen.bf16_bits_to_f32(x).astype(np.float64)
    wf = gen.bf16_bits_to_f32(wr).astype(np.float64)
    exact = xf @ wf.T + b.astype(np.float64)
    absdot = np.abs(xf) @ np.abs(wf).T + np.abs(b)
    n = wl.H // 32 + 5 + 1          # longest chain of fp32 roundings per logit
    bound = 1.01 * n * 2.0 ** -24 * absdot
    assert np.all(np.abs(got - exact) <= bound)
    # a dropped chunk or a transposed operand is far outside this bound
    assert np.max(np.abs(got - exact) / absdot) < 1e-5


def test_topk_matches_full_sort(orc):
    x, wr, b = _inputs(W.DECODE_35B, 8)
    l = orc.router_logits(x, wr, b)
    idx = orc.topk(l, 8)
    for t in range(8):
        order = np.lexsort((np.arange(l.shape[1]), -l[t].astype(np.float64)))
        assert list(idx[t]) == list(order[:8])


def test_topk_ties_go_to_lower_index(orc):
    l = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 0.0],
                  [5.0, 5.0, 5.0, 5.0, 5.0, 5.0]], np.float32)
    assert orc.topk(l, 3).tolist() == [[1, 2, 4], [0, 1, 2]]


def test_weights_are_softmax_of_chosen(orc):
    x, wr, b = _inputs(W.DECODE_35B, 8)
    idx, w, l = orc.route(x, wr, b, 8, renormalize=1)
    for t in range(8):
        ref = scipy.special.softmax(l[t, idx[t]].astype(np.float64))
        np.testing.assert_allclose(w[t], ref, rtol=1e-6)
        assert abs(w[t].sum() - 1.0) < 1e-6
        assert np.all(np.diff(w[t]) <= 0)          # rank order = descending weight
    idx0, w0, _ = orc.route(x, wr, b, 8, renormalize=0)
    assert np.array_equal(idx0, idx)
    for t in range(8):
        full = scipy.special.softmax(l[t].astype(np.float64))
        np.testing.assert_allclose(w0[t], full[idx[t]], rtol=1e-6)
        assert w0[t].sum() < 1.0


def test_routing_is_permutation_equivariant(orc):
    x, wr, b = _inputs(W.TINY, 4)
    perm = np.random.default_rng(3).permutation(wr.shape[0])
    idx, w, _ = orc.route(x, wr, b, 2)
    idx_p, w_p, _ = orc.route(x, wr[perm], b[perm], 2)
    assert np.array_equal(perm[idx_p], idx)
    np.testing.assert_array_equal(w_p, w)


def test_zipf_bias_skews_routing(orc):
    """Skewed routing concentrates choices (high hit rate), s=0 spreads them."""
    w = W.DECODE_35B
    counts = {}
    for s in (0.0, 1.1):
        c = np.zeros(w.E)
        for step in range(16):
            x = gen.activations(w, 0, step, 8)
            idx, _, _ = orc.route(x, gen.router_weight(w, 0), gen.router_bias(w, 0, s), w.k)
            np.add.at(c, idx.ravel(), 1)
        counts[s] = np.sort(c)[::-1]
    assert counts[1.1][:16].sum() > 2 * counts[0.0][:16].sum()
