"""How much a cross-layer prefetch could know ahead of time on the decode_35b inputs.

The prefetch the source pages describe streams weights a coming layer will probably
need while the current layer computes.  It pays only if some cheap signal names a
layer's misses before its router runs, and names few experts that would not have
been used.  The synthetic decode_35b activations are drawn independently for every
(layer, step), so such a signal should do no better than a guess drawn from the
experts' popularity.  This replays the workload's routing with the oracle's router
and its global LRU (the 1536-slot pool) and measures, for layer l+1's misses, the
share each predictor names while layer l runs:
* "previous step": the experts layer l+1 chose at the previous step;
* "previous layer": layer l's input routed by the router the 48 positions share, i.e.
  the experts layer l chose;
* "popularity": k experts drawn by how often each was chosen so far;
and, for the previous-layer predictor, the copies a prefetch would issue (predicted
experts not resident for layer l+1) per miss it would save.  The reading that the
cross-layer predictor is left out on these inputs rests on these numbers.
"""
import numpy as np

import oracle
from synthetic import gen, workloads as W


def test_misses_are_not_predictable_on_independent_activations():
    w = W.DECODE_35B
    steps = 12
    lru = oracle.LRU(W.n_slots(w), w.L, w.E)
    wr = gen.router_weight(w, 0)
    b = gen.router_bias(w, 0)
    rng = np.random.default_rng(0)
    counts = np.ones(w.E)
    prev_step = {}
    covered = {"previous step": 0, "previous layer": 0, "popularity": 0}
    n_miss = copies = 0
    pending = None        # (layer, predicted set, non-resident predicted) made while the last layer ran
    for s in range(steps):
        prev_layer = None
        for layer in range(w.L):
            x = gen.activations(w, layer, s, 1)
            idx, _, _ = oracle.route(x, wr, b, w.k, 1)
            chosen = set(idx.ravel().tolist())
            r = lru.step(layer, idx)
            misses = set(r["miss_expert"].tolist())
            if s >= 2 and prev_layer is not None and layer in prev_step:   # the pool has filled by now
                n_miss += len(misses)
                covered["previous step"] += len(misses & prev_step[layer])
                covered["previous layer"] += len(misses & prev_layer)
                pop = rng.choice(w.E, w.k, replace=False, p=counts / counts.sum())
                covered["popularity"] += len(misses & set(pop.tolist()))
                copies += pending
            # what a prefetch for the next layer would copy now: its predicted experts
            # (this layer's) that the next layer does not hold
            nxt = layer + 1
            if nxt < w.L:
                key_slot = lru.state()["key_slot"]
                pending = sum(1 for e in chosen if key_slot[nxt * w.E + e] < 0)
            else:
                pending = 0
            for e in chosen:
                counts[e] += 1
            prev_step[layer] = chosen
            prev_layer = chosen
    assert n_miss > 100
    share = {k: v / n_miss for k, v in covered.items()}
    saved = covered["previous layer"]
    print({k: round(v, 3) for k, v in share.items()}, "misses", n_miss,
          "prefetch copies per saved miss", round(copies / max(saved, 1), 2))
    # the previous step's experts are resident already: nothing to fetch
    assert share["previous step"] < 0.02
    # the previous layer's choice is one more draw from the same popularity
    assert share["previous layer"] < share["popularity"] + 0.06
    # and a prefetch on it would move several blocks over PCIe for every miss it saves
    assert copies > 2 * saved
