"""Run-time bandwidth adaptation of q* (host functions of the C ABI, no GPU):
moving estimates of PCIe and host-memory bandwidth and q* recomputed from them."""
import ctypes as C

import pytest

from expert_offload_fp4_b200 import _lib
from expert_offload_fp4_b200.api import BandwidthEstimate, qstar_split


def test_init_rejects_bad_arguments():
    L = _lib.load()
    est = _lib.BwEstimate()
    for alpha, bp, bh in [(0.0, 0, 0), (1.5, 0, 0), (0.5, -1.0, 0), (0.5, 0, float("inf"))]:
        assert L.moe_bw_init(C.byref(est), alpha, bp, bh) == _lib.MOE_EINVAL
    assert L.moe_bw_init(None, 0.5, 0, 0) == _lib.MOE_EINVAL


def test_first_observation_sets_then_moving_average():
    b = BandwidthEstimate(alpha=0.25)
    b.observe("pcie", 10e9, 0.2)                    # 50 GB/s
    assert b.b_pcie == pytest.approx(50.0, rel=1e-12)
    b.observe("pcie", 6e9, 0.1)                     # 60 GB/s observed
    assert b.b_pcie == pytest.approx(0.75 * 50.0 + 0.25 * 60.0, rel=1e-12)
    assert b.est.n_pcie == 2 and b.est.n_host == 0


def test_qstar_needs_both_links_then_matches_qstar_split():
    b = BandwidthEstimate(alpha=0.5)
    b.observe("pcie", 49.0e9, 1.0)
    with pytest.raises(_lib.MoeError):
        b.qstar(8)
    b.observe("host", 53.8e9, 1.0)
    # the first machine of the pages' table: 49.0 / 53.8 -> 91.1 %
    qg, qc, r = b.qstar(8)
    assert round(100 * r, 1) == 91.1
    assert (qg, qc, r) == qstar_split(8, b.b_pcie, b.b_host)


def test_estimate_tracks_a_bandwidth_change():
    b = BandwidthEstimate(alpha=0.5, b_pcie=52.7, b_host=77.3)
    assert b.qstar(10)[0] == 7                      # 68.2 % of 10 misses
    for _ in range(20):                             # the link drops to 25.1 GB/s, host to 63.2
        b.observe("pcie", 25.1e9, 1.0)
        b.observe("host", 63.2e9, 1.0)
    qg, qc, r = b.qstar(10)
    assert round(100 * r, 1) == 39.7 and (qg, qc) == (4, 6)


def test_observe_rejects_bad_arguments():
    L = _lib.load()
    b = BandwidthEstimate()
    assert L.moe_bw_observe(C.byref(b.est), 2, 1e9, 1.0) == _lib.MOE_EINVAL
    assert L.moe_bw_observe(C.byref(b.est), _lib.MOE_BW_PCIE, 0.0, 1.0) == _lib.MOE_EINVAL
    assert L.moe_bw_observe(C.byref(b.est), _lib.MOE_BW_HOST, 1e9, 0.0) == _lib.MOE_EINVAL
