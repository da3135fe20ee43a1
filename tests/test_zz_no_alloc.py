"""The allocation-free router entry point (moe_route_noalloc) against moe_route
and against the oracle's router.

moe_route_noalloc exists for callers that cannot allocate device memory where
they route (all of HBM handed out at start-up, or no cudaMalloc allowed inside a
decode step); it keeps its scratch in a static device array of the library.
Two calls in a row must both match the workspace-taking entry point and the
oracle (indices bit for bit, weights to fp32 rounding): the second call checks
that what the first left in the shared array does no harm.  A warm call must
leave the device's free memory unchanged.
This file is collected last so that a failure here stops a run only after every
other test has run.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import gen, workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from expert_offload_fp4_b200 import build
    build.build()
    import expert_offload_fp4_b200 as mod
    return mod


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def test_route_noalloc_matches_route_on_two_calls_in_a_row(m):
    cases = [(W.DECODE_35B, 8, 1, 0), (W.DECODE_284B, 13, 0, 1)]
    for wl, T, renorm, step in cases:
        x = _dev_bf16(gen.activations(wl, 0, step, T))
        wr = _dev_bf16(gen.router_weight(wl, 0))
        b = torch.from_numpy(gen.router_bias(wl, 0)).cuda()
        idx_a = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
        w_a = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
        ws = torch.zeros(m.route_workspace_bytes(T, wl.E), dtype=torch.uint8, device="cuda")
        m.route(x, wr, b, wl.k, renorm, idx_a, w_a, ws)
        idx_r, w_r, _ = oracle.route(gen.activations(wl, 0, step, T), gen.router_weight(wl, 0),
                                     gen.router_bias(wl, 0), wl.k, renorm)
        for call in range(2):
            idx_b = torch.full((T, wl.k), -1, dtype=torch.int32, device="cuda")
            w_b = torch.full((T, wl.k), -1.0, dtype=torch.float32, device="cuda")
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info()[0]
            m.route_noalloc(x, wr, b, wl.k, renorm, idx_b, w_b)
            torch.cuda.synchronize()
            if call == 1:        # warm: the scratch address is known, nothing is allocated
                assert torch.cuda.mem_get_info()[0] == free0
            assert np.array_equal(idx_b.cpu().numpy(), idx_a.cpu().numpy())
            assert np.array_equal(idx_b.cpu().numpy(), idx_r)
            np.testing.assert_allclose(w_b.cpu().numpy(), w_a.cpu().numpy(), rtol=3e-6, atol=1e-7)
            np.testing.assert_allclose(w_b.cpu().numpy(), w_r, rtol=3e-6, atol=1e-7)


def test_route_noalloc_rejects_sizes_beyond_its_scratch(m):
    wl = W.DECODE_35B
    T = 65536 // wl.E + 1
    x = torch.zeros((T, wl.H), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((wl.E, wl.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    with pytest.raises(m._lib.MoeError) as e:
        m.route_noalloc(x, wr, None, wl.k, 1, idx, w)
    assert e.value.code == m._lib.MOE_EINVAL and "65536" in str(e.value)
