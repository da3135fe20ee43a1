"""Arithmetic of the decode expert FFN, separated from the output's bf16 rounding.

The kernel's fp32 result (y_part summed over the ranks in rank order, before any
rounding to bf16) is compared with the oracle's float64-accumulated layer
rounded once to fp32: products of FP4 weights and activations are exact on
both sides and the kernel sums in fp32, so the two agree far inside the 2e-2
output tolerance; the bound below (ERR_FP32) is what fp32 accumulation with h
carried to ~22 bits allows.  The fused combine must give the same bf16 bits as
the standalone one (moe_combine) and as rounding that fp32 sum.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import gen, workloads as W

pytestmark = pytest.mark.gpu
ERR_FP32 = 1e-4


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


CASES = [("tiny", W.TINY, 4), ("35b_t1", W.DECODE_35B, 1), ("35b_t8", W.DECODE_35B, 8),
         ("284b_t1", W.DECODE_284B, 1)]


@pytest.mark.parametrize("name,w,T", CASES, ids=[c[0] for c in CASES])
def test_fp32_sum_before_rounding(m, name, w, T):
    L = 2
    pool = m.Pool(w.H, w.I, w.E, w.k, L, w.fmt, min(w.E * L, 64), max_tokens=T, host_layers=L)
    lo = m.DecodeLayer(pool, T)
    y_alt = torch.empty((T, w.H), dtype=torch.bfloat16, device="cuda")
    worst = 0.0
    for step in range(2):
        for layer in range(L):
            x = gen.activations(w, layer, step, T)
            wr = gen.router_weight(w, layer)
            b = gen.router_bias(w, layer)
            idx_r, w_r, _ = oracle.route(x, wr, b, w.k, 1)
            experts = {e: gen.expert_weights(w, layer, e) for e in sorted(set(idx_r.ravel().tolist()))}
            xd = bf16(x)
            m.route(xd, bf16(wr), dev(b), w.k, 1, lo.idx, lo.w, lo.ws)
            m.slot_lookup(pool, layer, lo.idx, lo.slot_of, lo.lookup)
            for e, _, _, _ in lo.lookup.miss_list():
                pool.load_expert(layer, e, experts[e])
            m.stream_misses(pool, layer, lo.lookup, lo.copy_stream)
            lo.status.zero_()
            m.expert_ffn(pool, layer, xd, lo.idx, lo.w, lo.slot_of, lo.y_part, lo.status, y=lo.y)
            m.combine(lo.y_part, y_alt)
            torch.cuda.synchronize()
            assert int(lo.status.item()) == 0
            assert np.array_equal(lo.idx.cpu().numpy(), idx_r)
            yp = lo.y_part.cpu().numpy()
            ys = np.zeros((T, w.H), np.float32)
            for j in range(w.k):                              # rank order, fp32
                ys = (ys + yp[:, j]).astype(np.float32)
            yf, _ = oracle.moe_decode(w.fmt, w.H, w.I, w.E, x, idx_r, w_r, experts)
            rms = float(np.sqrt(np.mean(yf.astype(np.float64) ** 2)))
            err = float(np.max(np.abs(ys.astype(np.float64) - yf)))
            assert err <= ERR_FP32 * rms, (step, layer, err / rms)
            worst = max(worst, err / rms)
            got = lo.y.view(torch.int16).cpu().numpy().view(np.uint16)
            assert np.array_equal(got, gen.f32_to_bf16_bits(ys))
            assert np.array_equal(got, y_alt.view(torch.int16).cpu().numpy().view(np.uint16))
    print(f"{name}: worst fp32 error / rms = {worst:.2e}")
    pool.close()


def test_repeated_calls_are_bit_identical(m):
    """The same call twice gives the same bits: fixed summation order everywhere."""
    w = W.DECODE_35B
    T = 8
    pool = m.Pool(w.H, w.I, w.E, w.k, 1, w.fmt, w.E, max_tokens=T, host_layers=1)
    for e in range(w.E):
        pool.load_expert(0, e, gen.expert_weights(w, 0, e))
    lo = m.DecodeLayer(pool, T)
    x = bf16(gen.activations(w, 0, 3, T))
    wr = bf16(gen.router_weight(w, 0))
    b = dev(gen.router_bias(w, 0))
    outs = []
    for _ in range(3):
        lo(0, x, wr, b)
        torch.cuda.synchronize()
        assert int(lo.status.item()) == 0
        outs.append((lo.y_part.cpu().numpy().copy(), lo.y.view(torch.int16).cpu().numpy().copy()))
    for yp, y in outs[1:]:
        assert np.array_equal(yp.view(np.uint32), outs[0][0].view(np.uint32))
        assert np.array_equal(y, outs[0][1])
    pool.close()
