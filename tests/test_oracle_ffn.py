"""Pins of the oracle's expert FFN, decode MoE layer and prefill token path.

* Structured experts (diagonal gate/up, permutation down, several block scales and
  tensor scales) give closed-form outputs: y_r = c_r * silu(a x_i + b x_j) * (u x_i).
  A swapped gate/up, a transposed down projection, a wrong nibble order or a
  wrong scale index changes them.
* The sparse top-k layer must equal a dense brute force over all experts.
* The prefill path equals the closed form on inputs that NVFP4 represents exactly.
"""
import math

import numpy as np
import pytest

from synthetic import gen, workloads as W

E2M1 = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def code_of(v):
    return E2M1[abs(v)] | (8 if v < 0 else 0)


def pack(codes):
    codes = np.asarray(codes, np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def silu(g):
    return g / (1.0 + math.exp(-g))


def structured_expert(fmt, H, I):
    """gate: g_i = x_i + 0.5*s1*x_{H/2+i}; up: u_i = 2 x_i (times tensor scales);
    down: y_r = h_{p(r)} (r < H/2), y_r = -0.5*s2*h_{q(r-H/2)} (r >= H/2)."""
    bs = 32 if fmt == "mxfp4" else 16
    half = H // 2
    assert I == half
    gc = np.zeros((I, H), np.uint8)
    uc = np.zeros((I, H), np.uint8)
    for i in range(I):
        gc[i, i] = code_of(1.0)
        gc[i, half + i] = code_of(0.5)
        uc[i, i] = code_of(2.0)
    p = [(3 * r + 1) % I for r in range(half)]
    q = [(5 * r + 7) % I for r in range(half)]
    dc = np.zeros((H, I), np.uint8)
    for r in range(half):
        dc[r, p[r]] = code_of(1.0)
        dc[half + r, q[r]] = code_of(-0.5)
    if fmt == "mxfp4":
        one, two, halfs = 127, 128, 126            # E8M0 bytes for 1, 2, 0.5
        ts = (1.0, 1.0, 1.0)
    else:
        one, two, halfs = 0x38, 0x40, 0x30         # E4M3 bytes for 1, 2, 0.5
        ts = (0.5, 0.25, 2.0)
    gs = np.full((I, H // bs), one, np.uint8)
    gs[:, (half // bs):] = two                     # s1 = 2 on the second half of K
    us = np.full((I, H // bs), one, np.uint8)
    ds = np.full((H, I // bs), one, np.uint8)
    ds[half:, :] = halfs                           # s2 = 0.5 on the lower half of rows
    tensors = {"gate": (pack(gc), gs, ts[0]), "up": (pack(uc), us, ts[1]),
               "down": (pack(dc), ds, ts[2])}

    def expected(x):
        g = [ts[0] * (x[i] + 0.5 * 2.0 * x[half + i]) for i in range(I)]
        u = [ts[1] * 2.0 * x[i] for i in range(I)]
        h = [silu(g[i]) * u[i] for i in range(I)]
        y = [ts[2] * h[p[r]] for r in range(half)] + \
            [ts[2] * -0.5 * 0.5 * h[q[r]] for r in range(half)]
        return np.array(y), np.array(h)
    return tensors, expected


@pytest.mark.parametrize("fmt,H", [("mxfp4", 64), ("mxfp4", 128), ("nvfp4", 32), ("nvfp4", 64)])
def test_structured_expert_closed_form(orc, fmt, H):
    tensors, expected = structured_expert(fmt, H, H // 2)
    rng = np.random.default_rng(H)
    x = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(rng.standard_normal(H).astype(np.float32)))
    y = orc.expert_ffn(fmt, H, H // 2, tensors, x)
    ref, _ = expected([float(v) for v in x])
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_decode_layer_combines_by_routing_weight(orc):
    H, I, E = 64, 32, 4
    experts = {}
    expect = {}
    for e in range(E):
        t, f = structured_expert("mxfp4", H, I)
        # expert e: scale every down block by 2^e via the E8M0 byte
        c, s, ts = t["down"]
        t["down"] = (c, (s.astype(np.int32) + e).astype(np.uint8), ts)
        experts[e] = t
        expect[e] = (lambda f, e: (lambda x: f(x)[0] * 2.0 ** e))(f, e)
    rng = np.random.default_rng(5)
    x = gen.f32_to_bf16_bits(rng.standard_normal((3, H)).astype(np.float32))
    idx = np.array([[2, 0], [1, 3], [3, 2]], np.int32)
    w = np.array([[0.7, 0.3], [0.55, 0.45], [0.9, 0.1]], np.float32)
    yf, yb = orc.moe_decode("mxfp4", H, I, E, x, idx, w, experts)
    xf = gen.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(3):
        ref = sum(float(w[t, j]) * expect[idx[t, j]](list(xf[t])) for j in range(2))
        np.testing.assert_allclose(yf[t], ref.astype(np.float32), rtol=1e-6, atol=1e-7)
        assert np.array_equal(yb[t], gen.f32_to_bf16_bits(yf[t]))


def test_sparse_equals_dense_brute_force_tiny(orc):
    w = W.TINY
    x = gen.activations(w, 0, 0, 4)
    wr = gen.router_weight(w, 0)
    b = gen.router_bias(w, 0)
    experts = {e: gen.expert_weights(w, 0, e) for e in range(w.E)}
    idx, wt, _ = orc.route(x, wr, b, w.k, 1)
    yf, _ = orc.moe_decode(w.fmt, w.H, w.I, w.E, x, idx, wt, experts)
    yd, mask = orc.moe_dense(w.fmt, w.H, w.I, w.E, w.k, 1, x, wr, b, experts)
    for t in range(4):
        assert sorted(np.nonzero(mask[t])[0].tolist()) == sorted(idx[t].tolist())
    rms = np.sqrt(np.mean(yd ** 2))
    assert rms > 0
    assert np.max(np.abs(yf - yd)) <= 1e-6 * rms
    # unnormalised variant: weights are the full softmax at the chosen experts
    idx0, wt0, _ = orc.route(x, wr, b, w.k, 0)
    yf0, _ = orc.moe_decode(w.fmt, w.H, w.I, w.E, x, idx0, wt0, experts)
    yd0, _ = orc.moe_dense(w.fmt, w.H, w.I, w.E, w.k, 0, x, wr, b, experts)
    assert np.max(np.abs(yf0 - yd0)) <= 1e-6 * rms


def test_prefill_token_closed_form_on_nvfp4_exact_inputs(orc):
    H, I = 64, 32
    t, f = structured_expert("nvfp4", H, I)
    rng = np.random.default_rng(11)
    # grid step 7/16 makes the token scale amax/2688 = 2^-10 and every block scale 448
    grid = np.array([0.5, 1, 1.5, 2, 3, 4, 6], np.float32) * np.float32(0.4375)
    x = rng.choice(grid, H) * rng.choice([-1, 1], H).astype(np.float32)
    x[::16] = 2.625                     # every 16-block holds the row amax (6 * 7/16)
    xb = gen.f32_to_bf16_bits(x)
    assert np.array_equal(gen.bf16_bits_to_f32(xb), x)
    yf, yb = orc.moe_prefill_token(H, I, 1, xb, np.array([0], np.int32),
                                   np.array([1.0], np.float32), {0: t})
    _, h = f([float(v) for v in x])
    hc, hs = orc.nvfp4_quantize_row(h.astype(np.float32), np.float32(1.0))
    hq = orc.dequant("nvfp4", hc[None], hs[None], 1.0)[0].astype(np.float64)
    half = H // 2
    p = [(3 * r + 1) % I for r in range(half)]
    q = [(5 * r + 7) % I for r in range(half)]
    ref = np.array([2.0 * hq[p[r]] for r in range(half)] + [2.0 * -0.25 * hq[q[r]] for r in range(half)])
    np.testing.assert_allclose(yf, ref.astype(np.float32), rtol=1e-6, atol=1e-9)
    # and h quantisation stays within NVFP4 error of the unquantised result
    ref_d, _ = f([float(v) for v in x])
    assert np.max(np.abs(yf - ref_d)) <= 0.25 * np.max(np.abs(ref_d))


def test_prefill_close_to_decode_on_real_shapes(orc):
    w = W.TINY
    x = gen.activations(w, 0, 0, 2)
    # prefill needs NVFP4 experts: take the decode-35B recipe on the tiny shape
    wn = W.Workload(name="t", H=256, I=256, E=16, k=2, L=1, fmt=W.NVFP4, seed=7, batches=(2,),
                    steps=1, zipf_s=0.0, weight_recipe="normal")
    experts = {e: gen.expert_weights(wn, 0, e) for e in (3, 9)}
    idx = np.array([3, 9], np.int32)
    wt = np.array([0.6, 0.4], np.float32)
    yp, _ = orc.moe_prefill_token(256, 256, 16, x[0], idx, wt, experts)
    yd, _ = orc.moe_decode("nvfp4", 256, 256, 16, x[:1], idx[None], wt[None], experts)
    rms = np.sqrt(np.mean(yd.astype(np.float64) ** 2))
    assert np.sqrt(np.mean((yp - yd[0]).astype(np.float64) ** 2)) < 0.2 * rms


@pytest.mark.parametrize("k", [-20, -6, 0, 7, 12, 30])
def test_prefill_x_quantisation_is_exact_on_grid_at_any_scale(orc, k):
    """A token whose every 16-block holds its amax and whose values sit on the E2M1
    grid is represented exactly, whatever its magnitude: the per-token FP32 scale
    absorbs 2^k and the block scales stay at 448."""
    rng = np.random.default_rng(k + 100)
    grid = np.array([0.5, 1, 1.5, 2, 3, 4, 6], np.float32) * np.float32(0.4375)
    x = rng.choice(grid, 256) * rng.choice([-1, 1], 256).astype(np.float32)
    x[::16] = -2.625
    x = np.ldexp(x, k).astype(np.float32)
    xb = gen.f32_to_bf16_bits(x)
    c, s, S = orc.prefill_quantize_x(xb)
    assert S == np.float32(2.0 ** (k - 10))
    assert np.all(s == 0x7E)                             # 448 in every block
    assert np.array_equal(orc.dequant("nvfp4", c[None], s[None], S)[0], x)


def test_batched_prefill_equals_per_token_oracle(orc):
    """oracle.prefill_batch (float64 matrix products over every token of an
    expert) against or_moe_prefill_token (plain per-token loops) on uneven groups:
    both take the same steps, only the order of the float64 additions inside a
    dot product differs, so they agree to float64 rounding.  A transposed weight,
    a wrong rank order or a dropped routing weight moves the output by O(rms)."""
    from oracle import prefill_batch
    w = W.Workload(name="pb", H=256, I=256, E=8, k=3, L=1, fmt=W.NVFP4, seed=31, batches=(40,),
                   steps=1, zipf_s=0.9, weight_recipe="normal")
    T = 40
    x = gen.activations(w, 0, 0, T)
    idx, wt, _ = orc.route(x, gen.router_weight(w, 0), gen.router_bias(w, 0), w.k, 1)
    experts = {e: gen.expert_weights(w, 0, e) for e in range(w.E)}
    yb = prefill_batch.moe_prefill(w.H, w.I, w.E, x, idx, wt, experts)
    counts = np.bincount(idx.ravel(), minlength=w.E)
    assert counts.min() != counts.max()            # the groups really are uneven
    for t in range(T):
        yt, _ = orc.moe_prefill_token(w.H, w.I, w.E, x[t], idx[t], wt[t], experts)
        rms = float(np.sqrt(np.mean(yt.astype(np.float64) ** 2)))
        assert float(np.max(np.abs(yb[t] - yt))) <= 1e-5 * rms, t
