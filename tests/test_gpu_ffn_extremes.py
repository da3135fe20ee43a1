"""The decode FFN's arithmetic at the edges of the formats, against the oracle.

Experts are built by hand in the canonical layout (E2M1 codes two per byte, the
lower element in the low nibble; E4M3 or E8M0 block scales):
* NVFP4, every code +6 and every scale the largest E4M3 value (448), with large
  positive activations: products and sums at their largest.
* NVFP4, runs of 16 codes of +6 or -6 with random signs, scales from the
  smallest subnormal E4M3 to 448, large activations of both signs with zeros.
* MXFP4, E8M0 exponents spread over 40 binades inside each 128-element segment
  (the kernel scales a block relative to the largest exponent of its segment in
  f16, so blocks far below it are flushed: their share is below 2^-24 of the
  segment's).
The kernel's fp32 rank-ordered sum (before bf16 rounding) must stay within
ERR_FP32 * rms of the oracle's float64 result; the tensor scales keep gate, up and
h in a moderate range so silu and the products stay finite on both sides.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import gen

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


def pack(codes4):
    """[rows, K] 4-bit codes -> [rows, K/2] bytes, the lower element in the low nibble."""
    c = codes4.astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def run_case(m, fmt, H, I, experts, x_f32):
    E, k, T = len(experts), 2, x_f32.shape[0]
    pool = m.Pool(H, I, E, k, 1, fmt, E, max_tokens=T, host_layers=1)
    for e, t in experts.items():
        pool.load_expert(0, e, t)
    idx = np.array([[e % E, (e + 1) % E] for e in range(T)], np.int32)
    w = np.array([[0.625, 0.375]] * T, np.float32)
    x_bits = gen.f32_to_bf16_bits(x_f32.astype(np.float32))
    idx_d, w_d = dev(idx), dev(w)
    slot_of = torch.empty_like(idx_d)
    res = m.slot_lookup(pool, 0, idx_d, slot_of)
    cs = torch.cuda.Stream()
    m.stream_misses(pool, 0, res, cs)
    cs.synchronize()
    xd = dev(x_bits.view(np.int16)).view(torch.bfloat16)
    y_part = torch.empty((T, k, H), dtype=torch.float32, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.expert_ffn(pool, 0, xd, idx_d, w_d, slot_of, y_part, status, y=y)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    yp = y_part.cpu().numpy()
    ys = np.zeros((T, H), np.float32)
    for j in range(k):
        ys = (ys + yp[:, j]).astype(np.float32)
    yf, _ = oracle.moe_decode(fmt, H, I, E, x_bits, idx, w, experts)
    assert np.all(np.isfinite(yf)) and np.all(np.isfinite(ys))
    rms = float(np.sqrt(np.mean(yf.astype(np.float64) ** 2)))
    assert rms > 0
    err = float(np.max(np.abs(ys.astype(np.float64) - yf)))
    pool.close()
    return err / rms


def test_nvfp4_largest_codes_and_scales(m):
    H, I, E = 2048, 768, 4
    rng = np.random.default_rng(11)
    x = np.abs(rng.standard_normal((2, H))) * 1e3 + 1.0
    sx = float(np.sum(x, axis=1).max())
    experts = {}
    for e in range(E):
        t = {}
        for name, rows, K, ts in (("gate", I, H, 8.0 / (2688 * sx)), ("up", I, H, 8.0 / (2688 * sx)),
                                  ("down", H, I, 1.0 / (2688 * I * 64.0))):
            t[name] = (pack(np.full((rows, K), 0x7, np.uint8)), np.full((rows, K // 16), 0x7E, np.uint8),
                       np.float32(ts * (1 + 0.1 * e)))
        experts[e] = t
    rel = run_case(m, "nvfp4", H, I, experts, x)
    print(f"largest codes and scales: fp32 error / rms = {rel:.2e}")
    assert rel <= ERR_FP32, rel


def test_nvfp4_sign_runs_and_scale_range(m):
    H, I, E = 2048, 768, 4
    rng = np.random.default_rng(12)
    x = rng.standard_normal((2, H)) * 3e4
    x[:, rng.random(H) < 0.1] = 0.0
    experts = {}
    e4m3 = np.concatenate([np.arange(1, 8), np.arange(8, 0x7F, 5), [0x7E]]).astype(np.uint8)
    for e in range(E):
        t = {}
        for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
            signs = rng.random((rows, K // 16)) < 0.5
            codes = np.where(np.repeat(signs, 16, axis=1), 0xF, 0x7).astype(np.uint8)
            scales = rng.choice(e4m3, size=(rows, K // 16))
            ts = 2e-7 if name != "down" else 1e-4
            t[name] = (pack(codes), scales, np.float32(ts))
        experts[e] = t
    rel = run_case(m, "nvfp4", H, I, experts, x)
    print(f"sign runs and scale range: fp32 error / rms = {rel:.2e}")
    assert rel <= ERR_FP32, rel


def test_mxfp4_exponent_spread_in_segments(m):
    H, I, E = 1024, 768, 4
    rng = np.random.default_rng(13)
    x = rng.standard_normal((2, H)) * 10.0
    experts = {}
    for e in range(E):
        t = {}
        for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
            codes = rng.integers(0, 16, size=(rows, K), dtype=np.uint8)
            # per 32-element block: the segment's first block near 2^-6, the others
            # anywhere down to 40 binades below it
            base = 127 - 6 if name != "down" else 127 - 8
            ex = base - rng.integers(0, 41, size=(rows, K // 32))
            ex[:, 0::4] = base
            t[name] = (pack(codes), ex.astype(np.uint8), np.float32(1.0))
        experts[e] = t
    rel = run_case(m, "mxfp4", H, I, experts, x)
    print(f"exponent spread: fp32 error / rms = {rel:.2e}")
    assert rel <= ERR_FP32, rel
