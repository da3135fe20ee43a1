"""Pins of the oracle's FP4 / scale codecs and its NVFP4 quantiser.

The E2M1 table comes from the OCP MX v1.0 spec (golden file); E4M3 is checked
against torch's float8_e4m3fn decoding and E8M0 against math.ldexp; the
quantisers against round-to-nearest-even facts and against the generator's
independent (vectorised, table-search) NVFP4 weight quantiser.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from synthetic import gen


def test_e2m1_matches_ocp_table(orc):
    rows = read_golden("e2m1_ocp_table.txt")
    assert len(rows) == 16
    for code, val in rows:
        v = orc.e2m1_value(int(code))
        assert v == float(val)
        assert math.copysign(1.0, v) == math.copysign(1.0, float(val))  # -0 for code 8


def test_e2m1_round_trip_all_codes(orc):
    for c in range(16):
        assert orc.e2m1_quantize(orc.e2m1_value(c)) == c


@pytest.mark.parametrize("v,code", [
    (0.25, 0), (0.2499, 0), (0.2501, 1), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4),
    (3.5, 6), (5.0, 6), (5.0001, 7), (6.0, 7), (7.0, 7), (1e9, 7), (-0.75, 10), (-5.0, 14),
    (-0.1, 8), (0.1, 0), (-100.0, 15)])
def test_e2m1_rne_ties_and_saturation(orc, v, code):
    # midpoints go to the even mantissa (codes 0, 2, 4, 6), beyond 6 saturates
    assert orc.e2m1_quantize(v) == code


def test_e8m0_all_bytes(orc):
    for b in range(255):
        assert orc.e8m0_value(b) == math.ldexp(1.0, b - 127)
    assert math.isnan(orc.e8m0_value(255))


def test_e4m3_all_bytes_match_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for b in range(256):
        v = orc.e4m3_value(b)
        if math.isnan(ref[b]):
            assert math.isnan(v)
        else:
            assert v == ref[b], b
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_quantize_matches_torch_in_range(orc):
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.uniform(0, 448, 2000), np.exp(rng.uniform(-12, 6, 2000)),
                           [2.0 ** -10, 1.5 * 2.0 ** -10, 0.0, 448.0, 440.0, 447.9]])
    vals = vals.astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals, ref):
        assert orc.e4m3_quantize(float(v)) == int(r), float(v)
    assert orc.e4m3_quantize(1e6) == 0x7E  # saturates to 448


def test_nvfp4_quantiser_matches_generator(orc):
    """The oracle's per-row quantiser and the generator's vectorised one are separate
    codes of the same recipe; they must agree bit for bit."""
    key = gen.stream_key(99, 4, 0, 0)
    codes, scales, S = gen._normal_nvfp4(key, 24, 256, 0.02)
    w = (gen.normals(key, 24 * 256) * 0.02).astype(np.float32).reshape(24, 256)
    for r in range(24):
        c, s = orc.nvfp4_quantize_row(w[r], np.float32(S))
        assert np.array_equal(s, scales[r])
        assert np.array_equal(c, codes[r])


def test_nvfp4_quantiser_error_bound(orc):
    rng = np.random.default_rng(1)
    v = rng.standard_normal(4096).astype(np.float32) * 3
    S = orc.token_scale(v)
    assert S == np.float32(np.float32(np.abs(v).max()) / np.float32(2688.0))
    c, s = orc.nvfp4_quantize_row(v, S)
    deq = orc.dequant("nvfp4", c[None, :], s[None, :], S)[0]
    for b in range(4096 // 16):
        blk = v[b * 16:(b + 1) * 16]
        q = orc.e4m3_value(int(s[b])) * float(S)
        # largest gap of the E2M1 grid is 2 (between 4 and 6): error <= q, and the
        # block amax lands within a scale-rounding step of 6*q
        assert np.max(np.abs(blk - deq[b * 16:(b + 1) * 16])) <= q * 1.0000001
        amax = float(np.abs(blk).max())
        assert abs(amax - 6 * q) <= 6 * q * 2 ** -3 + 1e-30
    # the token's amax element maps to +-6 times a scale of at most 448*S
    i = int(np.argmax(np.abs(v)))
    code = (c[i // 2] >> (4 * (i % 2))) & 15
    assert code & 7 in (6, 7)


def test_dequant_mxfp4_and_nvfp4(orc):
    rows = read_golden("e2m1_ocp_table.txt")
    e2m1 = np.array([float(v) for _, v in rows], np.float32)
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 256, (8, 32), dtype=np.uint8)      # 8 rows x 64 elements
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(8, 64)
    sc_mx = rng.integers(120, 135, (8, 2), dtype=np.uint8)
    got = orc.dequant("mxfp4", codes, sc_mx, 1.0)
    exp = e2m1[nib] * np.ldexp(np.float32(1), sc_mx.astype(np.int32) - 127).repeat(32, 1)
    assert np.array_equal(got, exp.astype(np.float32))
    sc_nv = rng.integers(0x30, 0x60, (8, 4), dtype=np.uint8)
    ts = np.float32(3.7e-5)
    got = orc.dequant("nvfp4", codes, sc_nv, ts)
    s_val = torch.from_numpy(sc_nv).view(torch.float8_e4m3fn).float().numpy().repeat(16, 1)
    exp = ((e2m1[nib] * s_val).astype(np.float32) * ts).astype(np.float32)
    assert np.array_equal(got, exp)
