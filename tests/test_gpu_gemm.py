"""The tcgen05 block-scaled NVFP4 GEMM against the oracle's dequantised operands.

D = dq(A) dq(B)^T: the oracle dequantises A and B (codes and E4M3 block
scales, canonical layout) and a float64 matmul gives the reference.  Products
of E2M1 x E4M3-scaled values are exact; the tensor core accumulates in fp32.
"""
import numpy as np
import pytest
import torch

import oracle
from synthetic import gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    from expert_offload_fp4_b200 import build
    build.build()
    import expert_offload_fp4_b200 as mod
    return mod


def operand(seed, rows, K, lo=0x28, hi=0x48):
    k = gen.stream_key(seed, 77, rows, K)
    codes = gen.uint64s(k, rows * K // 16).view(np.uint8)[: rows * K // 2].reshape(rows, K // 2).copy()
    sc = (gen.uint64s(gen.stream_key(seed, 78, rows, K), rows * K // 16) % np.uint64(hi - lo) + np.uint64(lo))
    return codes, sc.astype(np.uint8).reshape(rows, K // 16)


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 512), (128, 256, 2048)])
def test_nvfp4_gemm_matches_dequantised_product(m, M, N, K):
    ac, asc = operand(1, M, K)
    bc, bsc = operand(2, N, K)
    A = oracle.dequant("nvfp4", ac, asc, 1.0).astype(np.float64)
    B = oracle.dequant("nvfp4", bc, bsc, 1.0).astype(np.float64)
    ref = A @ B.T
    D = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    m.nvfp4_gemm(dev(ac), dev(asc), dev(bc), dev(bsc), D, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = D.cpu().numpy().astype(np.float64)
    scale = np.sqrt(np.mean(ref ** 2))
    err = np.max(np.abs(got - ref))
    assert err <= 1e-4 * scale + 1e-6 * np.max(np.abs(ref)), (err, scale)


def test_nvfp4_gemm_rejects_bad_shapes(m):
    t = torch.zeros(64, dtype=torch.uint8, device="cuda")
    D = torch.zeros(1, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(m._lib.MoeError):
        m._lib.check("moe_nvfp4_gemm", m._lib.load().moe_nvfp4_gemm(
            t.data_ptr(), t.data_ptr(), t.data_ptr(), t.data_ptr(), 100, 128, 256, D.data_ptr(),
            st.data_ptr(), None))
