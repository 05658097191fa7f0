"""The Blackwell tensor-core path (tcgen05.mma from swizzled K-major or MN-major
shared tiles into tensor memory) against a plain PyTorch fp32 product."""
from __future__ import annotations

import ctypes

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn

pytestmark = pytest.mark.gpu


def _run(A, Bm, N, K, bf16, a_mn, b_mn):
    C = torch.full((128, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = gdn.lib().gdn_selftest_umma(p(A), p(Bm), p(C), N, K, int(bf16), int(a_mn), int(b_mn), p(status),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "completion wait gave up"
    return C


@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("N", [32, 64, 128, 256])
@pytest.mark.parametrize("K", [64, 128])
def test_umma_gemm_matches_fp32_product(dtype, N, K, a_mn, b_mn):
    g = torch.Generator().manual_seed(N * 1000 + K)
    A = torch.randn(128, K, generator=g).to(dtype)      # A(m, k)
    Bm = torch.randn(N, K, generator=g).to(dtype)       # B(n, k)
    ref = A.float() @ Bm.float().T
    Ad = (A.T.contiguous() if a_mn else A).cuda()
    Bd = (Bm.T.contiguous() if b_mn else Bm).cuda()
    C = _run(Ad, Bd, N, K, dtype == torch.bfloat16, a_mn, b_mn).cpu()
    err = (C - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item(), f"max abs error {err}"
