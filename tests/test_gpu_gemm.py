"""The tcgen05 GEMM kernel alone (C = A B^T, bf16 in/out, fp32 accumulate) against an fp64 matmul
of the same bf16 inputs, on shapes that exercise partial M tiles, both column-tile widths, long K and the
CTA-pair kernel (large shapes)."""
import numpy as np
import pytest
import torch

from latent_mixture_experts_gemm_b200 import lmoe
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(128, 64, 64), (1, 64, 64), (37, 512, 128), (200, 192, 320), (1000, 256, 1024),
                                   (4096, 1024, 512), (8192, 4096, 1024), (300, 64, 4096),
                                   # CTA-pair tiles (256 x 256): a ragged last pair (the second CTA gets 104 rows),
                                   # and a ragged last column tile (the second CTA's B rows are all past N)
                                   (1000, 8192, 256), (2500, 2368, 320)])
def test_gemm_matches_fp64(M, N, K):
    g = torch.Generator().manual_seed(M * 31 + N * 7 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lmoe.lmoe_gemm_bf16(A.cuda(), B.cuda(), C, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = A.double() @ B.double().T
    got = C.cpu().double()
    # fp32 accumulation, one bf16 rounding of the output
    assert torch.all(torch.abs(got - ref) <= 2.0 ** -8 * torch.abs(ref) + 1e-3 * ref.std() + 1e-6)
    # one bf16 rounding of outputs up to |ref| ~ 8 is up to 2^-5 / 2 absolute: the max error scales with
    # the largest |ref|, so it is bounded elementwise above; the mean relative error stays small
    P.assert_close(got.numpy(), ref.numpy(), "C", max_vs_rms=2e-2, mean_rel=3e-3)
