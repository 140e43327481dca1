"""tcgen05 operand layouts: D = A B^T on one CTA vs torch, for every
(layout, shape) combination the mixer kernels use."""
import ctypes

import pytest
import torch

from gpu_helpers import selftest_lib

pytestmark = pytest.mark.gpu

CASES = [
    # a_layout, b_layout, N, K   (0 = K-major SW128, 1 = MN-major SW128, 2 = MN-major SW64, 3 = A in TMEM)
    (0, 0, 64, 128),    # [Q;K] K^T
    (0, 0, 128, 128),
    (0, 0, 256, 64),
    (0, 1, 64, 64),     # [P;I] T~
    (0, 1, 128, 128),   # [Q;K] S^T, 128 state rows
    (0, 1, 64, 128),    # [Q;K] S^T, 64 state rows
    (0, 2, 32, 128),    # [Q;K] S^T, 32 state rows
    (0, 2, 32, 64),     # [P T~; T~] R, 32 state rows
    (0, 2, 64, 128),    # [Q;K] [S_hi | S_lo], 32 state rows (two SW64 blocks)
    (0, 2, 64, 64),     # [P T~; T~] [R_hi | R_lo], 32 state rows
    (1, 1, 128, 64),    # K^T U
    (1, 1, 64, 64),
    (1, 2, 32, 64),
    # A in tensor memory (3): state rows x operand, the TMEM-resident chain
    (3, 1, 64, 128),    # S [W^T] : W^T MN-major, one 64-wide block
    (3, 0, 64, 128),    # S Q^T   : Q K-major, two K blocks
    (3, 1, 128, 64),    # U_d K   : K MN-major, two 64-wide blocks
    (3, 0, 64, 64),     # U P^T   : P K-major
    (3, 0, 256, 64),
    (3, 1, 128, 128),
]


@pytest.mark.parametrize("a_layout,b_layout,N,K", CASES)
def test_umma_layouts(a_layout, b_layout, N, K):
    lib = selftest_lib()
    g = torch.Generator(device="cuda").manual_seed(7)
    A = torch.randn(128, K, generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn(N, K, generator=g, device="cuda").to(torch.bfloat16)
    D = torch.full((128, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.gdn_selftest_umma(a_layout, b_layout, N, K, ctypes.c_void_p(A.data_ptr()),
                               ctypes.c_void_p(B.data_ptr()), ctypes.c_void_p(D.data_ptr()),
                               ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = A.float() @ B.float().T
    assert torch.allclose(D, ref, rtol=1e-4, atol=1e-3), (D - ref).abs().max().item()
