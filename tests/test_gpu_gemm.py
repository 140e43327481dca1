"""gdn_gemm_bf16 (tcgen05 + TMA, through the C ABI) against the fp64 product of the
same bf16 values.  Bound per element: |C - C_ref| <= 2^-8 |C_ref| + 2^-16 max|C_ref|
(one bf16 rounding of an fp32 accumulation)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import gdn
from gpu_helpers import err_word

pytestmark = pytest.mark.gpu


def gemm_error(c, ref):
    c = c.double().cpu().numpy()
    bound = 2.0**-8 * np.abs(ref) + 2.0**-16 * np.abs(ref).max()
    return float(np.max(np.abs(c - ref) - bound))


def rand_bf16(*shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 300, 128), (1, 16, 64), (513, 1000, 640),
                                   (4096, 512, 64)])
def test_gemm_matches_fp64(M, N, K):
    a, b = rand_bf16(M, K, seed=M + K), rand_bf16(N, K, seed=N + 7)
    err = err_word()
    ldc = (N + 7) // 8 * 8  # leading dimensions are 16-byte multiples
    c = torch.empty(M, ldc, dtype=torch.bfloat16, device="cuda")[:, :N]
    gdn.gemm_bf16(a.cuda(), b.cuda(), out=c, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    e = gemm_error(c, oracle.gemm(a, b))
    print(f"[parity] gemm {M}x{N}x{K}: excess over bound {e:.3e}")
    assert e <= 0


def test_gemm_strided_views_and_untouched_padding():
    """Row-strided operands (a column slice of a wider buffer) and an output written into
    the middle of a wider buffer: only the first N columns of each output row change."""
    M, N, K = 300, 264, 192
    big_a = rand_bf16(M, K + 64, seed=1).cuda()
    big_b = rand_bf16(N, K + 128, seed=2).cuda()
    out = torch.full((M, N + 40), 3.0, dtype=torch.bfloat16, device="cuda")
    a, b = big_a[:, 64:64 + K], big_b[:, :K]
    gdn.gemm_bf16(a, b, out=out[:, :N])
    torch.cuda.synchronize()
    assert gemm_error(out[:, :N], oracle.gemm(a.cpu(), b.cpu())) <= 0
    assert torch.all(out[:, N:] == 3.0)


@pytest.mark.parametrize("N,K", [(16480, 5120), (5120, 6144)])
def test_gemm_projection_shapes_sampled_rows(N, K):
    """The layer's two projection shapes at T = 4096 tokens, checked on 48 sampled rows."""
    M = 4096
    a = rand_bf16(M, K, seed=K, scale=0.5).cuda()
    b = rand_bf16(N, K, seed=N, scale=K ** -0.5).cuda()
    err = err_word()
    c = gdn.gemm_bf16(a, b, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = torch.randperm(M, generator=torch.Generator().manual_seed(9))[:48]
    e = gemm_error(c[rows], oracle.gemm(a[rows].cpu(), b.cpu()))
    print(f"[parity] gemm {M}x{N}x{K} (48 rows): excess over bound {e:.3e}")
    assert e <= 0


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(16480, 5120), (5120, 6144), (1001, 640)])
def test_few_rows_stream_the_weights(M, N, K):
    """M <= 4 rows (a decode step) go through the weight-streaming kernel: the whole product
    against fp64, with A a strided view (a row of the layer's input) and C's padding columns
    untouched."""
    a_full = rand_bf16(M, K + 64, seed=M * 31 + K)
    a = a_full[:, 32:32 + K]
    b = rand_bf16(N, K, seed=N + M, scale=K ** -0.5)
    err = err_word()
    ldc = (N + 7) // 8 * 8 + 8
    c_full = torch.full((M, ldc), 3.0, dtype=torch.bfloat16, device="cuda")
    c = c_full[:, :N]
    gdn.gemm_bf16(a_full.cuda()[:, 32:32 + K], b.cuda(), out=c, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    e = gemm_error(c, oracle.gemm(a, b))
    print(f"[parity] gemv {M}x{N}x{K}: excess over bound {e:.3e}")
    assert e <= 0
    assert torch.all(c_full[:, N:] == 3.0)
