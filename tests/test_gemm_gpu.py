"""The tcgen05 projection GEMM (axon_gemm_bf16) against a float64 product of
the same bf16 inputs on the CPU: ragged M, N and K (K not a multiple of the
64-deep stages), single and many tiles per block (the persistent schedule
wraps the two tensor-memory accumulators many times), the whole layer's
shapes, and row strides wider than the matrices.

Tolerance: the kernel accumulates in float32 and rounds the result to bf16
once, so each element is held to 1/128 of max(|ref|, rms(ref)) -- the bf16
rounding (2^-9 relative) with room for float32 accumulation over K terms.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _check(C, A, W, what):
    ref = A.double().cpu().numpy() @ W.double().cpu().numpy()
    got = C.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)), what
    scale = np.maximum(np.abs(ref), np.sqrt(np.mean(ref ** 2)) + 1e-30)
    err = np.abs(got - ref) / scale
    assert err.max() <= 1.0 / 128, f"{what}: worst {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}"


SHAPES = [(1, 8, 8), (200, 1536, 256), (200, 800, 768), (300, 520, 104), (48, 2560, 7680),
          (1000, 4096, 1024), (129, 264, 200), (4096, 15360, 64), (2048, 2560, 7680)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_matches_float64_product(cuda_lib, M, N, K):
    g = torch.Generator().manual_seed(M * 31 + N * 7 + K)
    A = (torch.randn(M, K, generator=g) / K ** 0.25).to(torch.bfloat16).cuda()
    W = (torch.randn(K, N, generator=g) / K ** 0.25).to(torch.bfloat16).cuda()
    C = cuda_lib.gemm_bf16(A, W)
    torch.cuda.synchronize()
    _check(C, A, W, f"M{M} N{N} K{K}")


def test_gemm_strided_rows_and_canaries(cuda_lib):
    """Row strides wider than the matrices (a column slice of a larger array);
    the columns outside the slice and the bytes around the output stay untouched."""
    M, N, K = 300, 264, 136
    g = torch.Generator().manual_seed(5)
    Abig = torch.randn(M, K + 24, generator=g).to(torch.bfloat16).cuda()
    Wbig = torch.randn(K, N + 40, generator=g).to(torch.bfloat16).cuda()
    A, W = Abig[:, 8:8 + K], Wbig[:, 16:16 + N]
    Cbig = torch.full((M + 2, N + 16), 7.0, dtype=torch.bfloat16, device="cuda")
    C = Cbig[1:1 + M, 8:8 + N]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # column slices are not contiguous tensors: pass their device addresses
    cuda_lib.axon_gemm_bf16(M, N, K, A.data_ptr(), A.stride(0), W.data_ptr(), W.stride(0), C.data_ptr(),
                            C.stride(0), err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check(C, A, W, "strided")
    keep = torch.ones_like(Cbig, dtype=torch.bool)
    keep[1:1 + M, 8:8 + N] = False
    assert torch.all(Cbig[keep] == 7.0)


def test_gemm_rejects_bad_arguments(cuda_lib):
    a = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")
    assert cuda_lib.axon_gemm_bf16(16, 12, 16, a, 16, a, 16, a.clone(), 16, raise_on_error=False) == 3   # N % 8
    assert cuda_lib.axon_gemm_bf16(16, 16, 0, a, 16, a, 16, a.clone(), 16, raise_on_error=False) == 1   # K == 0
    assert cuda_lib.axon_gemm_bf16(16, 16, 16, a, 16, a, 16, a, 16, raise_on_error=False) == 1          # C overlaps A
    assert cuda_lib.axon_gemm_bf16(0, 16, 16, None, 16, None, 16, None, 16, raise_on_error=False) == 0  # empty
