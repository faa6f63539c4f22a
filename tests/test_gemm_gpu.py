"""The tcgen05 projection GEMM (axon_gemm_bf16) against a float64 product of
the same bf16 inputs on the CPU: ragged M, N and K (K not a multiple of the
64-deep stages), single and many tiles per block (the persistent schedule
wraps the two tensor-memory accumulators many times), the whole layer's
shapes, and row strides wider than the matrices -- on every tiling
(axon_gemm_bf16_plan): single-CTA tiles 256 and 192 wide, CTA pairs with
whole tiles, and CTA pairs with the stream-K split (one tile split over
fifteen pairs, ragged shapes, the layer's shapes; its partial sums are added
in a fixed order, so repeated calls agree bit for bit).

Tolerance: the kernel accumulates in float32 and rounds the result to bf16
once, so each element is held to 1/128 of max(|ref|, rms(ref)) -- the bf16
rounding (2^-9 relative) with room for float32 accumulation over K terms.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _check(C, A, W, what, ref=None):
    if ref is None:
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


# (9472, 512, 256): 74 pair tiles, as many as a B200 runs at once, so the
# stream-K plan leaves no split tail (every tile whole through the split path)
PLAN_SHAPES = [(1, 8, 8), (256, 256, 64), (256, 256, 7680), (300, 520, 104), (129, 264, 200), (1000, 4096, 1024),
               (4096, 15360, 64), (2048, 2560, 7680), (2048, 7712, 7680), (2048, 15360, 2560), (9472, 512, 256)]


@pytest.fixture(scope="module")
def gemm_ws(cuda_lib):
    return torch.empty(cuda_lib.axon_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")


_PLAN_CASES = {}


def _plan_case(M, N, K):
    """Seeded operands of one shape and their float64 product (computed once
    for all plans)."""
    if (M, N, K) not in _PLAN_CASES:
        g = torch.Generator().manual_seed(M * 131 + N * 17 + K)
        A = (torch.randn(M, K, generator=g) / K ** 0.25).to(torch.bfloat16)
        W = (torch.randn(K, N, generator=g) / K ** 0.25).to(torch.bfloat16)
        _PLAN_CASES.clear()
        _PLAN_CASES[(M, N, K)] = (A.cuda(), W.cuda(), A.double().numpy() @ W.double().numpy())
    return _PLAN_CASES[(M, N, K)]


@pytest.mark.parametrize("plan", [1, 2, 3, 4, 0])
@pytest.mark.parametrize("M,N,K", PLAN_SHAPES)
def test_gemm_plans_match_float64_product(cuda_lib, gemm_ws, M, N, K, plan):
    A, W, ref = _plan_case(M, N, K)
    C = cuda_lib.gemm_bf16(A, W, plan=plan, workspace=gemm_ws)
    torch.cuda.synchronize()
    _check(C, A, W, f"plan {plan} M{M} N{N} K{K}", ref=ref)
    if plan in (0, 4):
        C2 = cuda_lib.gemm_bf16(A, W, plan=plan, workspace=gemm_ws)
        torch.cuda.synchronize()
        assert torch.equal(C.view(torch.int16), C2.view(torch.int16)), "stream-K result differs between calls"


def test_gemm_stream_k_strided_rows_and_canaries(cuda_lib, gemm_ws):
    """The stream-K pairs on row-strided operands and output: the columns
    outside the slice and the bytes around the output stay untouched."""
    M, N, K = 600, 776, 1096
    g = torch.Generator().manual_seed(11)
    Abig = torch.randn(M, K + 24, generator=g).to(torch.bfloat16).cuda()
    Wbig = torch.randn(K, N + 40, generator=g).to(torch.bfloat16).cuda()
    A, W = Abig[:, 8:8 + K], Wbig[:, 16:16 + N]
    Cbig = torch.full((M + 2, N + 16), 7.0, dtype=torch.bfloat16, device="cuda")
    C = Cbig[1:1 + M, 8:8 + N]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cuda_lib.axon_gemm_bf16_plan(M, N, K, A.data_ptr(), A.stride(0), W.data_ptr(), W.stride(0), C.data_ptr(),
                                 C.stride(0), err, 4, gemm_ws, gemm_ws.numel())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check(C, A, W, "stream-K strided")
    keep = torch.ones_like(Cbig, dtype=torch.bool)
    keep[1:1 + M, 8:8 + N] = False
    assert torch.all(Cbig[keep] == 7.0)


def test_gemm_plan_errors(cuda_lib, gemm_ws):
    a = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    call = cuda_lib.axon_gemm_bf16_plan
    assert call(256, 256, 256, a, 256, a, 256, c, 256, None, 4, None, 0, raise_on_error=False) == 4
    assert call(256, 256, 256, a, 256, a, 256, c, 256, None, 4, gemm_ws, 1024, raise_on_error=False) == 4
    assert call(256, 256, 256, a, 256, a, 256, c, 256, None, 7, gemm_ws, gemm_ws.numel(),
                raise_on_error=False) == 1
    ws_over_c = c.view(torch.uint8)
    assert call(256, 256, 256, a, 256, a, 256, c, 256, None, 4, ws_over_c, gemm_ws.numel(),
                raise_on_error=False) == 1


def test_gemm_stream_k_back_to_back_calls_share_a_workspace(cuda_lib, gemm_ws):
    """Stream-K products enqueued back to back with one workspace and no
    synchronisation (operands A, B, then A again): each call clears its flags
    on the stream before it runs, so the two A results agree bit for bit and
    B's matches B run on its own (no owner sees a flag or partial left by the
    call before)."""
    M, N, K = 2048, 2560, 7680
    g = torch.Generator().manual_seed(21)
    ops = [((torch.randn(M, K, generator=g) / K ** 0.25).to(torch.bfloat16).cuda(),
            (torch.randn(K, N, generator=g) / K ** 0.25).to(torch.bfloat16).cuda()) for _ in range(2)]
    outs = [cuda_lib.gemm_bf16(A, W, plan=4, workspace=gemm_ws, check=False) for A, W in (ops[0], ops[1], ops[0])]
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
    alone = cuda_lib.gemm_bf16(*ops[1], plan=4, workspace=torch.empty_like(gemm_ws))
    torch.cuda.synchronize()
    assert torch.equal(outs[1].view(torch.int16), alone.view(torch.int16))
