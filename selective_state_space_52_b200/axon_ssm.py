"""Python binding of the C ABI in include/axon_ssm.h (ctypes, argument marshalling only).

Every step of the layer core runs in the CUDA library ``libaxon_ssm.so`` built
in-tree by ``selective_state_space_52_b200.build``.  There is no CPU or PyTorch
fallback: importing this module raises if the library is missing, and every
call raises ``AxonError`` on a non-OK status.  PyTorch provides device memory
and the current stream.

Functions named like the C entry points take torch tensors (device, contiguous)
and pass their pointers through; ``scan_fwd`` and ``step`` additionally allocate
outputs / workspace with torch for convenience.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libaxon_ssm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"CUDA library not built: {LIB_PATH} is missing. "
        "Run `python -m selective_state_space_52_b200.build` (nvcc, sm_100a).")

_lib = ctypes.CDLL(LIB_PATH)

AXON_F32 = 0
AXON_BF16 = 1
STATUS = {0: "AXON_OK", 1: "AXON_ERR_INVALID_ARG", 2: "AXON_ERR_UNSUPPORTED",
          3: "AXON_ERR_ALIGNMENT", 4: "AXON_ERR_WORKSPACE", 5: "AXON_ERR_CUDA",
          6: "AXON_ERR_TIMEOUT"}

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

_lib.axon_ssm_abi_version.restype = _i
_lib.axon_ssm_abi_version.argtypes = []
_lib.axon_status_string.restype = ctypes.c_char_p
_lib.axon_status_string.argtypes = [_i]
_lib.axon_ssm_scan_workspace_bytes.restype = _sz
_lib.axon_ssm_scan_workspace_bytes.argtypes = [_i] * 6
_lib.axon_ssm_scan_launch_count.restype = _i
_lib.axon_ssm_scan_launch_count.argtypes = [_i] * 6
_SCAN_ARGS = [_i] * 6 + [_vp] * 15 + [_vp, _sz]
_lib.axon_ssm_scan_fwd.restype = _i
_lib.axon_ssm_scan_fwd.argtypes = _SCAN_ARGS + [_vp]
_lib.axon_ssm_scan_fwd_segments.restype = _i
_lib.axon_ssm_scan_fwd_segments.argtypes = _SCAN_ARGS + [_i, _vp]
_lib.axon_ssm_scan_fwd_noalloc.restype = _i
_lib.axon_ssm_scan_fwd_noalloc.argtypes = [_i] * 6 + [_vp] * 15 + [_i, _vp]
NOALLOC_SCRATCH_BYTES = 16 << 20
_lib.axon_ssm_scan_fwd_qsplit.restype = _i
_lib.axon_ssm_scan_fwd_qsplit.argtypes = [_i] * 8 + [_vp] * 15 + [_vp]
_lib.axon_ssm_scan_fwd_ex.restype = _i
_lib.axon_ssm_scan_fwd_ex.argtypes = [_i] * 7 + [_vp] * 15 + [_vp, _sz, _i, _vp]
_lib.axon_ssm_step_ex.restype = _i
_lib.axon_ssm_step_ex.argtypes = [_i] * 6 + [_vp] * 13 + [_vp]
AXON_DISC_FIRST_ORDER = 0
AXON_DISC_ZOH = 1
_DISC = {"first_order": AXON_DISC_FIRST_ORDER, "zoh": AXON_DISC_ZOH}
_lib.axon_ssm_step.restype = _i
_lib.axon_ssm_step.argtypes = [_i] * 5 + [_vp] * 13 + [_vp]
_lib.axon_ssm_dt_sum.restype = _i
_lib.axon_ssm_dt_sum.argtypes = [_i] * 4 + [_vp] * 3 + [_vp]
_lib.axon_ssm_carry_fold.restype = _i
_lib.axon_ssm_carry_fold.argtypes = [_i] * 5 + [_vp] * 4 + [_vp]
_lib.axon_ssm_scan_state.restype = _i
_lib.axon_ssm_scan_state.argtypes = [_i] * 6 + [_vp] * 12 + [_vp]
_lib.axon_ssd_wait_probe.restype = _i
_lib.axon_ssd_wait_probe.argtypes = [_vp, _i, _vp]
_lib.axon_ssd_workspace_bytes.restype = _sz
_lib.axon_ssd_workspace_bytes.argtypes = [_i] * 6
_lib.axon_ssd_scan_fwd.restype = _i
_lib.axon_ssd_scan_fwd.argtypes = [_i] * 6 + [_vp] * 10 + [_i, _vp, _sz, _vp]
_lib.axon_gemm_bf16.restype = _i
_lib.axon_exp2_fma.restype = _i
_lib.axon_peak_probe.restype = _i
_lib.axon_peak_probe.argtypes = [_i, _vp, _i, ctypes.c_longlong, _vp]
_lib.axon_exp2_fma.argtypes = [_vp, _vp, ctypes.c_longlong, _vp]
_lib.axon_gemm_bf16.argtypes = [_i] * 3 + [_vp, _i, _vp, _i, _vp, _i, _vp, _vp]
_lib.axon_gemm_bf16_plan.restype = _i
_lib.axon_gemm_bf16_plan.argtypes = [_i] * 3 + [_vp, _i, _vp, _i, _vp, _i, _vp, _i, _vp, _sz, _vp]
_lib.axon_gemm_workspace_bytes.restype = _sz
_lib.axon_gemm_workspace_bytes.argtypes = []
_lib.axon_ssm_block_workspace_bytes.restype = _sz
_lib.axon_ssm_block_workspace_bytes.argtypes = [_i] * 7
_lib.axon_ssm_block_fwd.restype = _i
_lib.axon_ssm_block_fwd.argtypes = [_i] * 7 + [_vp] * 14 + [_vp, _sz, _vp]


class AxonError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return AXON_F32
    if t == torch.bfloat16:
        return AXON_BF16
    raise TypeError(f"unsupported io dtype {t}; use float32 or bfloat16")


def _p(t):
    """Device pointer of a tensor (None -> NULL).  Tensors must be contiguous."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to the C ABI must be contiguous")
    return t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != 0:
        raise AxonError(rc, where)


# ------------------------------------------------------------ C entry points
def axon_ssm_abi_version() -> int:
    return _lib.axon_ssm_abi_version()


def axon_status_string(status: int) -> str:
    return _lib.axon_status_string(int(status)).decode()


def axon_ssm_scan_workspace_bytes(B, L, E, N=16, K=4, io=AXON_BF16) -> int:
    return int(_lib.axon_ssm_scan_workspace_bytes(B, L, E, N, K, io))


def axon_ssm_scan_launch_count(B, L, E, N=16, K=4, io=AXON_BF16) -> int:
    return int(_lib.axon_ssm_scan_launch_count(B, L, E, N, K, io))


def axon_ssm_scan_fwd(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias,
                      A_log, D, conv_cache_in, ssm_state_in, y, conv_cache_out,
                      ssm_state_out, workspace, workspace_bytes, stream=None, *,
                      raise_on_error=True) -> int:
    rc = _lib.axon_ssm_scan_fwd(B, L, E, N, K, io, _p(x), _p(z), _p(dt_raw), _p(Bm), _p(Cm),
                                _p(conv_w), _p(conv_b), _p(dt_bias), _p(A_log), _p(D),
                                _p(conv_cache_in), _p(ssm_state_in), _p(y),
                                _p(conv_cache_out), _p(ssm_state_out), _p(workspace),
                                int(workspace_bytes), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_scan_fwd")
    return rc


def axon_ssm_scan_fwd_segments(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b,
                               dt_bias, A_log, D, conv_cache_in, ssm_state_in, y,
                               conv_cache_out, ssm_state_out, workspace, workspace_bytes,
                               num_segments, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_ssm_scan_fwd_segments(B, L, E, N, K, io, _p(x), _p(z), _p(dt_raw), _p(Bm),
                                         _p(Cm), _p(conv_w), _p(conv_b), _p(dt_bias),
                                         _p(A_log), _p(D), _p(conv_cache_in),
                                         _p(ssm_state_in), _p(y), _p(conv_cache_out),
                                         _p(ssm_state_out), _p(workspace),
                                         int(workspace_bytes), int(num_segments),
                                         _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_scan_fwd_segments")
    return rc


def axon_ssm_scan_fwd_noalloc(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b,
                              dt_bias, A_log, D, conv_cache_in, ssm_state_in, y,
                              conv_cache_out, ssm_state_out, num_segments=0, stream=None, *,
                              raise_on_error=True) -> int:
    """The prefill with its time-split scratch in the library's own 16 MiB device
    array, for callers that cannot provide a workspace (see include/axon_ssm.h)."""
    rc = _lib.axon_ssm_scan_fwd_noalloc(B, L, E, N, K, io, _p(x), _p(z), _p(dt_raw), _p(Bm),
                                        _p(Cm), _p(conv_w), _p(conv_b), _p(dt_bias),
                                        _p(A_log), _p(D), _p(conv_cache_in),
                                        _p(ssm_state_in), _p(y), _p(conv_cache_out),
                                        _p(ssm_state_out), int(num_segments), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_scan_fwd_noalloc")
    return rc


def axon_ssm_scan_fwd_qsplit(B, L, E, N, K, io, disc, runs, x, z, dt_raw, Bm, Cm, conv_w, conv_b,
                             dt_bias, A_log, D, conv_cache_in, ssm_state_in, y, conv_cache_out,
                             ssm_state_out, stream=None, *, raise_on_error=True) -> int:
    """The prefill on the split-chunk quadrant scan with `runs` warps per 8
    channels (1, 2, 4 or 8), for tests and tuning."""
    rc = _lib.axon_ssm_scan_fwd_qsplit(B, L, E, N, K, io, int(disc), int(runs), _p(x), _p(z),
                                       _p(dt_raw), _p(Bm), _p(Cm), _p(conv_w), _p(conv_b),
                                       _p(dt_bias), _p(A_log), _p(D), _p(conv_cache_in),
                                       _p(ssm_state_in), _p(y), _p(conv_cache_out),
                                       _p(ssm_state_out), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_scan_fwd_qsplit")
    return rc


def axon_ssm_scan_fwd_ex(B, L, E, N, K, io, disc, x, z, dt_raw, Bm, Cm, conv_w, conv_b,
                         dt_bias, A_log, D, conv_cache_in, ssm_state_in, y, conv_cache_out,
                         ssm_state_out, workspace, workspace_bytes, num_segments=0, stream=None, *,
                         raise_on_error=True) -> int:
    rc = _lib.axon_ssm_scan_fwd_ex(B, L, E, N, K, io, int(disc), _p(x), _p(z), _p(dt_raw),
                                   _p(Bm), _p(Cm), _p(conv_w), _p(conv_b), _p(dt_bias),
                                   _p(A_log), _p(D), _p(conv_cache_in), _p(ssm_state_in), _p(y),
                                   _p(conv_cache_out), _p(ssm_state_out), _p(workspace),
                                   int(workspace_bytes), int(num_segments), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_scan_fwd_ex")
    return rc


def axon_ssm_step_ex(B, E, N, K, io, disc, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias,
                     A_log, D, conv_cache, ssm_state, y, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_ssm_step_ex(B, E, N, K, io, int(disc), _p(x), _p(z), _p(dt_raw), _p(Bm),
                               _p(Cm), _p(conv_w), _p(conv_b), _p(dt_bias), _p(A_log), _p(D),
                               _p(conv_cache), _p(ssm_state), _p(y), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_step_ex")
    return rc


def axon_ssm_step(B, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                  conv_cache, ssm_state, y, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_ssm_step(B, E, N, K, io, _p(x), _p(z), _p(dt_raw), _p(Bm), _p(Cm),
                            _p(conv_w), _p(conv_b), _p(dt_bias), _p(A_log), _p(D),
                            _p(conv_cache), _p(ssm_state), _p(y), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_step")
    return rc


def axon_ssm_dt_sum(B, L, E, io, dt_raw, dt_bias, dt_sum, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_ssm_dt_sum(B, L, E, io, _p(dt_raw), _p(dt_bias), _p(dt_sum), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_dt_sum")
    return rc


def axon_ssm_carry_fold(P, r, B, E, N, A_log, h_loc, dt_sum, h_in, stream=None, *,
                        raise_on_error=True) -> int:
    rc = _lib.axon_ssm_carry_fold(P, r, B, E, N, _p(A_log), _p(h_loc), _p(dt_sum), _p(h_in),
                                  _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_carry_fold")
    return rc


def axon_ssm_scan_state(B, L, E, N, K, io, x, dt_raw, Bm, conv_w, conv_b, dt_bias, A_log,
                        conv_cache_in, ssm_state_in, conv_cache_out, ssm_state_out, dt_sum, stream=None, *,
                        raise_on_error=True) -> int:
    rc = _lib.axon_ssm_scan_state(B, L, E, N, K, io, _p(x), _p(dt_raw), _p(Bm), _p(conv_w), _p(conv_b),
                                  _p(dt_bias), _p(A_log), _p(conv_cache_in), _p(ssm_state_in),
                                  _p(conv_cache_out), _p(ssm_state_out), _p(dt_sum), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_scan_state")
    return rc


def axon_ssd_wait_probe(status, limit, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_ssd_wait_probe(_p(status), int(limit), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssd_wait_probe")
    return rc


def axon_ssd_workspace_bytes(B, L, H, P=64, N=128, segments=0) -> int:
    return int(_lib.axon_ssd_workspace_bytes(B, L, H, P, N, segments))


def axon_ssd_scan_fwd(B, L, H, P, N, io, x, dt_raw, dt_bias, A_log, Bm, Cm, D, h0, y, h_out, segments,
                      workspace, workspace_bytes, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_ssd_scan_fwd(B, L, H, P, N, io, _p(x), _p(dt_raw), _p(dt_bias), _p(A_log), _p(Bm),
                                _p(Cm), _p(D), _p(h0), _p(y), _p(h_out), int(segments), _p(workspace),
                                int(workspace_bytes), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssd_scan_fwd")
    return rc


def axon_ssm_block_workspace_bytes(B, L, Dm, E, N=16, K=4, io=AXON_BF16) -> int:
    return int(_lib.axon_ssm_block_workspace_bytes(B, L, Dm, E, N, K, io))


def axon_ssm_block_fwd(B, L, Dm, E, N, K, io, X, W_in, W_x, W_out, conv_w, conv_b, dt_bias,
                       A_log, D, conv_cache_in, ssm_state_in, out, conv_cache_out, ssm_state_out,
                       workspace, workspace_bytes, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_ssm_block_fwd(B, L, Dm, E, N, K, io, _p(X), _p(W_in), _p(W_x), _p(W_out),
                                 _p(conv_w), _p(conv_b), _p(dt_bias), _p(A_log), _p(D),
                                 _p(conv_cache_in), _p(ssm_state_in), _p(out), _p(conv_cache_out),
                                 _p(ssm_state_out), _p(workspace), int(workspace_bytes),
                                 _stream(stream))
    if raise_on_error:
        _check(rc, "axon_ssm_block_fwd")
    return rc


def axon_gemm_bf16(M, N, K, A, lda, W, ldw, C, ldc, err=None, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_gemm_bf16(M, N, K, _p(A), int(lda), _p(W), int(ldw), _p(C), int(ldc), _p(err),
                             _stream(stream))
    if raise_on_error:
        _check(rc, "axon_gemm_bf16")
    return rc


# tilings of axon_gemm_bf16_plan (include/axon_ssm.h)
GEMM_AUTO, GEMM_SINGLE_256, GEMM_SINGLE_192, GEMM_PAIR, GEMM_PAIR_STREAMK = 0, 1, 2, 3, 4


def axon_gemm_workspace_bytes() -> int:
    return int(_lib.axon_gemm_workspace_bytes())


def axon_gemm_bf16_plan(M, N, K, A, lda, W, ldw, C, ldc, err=None, plan=GEMM_AUTO, workspace=None,
                        workspace_bytes=0, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_gemm_bf16_plan(M, N, K, _p(A), int(lda), _p(W), int(ldw), _p(C), int(ldc), _p(err),
                                  int(plan), _p(workspace), int(workspace_bytes), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_gemm_bf16_plan")
    return rc


def axon_exp2_fma(x, y, n, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_exp2_fma(_p(x), _p(y), int(n), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_exp2_fma")
    return rc


def axon_peak_probe(kind, out, blocks, iters, stream=None, *, raise_on_error=True) -> int:
    rc = _lib.axon_peak_probe(int(kind), _p(out), int(blocks), int(iters), _stream(stream))
    if raise_on_error:
        _check(rc, "axon_peak_probe")
    return rc


def exp2_fma(x, *, out=None, stream=None):
    """2^x of a contiguous float32 CUDA tensor through the FMA-pipe exp2."""
    import torch
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("exp2_fma: x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x) if out is None else out
    axon_exp2_fma(x.data_ptr(), y.data_ptr(), x.numel(), stream=stream)
    return y


def gemm_bf16(A, W, *, out=None, stream=None, check=True, plan=GEMM_AUTO, workspace=None):
    """C = A @ W for row-major bf16 A (M x K) and W (K x N) on the library's
    tcgen05 GEMM (float32 accumulation; ``plan``: one of the GEMM_* tilings,
    ``workspace``: a uint8 CUDA tensor of axon_gemm_workspace_bytes() bytes,
    needed by GEMM_PAIR_STREAMK).  With ``check`` the call waits for the
    device and raises AxonError (AXON_ERR_TIMEOUT) if a wait of the kernel
    gave up."""
    M, K = A.shape
    N = W.shape[1]
    C = torch.empty(M, N, dtype=torch.bfloat16, device=A.device) if out is None else out
    err = torch.zeros(1, dtype=torch.int32, device=A.device)
    nws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    axon_gemm_bf16_plan(M, N, K, A, A.stride(0), W, W.stride(0), C, C.stride(0), err, plan, workspace, nws,
                        stream=stream)
    if check and int(err.item()) != 0:
        raise AxonError(6, "axon_gemm_bf16 (a wait for a copy or a tensor-core product gave up)")
    return C


# ------------------------------------------------------------ conveniences
PARAM_KEYS = ("conv_w", "conv_b", "dt_bias", "A_log", "D")
WEIGHT_KEYS = ("W_in", "W_x", "W_out")


def scan_fwd(x, z, dt_raw, Bm, Cm, params: dict, cache=None, *, num_segments=None,
             out=None, workspace=None, stream=None, discretization="first_order", runs=None):
    """Prefill over (B, L, E) inputs on the GPU.

    ``params`` holds conv_w, conv_b, dt_bias, A_log, D (float32, on the device);
    ``cache`` is None or (conv_cache, ssm_state).  Returns
    ``(y, (conv_cache, ssm_state))`` -- the cache pair of the Axon-SSM page's
    "Autoregressive decoding" section, ready for the next call or for ``step``.
    ``runs`` (tests and tuning) forces the split-chunk quadrant scan with that
    many warps per 8 channels.
    """
    Bsz, L, E = x.shape
    K = params["conv_w"].shape[1]
    N = params["A_log"].shape[1]
    io = _dtype_code(x.dtype)
    dev = x.device
    cc_in, ss_in = (None, None) if cache is None else cache
    if out is None:
        y = torch.empty_like(x)
        cc_out = torch.empty(Bsz, K - 1, E, dtype=x.dtype, device=dev)
        ss_out = torch.empty(Bsz, E, N, dtype=torch.float32, device=dev)
    else:
        y, cc_out, ss_out = out
    if workspace is None:
        if num_segments is None:
            nbytes = axon_ssm_scan_workspace_bytes(Bsz, L, E, N, K, io)
        else:
            nbytes = max(num_segments - 1, 0) * Bsz * E * (N + 1) * 4
        if nbytes > 0:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (Bsz, L, E, N, K, io, x, z, dt_raw, Bm, Cm, *(params[k] for k in PARAM_KEYS),
            cc_in, ss_in, y, cc_out, ss_out, workspace, wsz)
    if runs is not None:
        axon_ssm_scan_fwd_qsplit(Bsz, L, E, N, K, io, _DISC[discretization], runs, *args[6:-2],
                                 stream=stream)
    elif discretization != "first_order":
        axon_ssm_scan_fwd_ex(Bsz, L, E, N, K, io, _DISC[discretization], *args[6:],
                             num_segments or 0, stream=stream)
    elif num_segments is None:
        axon_ssm_scan_fwd(*args, stream=stream)
    else:
        axon_ssm_scan_fwd_segments(*args, num_segments, stream=stream)
    return y, (cc_out, ss_out)


def step(x, z, dt_raw, Bm, Cm, params: dict, cache, *, y=None, stream=None,
         discretization="first_order"):
    """One cached decode step; ``cache = (conv_cache, ssm_state)`` is updated in place."""
    Bsz, E = x.shape
    K = params["conv_w"].shape[1]
    N = params["A_log"].shape[1]
    conv_cache, ssm_state = cache
    if y is None:
        y = torch.empty_like(x)
    args = (x, z, dt_raw, Bm, Cm, *(params[k] for k in PARAM_KEYS), conv_cache, ssm_state, y)
    if discretization != "first_order":
        axon_ssm_step_ex(Bsz, E, N, K, _dtype_code(x.dtype), _DISC[discretization], *args,
                         stream=stream)
    else:
        axon_ssm_step(Bsz, E, N, K, _dtype_code(x.dtype), *args, stream=stream)
    return y


def block_error_flag(workspace) -> int:
    """The whole layer's GEMM error flag (the workspace's first int) after the
    call that used ``workspace`` has completed.  Synchronises the device."""
    torch.cuda.synchronize(workspace.device)
    return int(workspace[:4].view(torch.int32).item())


def block_fwd(X, weights: dict, params: dict, cache=None, *, out=None, workspace=None, stream=None,
              check=True):
    """The whole Axon-SSM layer on (B, L, Dm) bf16 input ``X``.

    ``weights`` holds W_in (Dm, 2E), W_x (E, E+2N), W_out (E, Dm) in bf16;
    ``params`` and ``cache`` as for ``scan_fwd``.  Returns
    ``(out, (conv_cache, ssm_state))``.  With ``check`` (the default) the call
    waits for the device and raises AxonError (AXON_ERR_TIMEOUT) if a wait of
    a projection GEMM gave up; ``check=False`` returns at once (read the flag
    with ``block_error_flag(workspace)``).
    """
    Bsz, L, Dm = X.shape
    E = weights["W_in"].shape[1] // 2
    K = params["conv_w"].shape[1]
    N = params["A_log"].shape[1]
    dev = X.device
    cc_in, ss_in = (None, None) if cache is None else cache
    if out is None:
        y = torch.empty_like(X)
        cc_out = torch.empty(Bsz, K - 1, E, dtype=X.dtype, device=dev)
        ss_out = torch.empty(Bsz, E, N, dtype=torch.float32, device=dev)
    else:
        y, cc_out, ss_out = out
    io = _dtype_code(X.dtype)
    nbytes = axon_ssm_block_workspace_bytes(Bsz, L, Dm, E, N, K, io)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    wsz = workspace.numel() * workspace.element_size()
    axon_ssm_block_fwd(Bsz, L, Dm, E, N, K, io, X, weights["W_in"], weights["W_x"], weights["W_out"],
                       *(params[k] for k in PARAM_KEYS), cc_in, ss_in, y, cc_out, ss_out,
                       workspace, wsz, stream=stream)
    if check and Bsz * E > 0 and block_error_flag(workspace) != 0:
        raise AxonError(6, "axon_ssm_block_fwd (a wait of a projection GEMM gave up)")
    return y, (cc_out, ss_out)


def dt_sum(dt_raw, dt_bias, *, stream=None):
    """(B, E) float32: the sum over the sequence of clip(softplus(dt_raw + dt_bias))."""
    Bsz, L, E = dt_raw.shape
    out = torch.empty(Bsz, E, dtype=torch.float32, device=dt_raw.device)
    axon_ssm_dt_sum(Bsz, L, E, _dtype_code(dt_raw.dtype), dt_raw, dt_bias, out, stream=stream)
    return out


def scan_state(x, dt_raw, Bm, params: dict, cache=None, *, stream=None):
    """The state-only prefill (first order): returns ((conv_cache, ssm_state),
    dt_sum) -- the final caches and the (B, E) float32 sum of the step sizes --
    without z, C, D or y."""
    Bsz, L, E = x.shape
    K = params["conv_w"].shape[1]
    N = params["A_log"].shape[1]
    cc_in, ss_in = (None, None) if cache is None else cache
    dev = x.device
    cc_out = torch.empty(Bsz, K - 1, E, dtype=x.dtype, device=dev)
    ss_out = torch.empty(Bsz, E, N, dtype=torch.float32, device=dev)
    dts = torch.empty(Bsz, E, dtype=torch.float32, device=dev)
    axon_ssm_scan_state(Bsz, L, E, N, K, _dtype_code(x.dtype), x, dt_raw, Bm, params["conv_w"], params["conv_b"],
                        params["dt_bias"], params["A_log"], cc_in, ss_in, cc_out, ss_out, dts, stream=stream)
    return (cc_out, ss_out), dts


def carry_fold(r, A_log, h_loc_all, dt_sum_all, *, stream=None):
    """The state entering slice r of a time-split sequence from the stacked
    (P,B,E,N) end states and (P,B,E) dt sums of all slices."""
    P, Bsz, E, N = h_loc_all.shape
    out = torch.empty(Bsz, E, N, dtype=torch.float32, device=h_loc_all.device)
    axon_ssm_carry_fold(P, r, Bsz, E, N, A_log, h_loc_all, dt_sum_all, out, stream=stream)
    return out


def ssd_error_flag(workspace) -> int:
    """The SSD walk's error flag (the workspace's first int) after the call
    that used ``workspace`` has completed: 1 if a wait for a tensor-core
    product gave up.  Synchronises the device."""
    torch.cuda.synchronize(workspace.device)
    return int(workspace[:4].view(torch.int32).item())


def ssd_scan(x, dt_raw, Bm, Cm, params: dict, h0=None, *, out=None, workspace=None, stream=None, segments=0,
             check=True):
    """The Mamba-2 (SSD) layer core on x (B,L,H,P) bf16; ``params`` holds
    dt_bias, A_log, D (H,) float32; ``segments`` = 0 lets the library cut the
    sequence for the current device.  Returns (y, h_out (B,H,P,N)).

    With ``check`` (the default) the call waits for the device and reads the
    walk's error flag from the workspace, raising ``AxonError``
    (AXON_ERR_TIMEOUT) if a wait for a tensor-core product gave up, in which
    case y and h_out are undefined.  ``check=False`` returns without waiting;
    the caller then reads the flag with ``ssd_error_flag(workspace)``."""
    Bsz, L, H, P = x.shape
    N = Bm.shape[2]
    if out is None:
        y = torch.empty_like(x)
        h_out = torch.empty(Bsz, H, P, N, dtype=torch.float32, device=x.device)
    else:
        y, h_out = out
    if workspace is None:
        with torch.cuda.device(x.device):
            nbytes = axon_ssd_workspace_bytes(Bsz, L, H, P, N, segments)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    axon_ssd_scan_fwd(Bsz, L, H, P, N, _dtype_code(x.dtype), x, dt_raw, params["dt_bias"], params["A_log"],
                      Bm, Cm, params["D"], h0, y, h_out, segments, workspace,
                      workspace.numel() * workspace.element_size(), stream=stream)
    if check and L > 0 and Bsz * H > 0 and ssd_error_flag(workspace) != 0:
        raise AxonError(6, "axon_ssd_scan_fwd (a wait for a tensor-core product gave up)")
    return y, h_out
