"""fp64 CPU oracle for the selective-scan (S6) layer core -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does, and this package never imports the product.

The arithmetic lives in ``axon_ssm_oracle.c`` (plain C, double precision, one
thread; a second build of the same file with -fopenmp spreads independent
channels over the host's cores for the full-size checks, with identical
bits).  This module compiles it with gcc on first use and exposes numpy
wrappers.  Every function cites the passage of the page "Axon-SSM: Selective
State Space Model for Apple Silicon" (or the wiki page "Selective State Space
Models (Mamba)") that it follows; see the C source for the step list.

Parity pins (tests/test_oracle_pins.py) tie every function here to something
other than itself (for the conv stage: numpy.correlate and scipy's expit; for
the whole layer: closed forms with W_x = 0 and with dt at its upper clip): the recurrence == convolution identity and the worked
example of the Ultralytics glossary page "State Space Models (SSM)", the
geometric-series closed form, the A_log = log(1..N) initialisation, a brute
force of the unrolled (attention-like) form, and decode == prefill.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "axon_ssm_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle_axon_ssm.so")
_LIB_OMP_PATH = os.path.join(_BUILD_DIR, "liboracle_axon_ssm_omp.so")
_lock = threading.Lock()
_libs = {}

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile the C oracle into a shared library with gcc (no -ffast-math).

    ``openmp=True`` builds the same source a second time with -fopenmp: its
    channel loop then runs on all host cores (OMP_NUM_THREADS caps them), with
    each channel's arithmetic unchanged, so both builds give identical bits.
    """
    os.makedirs(_BUILD_DIR, exist_ok=True)
    path = _LIB_OMP_PATH if openmp else _LIB_PATH
    stale = (not os.path.exists(path)
             or os.path.getmtime(path) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = path + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", *(["-fopenmp"] if openmp else []), "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, path)
    return path


def _load(openmp: bool = False):
    with _lock:
        lib = _libs.get(openmp)
        if lib is None:
            # AXON_ORACLE_LIB points the pins at another build of this source
            # (the mutation tests plant mistakes in copies of it).
            env = os.environ.get("AXON_ORACLE_LIB_OMP" if openmp else "AXON_ORACLE_LIB")
            path = env or build(openmp=openmp)
            lib = ctypes.CDLL(path)
            lib.oracle_silu.restype = ctypes.c_double
            lib.oracle_silu.argtypes = [ctypes.c_double]
            lib.oracle_dt.restype = ctypes.c_double
            lib.oracle_dt.argtypes = [ctypes.c_double]
            lib.oracle_scan_core.restype = None
            lib.oracle_scan_core.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _dp, _dp,
                                             _dp, _dp, ctypes.c_double, ctypes.c_int,
                                             _dp, _dp]
            lib.oracle_ssm_scan_fwd.restype = ctypes.c_int
            lib.oracle_ssm_scan_fwd.argtypes = [ctypes.c_int] * 5 + [_dp] * 12 + [_dp] * 3 + [ctypes.c_int]
            lib.oracle_ssm_step.restype = ctypes.c_int
            lib.oracle_ssm_step.argtypes = [ctypes.c_int] * 4 + [_dp] * 10 + [_dp] * 3 + [ctypes.c_int]
            lib.oracle_conv_silu.restype = ctypes.c_int
            lib.oracle_conv_silu.argtypes = [ctypes.c_int] * 4 + [_dp] * 5
            lib.oracle_ssd_scan.restype = ctypes.c_int
            lib.oracle_ssd_scan.argtypes = [ctypes.c_int] * 5 + [_dp] * 10
            lib.oracle_threads.restype = ctypes.c_int
            lib.oracle_threads.argtypes = []
            _libs[openmp] = lib
    return lib


def threads(parallel: bool = False) -> int:
    """Host threads the prefill's channel loop uses in the chosen build."""
    return int(_load(parallel).oracle_threads())


def _f64(a) -> np.ndarray:
    """Exact upcast to a contiguous float64 array (bf16/fp32 values are kept bit-exact)."""
    if hasattr(a, "detach"):  # a torch tensor: upcast through torch, no re-rounding
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def silu(v: float) -> float:
    """SiLU(v) = v * sigmoid(v) (Axon-SSM page, "Gating")."""
    return _load().oracle_silu(float(v))


def dt_from_raw(v: float) -> float:
    """clip(softplus(v), 1e-4, 100) (Axon-SSM page, "Selective mechanism")."""
    return _load().oracle_dt(float(v))


def scan_core(u, dt, A, Bm, Cm, D=0.0, h0=None, zoh=False):
    """Recurrence only, one channel: u, dt (L,); A (N,) negative diagonal; Bm, Cm (L,N).

    Follows the toy ``selective_scan`` of the wiki page "Selective State Space
    Models (Mamba)" (discretise, zero state, loop over t) plus the D skip of the
    Axon-SSM recurrence equation.  Returns (y (L,), h_final (N,)).
    """
    u, dt, A, Bm, Cm = (_f64(v) for v in (u, dt, A, Bm, Cm))
    L = u.shape[0]
    N = A.shape[0]
    assert dt.shape == (L,) and Bm.shape == (L, N) and Cm.shape == (L, N)
    h = np.zeros(N) if h0 is None else _f64(h0).copy()
    y = np.zeros(L)
    _load().oracle_scan_core(L, N, _ptr(u), _ptr(dt), _ptr(A), _ptr(Bm), _ptr(Cm),
                             float(D), int(bool(zoh)), _ptr(h), _ptr(y))
    return y, h


def scan_fwd(x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
             conv_cache=None, ssm_state=None, zoh=False, parallel=False):
    """Layer core over a sequence (prefill), fp64.

    x, z, dt_raw: (B,L,E); Bm, Cm: (B,L,N); conv_w (E,K); conv_b, dt_bias, D (E,);
    A_log (E,N); conv_cache (B,K-1,E) or None; ssm_state (B,E,N) or None.
    Returns (y (B,L,E), conv_cache_out (B,K-1,E), ssm_state_out (B,E,N)).
    ``parallel`` runs the OpenMP build of the same source (identical bits).
    """
    x, z, dt_raw, Bm, Cm = (_f64(v) for v in (x, z, dt_raw, Bm, Cm))
    conv_w, conv_b, dt_bias, A_log, D = (_f64(v) for v in (conv_w, conv_b, dt_bias, A_log, D))
    Bsz, L, E = x.shape
    E2, K = conv_w.shape
    N = A_log.shape[1]
    assert E2 == E and Bm.shape == (Bsz, L, N) and Cm.shape == (Bsz, L, N)
    cc = None if conv_cache is None else _f64(conv_cache)
    ss = None if ssm_state is None else _f64(ssm_state)
    y = np.zeros((Bsz, L, E))
    cc_out = np.zeros((Bsz, K - 1, E))
    ss_out = np.zeros((Bsz, E, N))
    rc = _load(parallel).oracle_ssm_scan_fwd(Bsz, L, E, N, K, _ptr(x), _ptr(z), _ptr(dt_raw),
                                     _ptr(Bm), _ptr(Cm), _ptr(conv_w), _ptr(conv_b),
                                     _ptr(dt_bias), _ptr(A_log), _ptr(D), _ptr(cc), _ptr(ss),
                                     _ptr(y), _ptr(cc_out), _ptr(ss_out), int(bool(zoh)))
    if rc != 0:
        raise RuntimeError("oracle_ssm_scan_fwd failed")
    return y, cc_out, ss_out


def step(x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
         conv_cache, ssm_state, zoh=False):
    """One cached decode step (Axon-SSM page, "Autoregressive decoding").

    x, z, dt_raw: (B,E); Bm, Cm: (B,N); conv_cache (B,K-1,E); ssm_state (B,E,N).
    Returns (y (B,E), conv_cache_new, ssm_state_new); the inputs are not modified.
    """
    x, z, dt_raw, Bm, Cm = (_f64(v) for v in (x, z, dt_raw, Bm, Cm))
    conv_w, conv_b, dt_bias, A_log, D = (_f64(v) for v in (conv_w, conv_b, dt_bias, A_log, D))
    cc = _f64(conv_cache).copy()
    ss = _f64(ssm_state).copy()
    Bsz, E = x.shape
    K = conv_w.shape[1]
    N = A_log.shape[1]
    y = np.zeros((Bsz, E))
    rc = _load().oracle_ssm_step(Bsz, E, N, K, _ptr(x), _ptr(z), _ptr(dt_raw), _ptr(Bm),
                                 _ptr(Cm), _ptr(conv_w), _ptr(conv_b), _ptr(dt_bias),
                                 _ptr(A_log), _ptr(D), _ptr(cc), _ptr(ss), _ptr(y),
                                 int(bool(zoh)))
    if rc != 0:
        raise RuntimeError("oracle_ssm_step failed")
    return y, cc, ss


def conv_silu(x, conv_w, conv_b, conv_cache=None):
    """u = SiLU(causal depthwise conv1d(x)) over (B,L,E), fp64: the conv output
    that feeds the projection f_proj of the full layer (Axon-SSM page,
    "Selective mechanism")."""
    x, conv_w, conv_b = (_f64(v) for v in (x, conv_w, conv_b))
    Bsz, L, E = x.shape
    K = conv_w.shape[1]
    cc = None if conv_cache is None else _f64(conv_cache)
    u = np.zeros((Bsz, L, E))
    rc = _load().oracle_conv_silu(Bsz, L, E, K, _ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(cc), _ptr(u))
    if rc != 0:
        raise RuntimeError("oracle_conv_silu failed")
    return u


def _round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float64."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def block_fwd(X, W_in, W_x, W_out, conv_w, conv_b, dt_bias, A_log, D,
              conv_cache=None, ssm_state=None, zoh=False, bf16_intermediates=False):
    """The whole Axon-SSM layer, fp64, in the page's order:

      (x, z) = split(X W_in)                 ("Gating": the input projection makes
                                              the two branches; W_in is (Dm, 2E),
                                              x = first E columns)
      u = SiLU(conv(x))                      (conv output)
      (dt_raw, B, C) = split(u W_x)          ("Selective mechanism": f_proj is a
                                              linear map of the conv output; W_x is
                                              (E, E + 2N): dt_raw, then B, then C)
      y = scan(x, z, dt_raw, B, C)           (the layer core: recurrence, D skip,
                                              SiLU(z) gate -- ``scan_fwd``)
      out = y W_out                          ("Gating": y_out = W_out (y_ssm * SiLU(z)))

    The matrix products are numpy's (fp64); the scan is the C oracle.  With
    ``bf16_intermediates`` the values a bf16 layer stores between its stages
    (x, z, u, dt_raw, B, C and y) are rounded to bf16 where it stores them;
    everything else stays fp64.
    Returns (out (B,L,Dm), conv_cache_out, ssm_state_out).
    """
    X, W_in, W_x, W_out = (_f64(v) for v in (X, W_in, W_x, W_out))
    E = W_in.shape[1] // 2
    N = _f64(A_log).shape[1]
    assert W_in.shape[1] == 2 * E and W_x.shape == (E, E + 2 * N) and W_out.shape[0] == E
    rnd = _round_bf16 if bf16_intermediates else (lambda a: a)
    xz = X @ W_in
    x, z = rnd(xz[..., :E]), rnd(xz[..., E:])
    u = rnd(conv_silu(x, conv_w, conv_b, conv_cache))
    p = u @ W_x
    dt_raw, Bm, Cm = rnd(p[..., :E]), rnd(p[..., E:E + N]), rnd(p[..., E + N:])
    y, cc, ss = scan_fwd(x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                         conv_cache, ssm_state, zoh=zoh)
    return rnd(y) @ W_out, cc, ss


def ssd_scan(x, dt_raw, dt_bias, A_log, Bm, Cm, D, h0=None):
    """The Mamba-2 (SSD) layer core with one scalar decay per head, fp64 (wiki
    page "Selective State Space Models (Mamba)", section "Mamba-2 block (SSD)").

    x (B,L,H,P); dt_raw (B,L,H); dt_bias, A_log, D (H,); Bm, Cm (B,L,N) shared
    by all heads; h0 (B,H,P,N) or None.  Returns (y (B,L,H,P), h_out (B,H,P,N)).
    """
    x, dt_raw, Bm, Cm = (_f64(v) for v in (x, dt_raw, Bm, Cm))
    dt_bias, A_log, D = (_f64(v) for v in (dt_bias, A_log, D))
    Bsz, L, H, P = x.shape
    N = Bm.shape[2]
    hh = None if h0 is None else _f64(h0)
    y = np.zeros((Bsz, L, H, P))
    h_out = np.zeros((Bsz, H, P, N))
    rc = _load().oracle_ssd_scan(Bsz, L, H, P, N, _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A_log),
                                 _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(hh), _ptr(y), _ptr(h_out))
    if rc != 0:
        raise RuntimeError("oracle_ssd_scan failed")
    return y, h_out


def scan_channels(inputs: dict, channels, zoh=False):
    """Oracle over a subset of (b, e) channels of a full-size problem.

    Channels are independent (the recurrence is per channel and state), so a
    sample of them can be checked at any L.  ``inputs`` holds the same tensors the
    CUDA path receives; ``channels`` is a list of (b, e).  Returns a dict with
    y (len(channels), L), conv_cache (len, K-1), ssm_state (len, N).
    """
    ys, ccs, sss = [], [], []
    for b, e in channels:
        sl = slice(e, e + 1)
        cc = inputs.get("conv_cache")
        ss = inputs.get("ssm_state")
        y, cco, sso = scan_fwd(
            inputs["x"][b:b + 1, :, sl], inputs["z"][b:b + 1, :, sl],
            inputs["dt_raw"][b:b + 1, :, sl], inputs["B"][b:b + 1], inputs["C"][b:b + 1],
            inputs["conv_w"][sl], inputs["conv_b"][sl], inputs["dt_bias"][sl],
            inputs["A_log"][sl], inputs["D"][sl],
            None if cc is None else cc[b:b + 1, :, sl],
            None if ss is None else ss[b:b + 1, sl], zoh=zoh)
        ys.append(y[0, :, 0])
        ccs.append(cco[0, :, 0])
        sss.append(sso[0, 0])
    return {"y": np.stack(ys), "conv_cache": np.stack(ccs), "ssm_state": np.stack(sss)}
