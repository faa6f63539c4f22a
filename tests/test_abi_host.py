"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments with the documented status before
launching anything.

Every call below fails argument validation, so no kernel is ever launched
with the fake (never dereferenced) pointers used here; these tests are safe
with or without a GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_52_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if fn.endswith(".h"):
            src = open(os.path.join(HEADER_DIR, fn)).read()
            names += re.findall(r"AXON_API\s+[\w\s\*]+?\b(axon_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ("axon_ssm_scan_fwd", "axon_ssm_step", "axon_ssm_scan_workspace_bytes",
                     "axon_status_string", "axon_ssm_abi_version", "axon_ssm_scan_fwd_segments"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from selective_state_space_52_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings_and_version(lib):
    lib.axon_status_string.restype = ctypes.c_char_p
    assert lib.axon_status_string(0) == b"AXON_OK"
    assert lib.axon_status_string(4) == b"AXON_ERR_WORKSPACE"
    assert lib.axon_status_string(99) == b"AXON_ERR_UNKNOWN"
    assert lib.axon_ssm_abi_version() == 1


def test_workspace_query(lib):
    q = lib.axon_ssm_scan_workspace_bytes
    q.restype = ctypes.c_size_t
    # (P_max - 1) * B * E * (N + 1) * 4 with P_max = min(64, L // 128)
    assert q(1, 2048, 7680, 16, 4, 1) == 15 * 7680 * 17 * 4
    assert q(1, 65536, 2048, 16, 4, 1) == 63 * 2048 * 17 * 4
    assert q(64, 128, 7680, 16, 4, 1) == 0          # short sequences never split
    assert q(1, 64, 32, 16, 4, 0) == 0
    assert q(1, 4096, 64, 8, 4, 0) == 0             # unsupported N -> 0
    assert q(1, 4096, 60, 16, 4, 1) == 0            # E % 8 != 0 for bf16 -> rejected -> 0


# A fake, 16-byte aligned, never-dereferenced device address.
FAKE = 1 << 40


def _scan(lib, **over):
    a = dict(B=1, L=64, E=32, N=16, K=4, io=0,
             x=FAKE, z=FAKE + 0x10000, dt_raw=FAKE + 0x20000, Bm=FAKE + 0x30000, Cm=FAKE + 0x40000,
             conv_w=FAKE + 0x50000, conv_b=FAKE + 0x60000, dt_bias=FAKE + 0x70000,
             A_log=FAKE + 0x80000, D=FAKE + 0x90000, cc_in=None, ss_in=None,
             y=FAKE + 0xA0000, cc_out=FAKE + 0xB0000, ss_out=FAKE + 0xC0000,
             ws=None, ws_bytes=0, segs=0)
    a.update(over)
    f = lib.axon_ssm_scan_fwd_segments
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 15 + [ctypes.c_void_p, ctypes.c_size_t,
                                                               ctypes.c_int, ctypes.c_void_p]
    return f(a["B"], a["L"], a["E"], a["N"], a["K"], a["io"], a["x"], a["z"], a["dt_raw"],
             a["Bm"], a["Cm"], a["conv_w"], a["conv_b"], a["dt_bias"], a["A_log"], a["D"],
             a["cc_in"], a["ss_in"], a["y"], a["cc_out"], a["ss_out"], a["ws"], a["ws_bytes"],
             a["segs"], None)


OK, INVALID, UNSUPPORTED, ALIGNMENT, WORKSPACE = 0, 1, 2, 3, 4


@pytest.mark.parametrize("over,status", [
    (dict(B=-1), INVALID),
    (dict(L=-5), INVALID),
    (dict(E=-8), INVALID),
    (dict(N=8), UNSUPPORTED),
    (dict(N=32), UNSUPPORTED),
    (dict(K=3), UNSUPPORTED),
    (dict(io=7), UNSUPPORTED),
    (dict(B=70000), UNSUPPORTED),
    (dict(E=30), ALIGNMENT),                      # fp32 needs E % 4 == 0
    (dict(E=36, io=1), ALIGNMENT),                # bf16 needs E % 8 == 0
    (dict(x=None), INVALID),
    (dict(Bm=None), INVALID),
    (dict(y=None), INVALID),
    (dict(conv_w=None), INVALID),
    (dict(D=None), INVALID),
    (dict(cc_out=None), INVALID),
    (dict(ss_out=None), INVALID),
    (dict(x=FAKE + 4), ALIGNMENT),
    (dict(y=FAKE + 0xA0008), ALIGNMENT),
    (dict(cc_in=FAKE + 0xD0002), ALIGNMENT),
    (dict(y=FAKE), INVALID),                      # y overlaps x
    (dict(y=FAKE + 0x40000), INVALID),            # y overlaps Cm
    (dict(cc_in=FAKE + 0xB0010), INVALID),        # partial overlap of the cache in/out
    (dict(ss_in=FAKE + 0xC0040), INVALID),        # partial overlap of the state in/out
    (dict(ss_out=FAKE + 0xB0000 + 64), INVALID),  # state overlaps conv cache
    (dict(segs=-1), INVALID),
    (dict(segs=65, L=100000), INVALID),           # more than 64 segments
    (dict(segs=32, L=64), INVALID),               # segments shorter than the conv window
    (dict(segs=2, L=256), WORKSPACE),             # split needs workspace, none given
    (dict(segs=2, L=256, ws=FAKE + 0x100000, ws_bytes=100), WORKSPACE),
    (dict(segs=2, L=256, ws=FAKE + 0x100004, ws_bytes=1 << 20), ALIGNMENT),
])
def test_scan_rejects_bad_arguments(lib, over, status):
    assert _scan(lib, **over) == status


def test_scan_noop_sizes_launch_nothing(lib):
    # B == 0 or E == 0: nothing to do, OK without touching the device
    assert _scan(lib, B=0) == OK
    assert _scan(lib, E=0) == OK


def _step(lib, **over):
    a = dict(B=2, E=16, N=16, K=4, io=1,
             x=FAKE, z=FAKE + 0x10000, dt_raw=FAKE + 0x20000, Bm=FAKE + 0x30000, Cm=FAKE + 0x40000,
             conv_w=FAKE + 0x50000, conv_b=FAKE + 0x60000, dt_bias=FAKE + 0x70000,
             A_log=FAKE + 0x80000, D=FAKE + 0x90000, cc=FAKE + 0xA0000, ss=FAKE + 0xB0000,
             y=FAKE + 0xC0000)
    a.update(over)
    f = lib.axon_ssm_step
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 14
    return f(a["B"], a["E"], a["N"], a["K"], a["io"], a["x"], a["z"], a["dt_raw"], a["Bm"],
             a["Cm"], a["conv_w"], a["conv_b"], a["dt_bias"], a["A_log"], a["D"], a["cc"],
             a["ss"], a["y"], None)


@pytest.mark.parametrize("over,status", [
    (dict(B=-2), INVALID),
    (dict(N=4), UNSUPPORTED),
    (dict(K=2), UNSUPPORTED),
    (dict(E=12), ALIGNMENT),
    (dict(x=None), INVALID),
    (dict(cc=None), INVALID),
    (dict(ss=None), INVALID),
    (dict(y=None), INVALID),
    (dict(ss=FAKE + 0xB0004), ALIGNMENT),
    (dict(y=FAKE + 0xA0000), INVALID),             # y overlaps the conv cache
    (dict(ss=FAKE + 0xA0000 + 32), INVALID),       # state overlaps the conv cache
    (dict(x=FAKE + 0xC0000), INVALID),             # x overlaps y
])
def test_step_rejects_bad_arguments(lib, over, status):
    assert _step(lib, **over) == status


def test_step_noop_sizes(lib):
    assert _step(lib, B=0) == OK
    assert _step(lib, E=0) == OK


def test_discretization_enum_is_checked(lib):
    f = lib.axon_ssm_scan_fwd_ex
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p] * 15 + [ctypes.c_void_p, ctypes.c_size_t,
                                                               ctypes.c_int, ctypes.c_void_p]
    ptrs = [FAKE + 0x10000 * i for i in range(15)]
    assert f(1, 64, 32, 16, 4, 0, 2, *ptrs, None, 0, 0, None) == UNSUPPORTED
    assert f(1, 64, 32, 8, 4, 0, 1, *ptrs, None, 0, 0, None) == UNSUPPORTED    # N checked as usual
    g = lib.axon_ssm_step_ex
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 14
    assert g(2, 16, 16, 4, 1, -1, *ptrs[:13], None) == UNSUPPORTED
    assert g(2, 16, 16, 4, 1, 1, None, *ptrs[1:13], None) == INVALID


def test_binding_module_exposes_c_names():
    from selective_state_space_52_b200 import axon_ssm
    for name in declared_symbols():
        assert callable(getattr(axon_ssm, name)), name


def _block(lib, **over):
    a = dict(B=1, L=64, Dm=256, E=768, N=16, K=4, io=1, ws_bytes=1 << 34)
    ptr_names = ["X", "W_in", "W_x", "W_out", "conv_w", "conv_b", "dt_bias", "A_log", "D",
                 "cc_in", "ss_in", "out", "cc_out", "ss_out", "ws"]
    for i, n in enumerate(ptr_names):
        a[n] = FAKE + (i << 32)          # far apart: no overlaps unless a case makes one
    a["cc_in"] = a["ss_in"] = None
    a.update(over)
    f = lib.axon_ssm_block_fwd
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p] * 14 + [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    return f(a["B"], a["L"], a["Dm"], a["E"], a["N"], a["K"], a["io"], *(a[n] for n in ptr_names[:14]),
             a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("over,status", [
    (dict(B=-1), INVALID),
    (dict(io=0), UNSUPPORTED),                     # the whole layer is bf16 only
    (dict(N=8), UNSUPPORTED),
    (dict(Dm=260), ALIGNMENT),
    (dict(E=772), ALIGNMENT),
    (dict(X=None), INVALID),
    (dict(W_x=None), INVALID),
    (dict(ws=None), INVALID),
    (dict(W_in=FAKE + 8), ALIGNMENT),
    (dict(ws_bytes=1024), WORKSPACE),
    (dict(out=FAKE), INVALID),                     # out overlaps X
    (dict(ws=FAKE + (2 << 32)), INVALID),          # workspace overlaps W_x
])
def test_block_rejects_bad_arguments(lib, over, status):
    assert _block(lib, **over) == status


def test_block_workspace_query(lib):
    q = lib.axon_ssm_block_workspace_bytes
    q.restype = ctypes.c_size_t
    q.argtypes = [ctypes.c_int] * 7
    need = q(1, 2048, 2560, 7680, 16, 4, 1)
    assert need >= 5 * 2048 * 7680 * 2 + 2 * 2048 * 16 * 2   # x, z, u, dt_raw, y (M, E) and B, C (M, N) in bf16
    assert q(1, 2048, 2560, 7680, 16, 4, 0) == 0          # fp32 io: not supported
    assert _block(lib, ws_bytes=need - 1, L=2048, Dm=2560, E=7680) == WORKSPACE


def test_time_split_pieces_reject_bad_arguments(lib):
    s = lib.axon_ssm_dt_sum
    s.restype = ctypes.c_int
    s.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 4
    assert s(-1, 8, 16, 1, FAKE, FAKE + 0x10000, FAKE + 0x20000, None) == INVALID
    assert s(1, 8, 16, 5, FAKE, FAKE + 0x10000, FAKE + 0x20000, None) == UNSUPPORTED
    assert s(1, 8, 16, 1, FAKE, None, FAKE + 0x20000, None) == INVALID
    assert s(1, 8, 16, 1, FAKE + 2, FAKE + 0x10000, FAKE + 0x20000, None) == ALIGNMENT
    assert s(1, 8, 16, 1, FAKE, FAKE + 0x10000, FAKE + 16, None) == INVALID      # sum overlaps dt_raw
    assert s(0, 8, 16, 1, FAKE, FAKE + 0x10000, FAKE + 0x20000, None) == OK       # nothing to do
    f = lib.axon_ssm_carry_fold
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 5
    args = (FAKE, FAKE + 0x100000, FAKE + 0x200000, FAKE + 0x300000, None)
    assert f(4, 0, 1, 16, 16, *args) == INVALID          # slice 0 has no carry to fold
    assert f(4, 4, 1, 16, 16, *args) == INVALID          # r < P
    assert f(0, 1, 1, 16, 16, *args) == INVALID
    assert f(4, 1, 1, 16, 8, *args) == UNSUPPORTED
    assert f(4, 1, 1, 16, 16, FAKE, FAKE + 0x100000, FAKE + 0x200000, FAKE + 0x100000, None) == INVALID
    assert f(4, 1, 1, 16, 16, FAKE, FAKE + 0x100004, FAKE + 0x200000, FAKE + 0x300000, None) == ALIGNMENT


def test_ssd_rejects_bad_arguments(lib):
    f = lib.axon_ssd_scan_fwd
    f.restype = ctypes.c_int
    f.argtypes = ([ctypes.c_int] * 6 + [ctypes.c_void_p] * 10 +
                  [ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p])
    ptrs = [FAKE + (i << 32) for i in range(10)]      # x, dt_raw, dt_bias, A_log, B, C, D, h0, y, h_out
    ws = FAKE + (10 << 32)

    def call(B=1, L=128, H=2, P=64, N=128, io=1, segments=1, ws_ptr=ws, ws_bytes=1 << 30, **over):
        p = list(ptrs)
        for i, v in over.items():
            p[int(i[1:])] = v
        return f(B, L, H, P, N, io, *p, segments, ws_ptr, ws_bytes, None)

    assert call(B=-1) == INVALID
    assert call(segments=-1) == INVALID
    assert call(ws_ptr=None) == INVALID                         # a workspace is needed when L > 0
    assert call(P=32) == UNSUPPORTED
    assert call(N=64) == UNSUPPORTED
    assert call(io=0) == UNSUPPORTED                            # bf16 only
    assert call(p0=None) == INVALID
    assert call(p9=None) == INVALID
    assert call(p2=FAKE + 8) == ALIGNMENT
    assert call(ws_bytes=100) == WORKSPACE
    assert call(p8=ptrs[0]) == INVALID                          # y overlaps x
    assert call(p9=ptrs[7] + 16) == INVALID                     # h_out partly overlaps h0
    assert call(B=0) == OK
    q = lib.axon_ssd_workspace_bytes
    q.restype = ctypes.c_size_t
    q.argtypes = [ctypes.c_int] * 6
    # one segment: a 256-byte error flag and the per-chunk decays (two
    # 128-token chunks per batch row: acum, log2 dt - acum, w, v per token and head)
    prep = 2 * 3 * 2 * 4 * 128 * 4
    assert q(2, 130, 3, 64, 128, 1) == 256 + prep
    # two segments (one chunk each): the state-only walk over the first segment
    # adds one local end state per (b, h) and its decay, plus the copy of h0
    state = 2 * 3 * 64 * 128 * 4
    assert q(2, 130, 3, 64, 128, 2) == 256 + prep + state + 256 + state
    assert q(2, 130, 3, 64, 128, 5) == q(2, 130, 3, 64, 128, 2)     # at most one segment per chunk
    assert q(2, 0, 3, 64, 128, 0) == 0
    assert q(1, 128, 1, 32, 128, 0) == 0
    assert q(1, 128, 1, 64, 128, -1) == 0


def _ceil(a, b):
    return -(-a // b)


def _up256(n):
    return _ceil(n, 256) * 256


def ssd_plan_bytes(B, L, H, segments, sms=148):
    """The SSD call's plan restated: 128-token chunks; segments so that the
    full walks give one per SM (or as requested), at most one per chunk and 64;
    the first walk's pieces so that it gives three per SM; the workspace is an
    error flag, four floats per token and head, and per piece a local state and
    its decay plus a copy of h0."""
    nC = _ceil(L, 128)
    if nC <= 1:
        segs, cps = 1, max(nC, 1)
    else:
        want = segments if segments > 0 else max(1, sms // (B * H))
        want = min(want, nC, 64)
        cps = _ceil(nC, want)
        segs = _ceil(nC, cps)
    pcs = 1
    if segs > 1:
        pcs = min(max(1, 3 * sms // ((segs - 1) * B * H)), cps)
    cpp = _ceil(cps, pcs)
    pcs = _ceil(cps, cpp)
    if nC == 0:
        return 0, segs, pcs
    total = 256 + _up256(B * H * nC * 4 * 128 * 4)
    if segs > 1:
        extra = (segs - 1) * pcs
        total += _up256(extra * B * H * 64 * 128 * 4) + _up256(extra * B * H * 4) + _up256(B * H * 64 * 128 * 4)
    return total, segs, pcs


@pytest.mark.parametrize("B,L,H", [(1, 4096, 64), (2, 1000, 3), (1, 65536, 1), (8, 2048, 32), (1, 129, 2),
                                   (4, 128, 8), (1, 300000, 2)])
@pytest.mark.parametrize("segments", [0, 1, 2, 5, 100])
def test_ssd_plan_and_workspace(lib, B, L, H, segments):
    q = lib.axon_ssd_workspace_bytes
    q.restype = ctypes.c_size_t
    q.argtypes = [ctypes.c_int] * 6
    want, segs, pcs = ssd_plan_bytes(B, L, H, segments)
    assert q(B, L, H, 64, 128, segments) == want, (segs, pcs)
    assert segs <= 64 and segs <= max(1, _ceil(L, 128))


def test_ssd_wait_probe_rejects_bad_arguments(lib):
    f = lib.axon_ssd_wait_probe
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    assert f(None, 64, None) == INVALID
    assert f(FAKE + 2, 64, None) == INVALID                     # not 4-byte aligned
    assert f(FAKE, 0, None) == INVALID
    assert f(FAKE, (1 << 16) + 1, None) == INVALID


def test_exp2_fma_argument_checks(lib):
    """The FMA-pipe exp2's host checks (nothing is launched on an error)."""
    f = lib.axon_exp2_fma
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p]
    assert f(None, None, 0, None) == 0                          # nothing to do
    assert f(FAKE, FAKE + 4096, -1, None) == INVALID
    assert f(None, FAKE, 8, None) == INVALID
    assert f(FAKE, None, 8, None) == INVALID
    assert f(FAKE + 4, FAKE + 4096, 8, None) == ALIGNMENT
    assert f(FAKE, FAKE + 16, 8, None) == INVALID               # partial overlap


def _scan_state(lib, **over):
    a = dict(B=1, L=64, E=32, N=16, K=4, io=0)
    names = ["x", "dt_raw", "Bm", "conv_w", "conv_b", "dt_bias", "A_log", "cc_in", "ss_in", "cc_out", "ss_out", "dts"]
    for i, n in enumerate(names):
        a[n] = FAKE + (i << 32)
    a["cc_in"] = a["ss_in"] = None
    a.update(over)
    f = lib.axon_ssm_scan_state
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 12 + [ctypes.c_void_p]
    return f(a["B"], a["L"], a["E"], a["N"], a["K"], a["io"], *(a[n] for n in names), None)


@pytest.mark.parametrize("over,status", [
    (dict(N=8), UNSUPPORTED),
    (dict(K=3), UNSUPPORTED),
    (dict(io=7), UNSUPPORTED),
    (dict(E=30), ALIGNMENT),                       # fp32 needs E % 4 == 0
    (dict(B=-1), INVALID),
    (dict(dts=None), INVALID),
    (dict(x=None), INVALID),
    (dict(Bm=None), INVALID),
    (dict(conv_w=FAKE + 8), ALIGNMENT),
    (dict(ss_out=FAKE + (9 << 32) + 16), INVALID),    # overlaps the conv cache output
    (dict(dts=FAKE), INVALID),                        # overlaps x
    (dict(cc_in=FAKE + (9 << 32) + 16), INVALID),     # partly overlaps the conv cache output
])
def test_scan_state_argument_checks(lib, over, status):
    """The state-only scan's host checks: nothing is launched on an error."""
    assert _scan_state(lib, **over) == status


def test_scan_state_empty_is_ok(lib):
    assert _scan_state(lib, B=0) == OK
    assert _scan_state(lib, E=0) == OK


def test_peak_probe_argument_checks(lib):
    f = lib.axon_peak_probe
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_void_p]
    assert f(2, FAKE, 1, 1, None) == UNSUPPORTED
    assert f(0, None, 1, 1, None) == INVALID
    assert f(0, FAKE, 0, 1, None) == INVALID
    assert f(1, FAKE, 1, -1, None) == INVALID
    assert f(0, FAKE + 4, 1, 1, None) == ALIGNMENT


def test_gemm_plan_argument_checks(lib):
    """The tiling-choosing GEMM entry: plan range, the stream-K workspace
    (missing, too small, misaligned, overlapping an operand) -- all refused
    before anything is enqueued."""
    q = lib.axon_gemm_workspace_bytes
    q.restype = ctypes.c_size_t
    q.argtypes = []
    need = q()
    assert need == 128 * 2 * 128 * 256 * 4 + 128 * 2 * 4 * 4   # 128 pairs: two 128 x 256 float32 partials, 8 flags
    f = lib.axon_gemm_bf16_plan
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p, ctypes.c_int] * 3 + [ctypes.c_void_p, ctypes.c_int,
                                                                          ctypes.c_void_p, ctypes.c_size_t,
                                                                          ctypes.c_void_p]
    A, W, C, ws = FAKE, FAKE + (1 << 32), FAKE + (2 << 32), FAKE + (3 << 32)

    def call(plan, workspace=ws, nbytes=need, **kw):
        a = dict(M=256, N=256, K=64)
        a.update(kw)
        return f(a["M"], a["N"], a["K"], A, a["K"], W, a["N"], C, a["N"], None, plan, workspace, nbytes, None)

    assert call(5) == INVALID
    assert call(-1) == INVALID
    assert call(4, workspace=None, nbytes=0) == WORKSPACE          # stream-K needs the workspace
    assert call(4, nbytes=need - 1) == WORKSPACE
    assert call(4, workspace=ws + 4) == ALIGNMENT
    assert call(3, workspace=ws + 4) == ALIGNMENT                  # a given workspace is checked for every plan
    assert call(4, workspace=A + 64) == INVALID                     # overlaps A
    assert call(4, workspace=C - 1024) == INVALID                   # overlaps C
    assert call(4, M=0) == OK                                       # empty product
    assert call(4, N=12) == ALIGNMENT                               # N % 8
