"""GPU parity of the exact zero-order-hold discretisation (Bbar = (exp(dt A) - 1)/A B,
Axon-SSM page, "ZOH discretisation"), selected through axon_ssm_scan_fwd_ex /
axon_ssm_step_ex, against the fp64 oracle run with zoh=True.

Covers the direct walk (many channels), the quadrant and eighths scans and
the run-split chunked kernel (fewer channels), the segment-carry split, the
decode step, decode == prefill, and dt at both clips (dt = 1e-4 makes dt*A
tiny: the series branch of the input factor; dt = 100 makes exp(dt A) vanish:
Bbar = B / |A|).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import axon_ssm
from selective_state_space_52_b200 import workloads as W

from gpu_util import check_close, state_tol, to_dev, tol_for

pytestmark = pytest.mark.gpu


def _gpu(inp, num_segments=None):
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    y, (cc, ss) = axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params,
                                    (d["conv_cache"], d["ssm_state"]), num_segments=num_segments,
                                    discretization="zoh")
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), cc.cpu(), ss.cpu().numpy()


def _ref(inp):
    return oracle.scan_fwd(inp["x"], inp["z"], inp["dt_raw"], inp["B"], inp["C"], inp["conv_w"],
                           inp["conv_b"], inp["dt_bias"], inp["A_log"], inp["D"],
                           inp["conv_cache"], inp["ssm_state"], zoh=True)


def _compare(inp, io, what, num_segments=None):
    y, cc, ss = _gpu(inp, num_segments)
    y_ref, cc_ref, ss_ref = _ref(inp)
    check_close(y, y_ref, tol_for(io, y_ref), what + " y")
    check_close(ss, ss_ref, state_tol(ss_ref), what + " state")
    assert torch.equal(cc, torch.from_numpy(cc_ref).to(cc.dtype))


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E,L", [(1, 8, 300), (2, 264, 1000), (1, 1000, 257), (1, 7680, 96),
                                   (8, 4800, 40), (1, 14800, 100), (1, 29600, 40), (16, 4800, 24),
                                   (2, 2048, 130)])
def test_zoh_chunked_kernel(cuda_lib, io, B, E, L):
    inp = W.make_inputs(W.custom(B, L, E, io=io, seed=7000 + E + L), with_state=True)
    _compare(inp, io, f"zoh B{B} E{E} L{L} {io}", num_segments=1)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shift", [-200.0, 0.0, 200.0])
def test_zoh_dt_at_the_clips(cuda_lib, io, shift):
    inp = W.make_inputs(W.custom(1, 120, 64, io=io, seed=7100 + int(abs(shift))), with_state=True)
    inp["dt_raw"] = (inp["dt_raw"].float() * 0.01 + shift).to(inp["dt_raw"].dtype)
    _compare(inp, io, f"zoh dt shift {shift}", num_segments=1)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_zoh_segment_split(cuda_lib, io):
    inp = W.make_inputs(W.custom(2, 1000, 48, io=io, seed=7200), with_state=True)
    _compare(inp, io, "zoh split", num_segments=7)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_zoh_decode_equals_prefill(cuda_lib, io):
    L0, L = 11, 27
    inp = W.make_inputs(W.custom(5, L, 264, io=io, seed=7300), with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    y0, cache = axon_ssm.scan_fwd(*(d[k][:, :L0].contiguous() for k in ("x", "z", "dt_raw", "B", "C")),
                                  params, (d["conv_cache"], d["ssm_state"]), discretization="zoh")
    ys = [y0.float().cpu().numpy()]
    for t in range(L0, L):
        yt = axon_ssm.step(*(d[k][:, t].contiguous() for k in ("x", "z", "dt_raw", "B", "C")),
                           params, cache, discretization="zoh")
        ys.append(yt.float().cpu().numpy()[:, None, :])
    torch.cuda.synchronize()
    y_ref, cc_ref, ss_ref = _ref(inp)
    y = np.concatenate(ys, axis=1)
    check_close(y, y_ref, tol_for(io, y_ref), "zoh decode y")
    check_close(cache[1].cpu().numpy(), ss_ref, state_tol(ss_ref), "zoh decode state")
    assert torch.equal(cache[0].cpu(), torch.from_numpy(cc_ref).to(cache[0].dtype))


def test_zoh_differs_from_first_order(cuda_lib):
    """The flag changes the result (guards against the flag being ignored)."""
    inp = W.make_inputs(W.custom(1, 64, 32, io="f32", seed=7400), with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    args = (d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, (d["conv_cache"], d["ssm_state"]))
    y1, _ = axon_ssm.scan_fwd(*args)
    y2, _ = axon_ssm.scan_fwd(*args, discretization="zoh")
    assert not torch.allclose(y1, y2, rtol=1e-3, atol=1e-5)
