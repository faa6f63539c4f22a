"""The five measured workloads at full size, in the launch configuration the
benchmark times (the library's own plan), checked against the fp64 oracle on
every element.

The oracle runs as its OpenMP build (the same C source, its channel loop
spread over the host's cores, identical bits to the single-threaded build) on
blocks of channels or batch rows, so that host memory stays bounded: each
block's outputs are compared before the next block is computed.  y, the final
ssm_state and the conv_cache are all compared; the decode workload prefills
128 tokens and then runs 512 cached steps, and every step's output for every
(b, e) is compared with the oracle over the whole 640-token sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import axon_ssm
from selective_state_space_52_b200 import workloads as W

from gpu_util import check_close, compare_scan, state_tol, to_dev, tol_for

pytestmark = pytest.mark.gpu

SEQ_KEYS = ("x", "z", "dt_raw")
PARAM_E = ("conv_w", "conv_b", "dt_bias", "A_log", "D")


def oracle_block(inp, b0, b1, e0, e1):
    """The oracle (OpenMP build) on batch rows b0:b1 and channels e0:e1."""
    sl = slice(e0, e1)
    args = [inp[k][b0:b1, :, sl].contiguous() for k in SEQ_KEYS]
    args += [inp["B"][b0:b1], inp["C"][b0:b1]]
    args += [inp[k][sl] for k in PARAM_E]
    cc = inp.get("conv_cache")
    ss = inp.get("ssm_state")
    return oracle.scan_fwd(*args,
                           None if cc is None else cc[b0:b1, :, sl].contiguous(),
                           None if ss is None else ss[b0:b1, sl].contiguous(),
                           parallel=True)


def compare_full(wl, inp, y, cc, ss, e_block=512, b_block=8):
    """Every element of y (B,L,E), the conv cache and the state against the oracle."""
    B, L, E = wl.B, wl.L, wl.E
    eb = E if B > 1 else e_block
    bb = b_block if B > 1 else 1
    for b0 in range(0, B, bb):
        b1 = min(B, b0 + bb)
        for e0 in range(0, E, eb):
            e1 = min(E, e0 + eb)
            y_ref, cc_ref, ss_ref = oracle_block(inp, b0, b1, e0, e1)
            what = f"{wl.name} b{b0}:{b1} e{e0}:{e1}"
            yg = y[b0:b1, :, e0:e1].float().cpu().numpy()
            check_close(yg, y_ref, tol_for(wl.io, y_ref), what + " y")
            sg = ss[b0:b1, e0:e1].cpu().numpy()
            check_close(sg, ss_ref, state_tol(ss_ref), what + " ssm_state")
            ccg = cc[b0:b1, :, e0:e1].cpu()
            assert torch.equal(ccg, torch.from_numpy(cc_ref).to(ccg.dtype)), what + " conv_cache"


def test_tiny_workload_full_compare(cuda_lib):
    wl = W.WORKLOADS[0]
    inp = W.make_inputs(wl)
    compare_scan(inp, wl.io, with_state=False, what=wl.name)


@pytest.mark.parametrize("name", ["bit_axon_layer", "mamba_block", "long_seq"])
def test_prefill_workload_every_element(cuda_lib, name):
    wl = W.WORKLOAD_BY_NAME[name]
    inp = W.make_inputs(wl)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    y, (cc, ss) = axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, None)
    torch.cuda.synchronize()
    del d
    compare_full(wl, inp, y, cc, ss)


def test_decode_workload_every_element(cuda_lib):
    """128-token prefill, then 512 cached steps: every (step, b, e) output, the
    prefill's outputs and the final caches against the oracle over 640 tokens."""
    wl = W.WORKLOAD_BY_NAME["decode"]
    inp = W.make_inputs(wl)
    steps = W.make_decode_inputs(wl, wl.decode_steps)
    d = to_dev(inp)
    ds = to_dev(steps)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    y0, cache = axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, None)
    ys = torch.empty(wl.decode_steps, wl.B, wl.E, dtype=wl.torch_io, device="cuda")
    for s in range(wl.decode_steps):
        axon_ssm.step(ds["x"][s], ds["z"][s], ds["dt_raw"][s], ds["B"][s], ds["C"][s], params,
                      cache, y=ys[s])
    torch.cuda.synchronize()
    del ds, d
    # the oracle sees one sequence of 128 + 512 tokens per batch row
    full = dict(inp)
    for k in ("x", "z", "dt_raw", "B", "C"):
        full[k] = torch.cat([inp[k], steps[k].transpose(0, 1)], dim=1)
    y_all = torch.cat([y0, ys.transpose(0, 1)], dim=1)            # (B, 640, E) on the device
    wl_full = W.Workload(wl.name, wl.B, wl.L + wl.decode_steps, wl.E, wl.io, wl.seed)
    compare_full(wl_full, full, y_all, cache[0], cache[1])
