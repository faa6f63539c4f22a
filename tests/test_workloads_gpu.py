"""The five measured workloads at full size, in the launch configuration the
benchmark times (the library's own plan), checked against the fp64 oracle.

The tiny workload is compared in full.  The large ones are compared on sampled
(b, e) channels over their whole length: channels are independent, so the
oracle computes each sampled channel alone (first, last and block-boundary
channels included).  The decode workload prefills 128 tokens and then runs
512 cached steps; every step's output is checked on the sampled channels.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import axon_ssm
from selective_state_space_52_b200 import workloads as W

from gpu_util import check_close, compare_scan, state_tol, to_dev, tol_for

pytestmark = pytest.mark.gpu


def sample_channels(B, E, n=24, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [(0, 0), (0, E - 1), (B - 1, 0), (B - 1, E - 1), (0, min(127, E - 1)),
             (0, min(128, E - 1)), (B // 2, E // 2)]
    extra = [(int(rng.integers(B)), int(rng.integers(E))) for _ in range(n - len(fixed))]
    return sorted(set(fixed + extra))


def test_tiny_workload_full_compare(cuda_lib):
    wl = W.WORKLOADS[0]
    inp = W.make_inputs(wl)
    compare_scan(inp, wl.io, with_state=False, what=wl.name)


@pytest.mark.parametrize("name", ["bit_axon_layer", "mamba_block", "long_seq"])
def test_prefill_workload_sampled(cuda_lib, name):
    wl = W.WORKLOAD_BY_NAME[name]
    inp = W.make_inputs(wl)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    y, (cc, ss) = axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, None)
    torch.cuda.synchronize()
    chans = sample_channels(wl.B, wl.E, n=16 if name == "long_seq" else 24, seed=wl.seed)
    ref = oracle.scan_channels(inp, chans)
    for i, (b, e) in enumerate(chans):
        yg = y[b, :, e].float().cpu().numpy()
        check_close(yg, ref["y"][i], tol_for(wl.io, ref["y"][i]), f"{name} y[{b},:,{e}]")
        sg = ss[b, e].cpu().numpy()
        check_close(sg, ref["ssm_state"][i], state_tol(ref["ssm_state"][i]), f"{name} state[{b},{e}]")
        ccg = cc[b, :, e].cpu()
        assert torch.equal(ccg, torch.from_numpy(ref["conv_cache"][i]).to(ccg.dtype))
    assert torch.isfinite(y.float()).all()


def test_decode_workload_sampled(cuda_lib):
    wl = W.WORKLOAD_BY_NAME["decode"]
    inp = W.make_inputs(wl)
    steps = W.make_decode_inputs(wl, wl.decode_steps)
    d = to_dev(inp)
    ds = to_dev(steps)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    y0, cache = axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, None)
    chans = sample_channels(wl.B, wl.E, n=12, seed=4)
    ys = []
    idx_b = torch.tensor([b for b, _ in chans], device="cuda")
    idx_e = torch.tensor([e for _, e in chans], device="cuda")
    y = torch.empty(wl.B, wl.E, dtype=wl.torch_io, device="cuda")
    for s in range(wl.decode_steps):
        axon_ssm.step(ds["x"][s], ds["z"][s], ds["dt_raw"][s], ds["B"][s], ds["C"][s], params,
                      cache, y=y)
        ys.append(y[idx_b, idx_e].float())
    torch.cuda.synchronize()
    ys = torch.stack(ys, dim=1).cpu().numpy()          # (channels, steps)
    # oracle: the prefill followed by the steps is one sequence of 128 + 512 tokens
    full = dict(inp)
    for k in ("x", "z", "dt_raw", "B", "C"):
        full[k] = torch.cat([inp[k], steps[k].transpose(0, 1)], dim=1)
    ref = oracle.scan_channels(full, chans)
    y0c = y0[idx_b, :, idx_e].float().cpu().numpy()
    for i, (b, e) in enumerate(chans):
        r = ref["y"][i]
        check_close(y0c[i], r[:wl.L], tol_for(wl.io, r[:wl.L]), f"decode prefill [{b},{e}]")
        check_close(ys[i], r[wl.L:], tol_for(wl.io, r[wl.L:]), f"decode steps [{b},{e}]")
        sg = cache[1][b, e].cpu().numpy()
        check_close(sg, ref["ssm_state"][i], state_tol(ref["ssm_state"][i]), f"decode state [{b},{e}]")
        assert torch.equal(cache[0][b, :, e].cpu(),
                           torch.from_numpy(ref["conv_cache"][i]).to(cache[0].dtype))
