"""GPU parity of the time-split pieces: axon_ssm_dt_sum and axon_ssm_carry_fold
against numpy in fp64, and the whole protocol (shard.sliced_scan_local: every
slice's first pass, the fold, the second pass, with the CUDA operations) over
2-4 slices of one sequence against the oracle's scan of the whole sequence,
with the scan's tolerances (tests/gpu_util.py)."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import workloads as W

from gpu_util import check_close, state_tol, to_dev, tol_for

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_dt_sum_matches_numpy(cuda_lib, io):
    from selective_state_space_52_b200 import axon_ssm
    inp = W.make_inputs(W.custom(3, 1000, 264, io=io, seed=95))
    d = to_dev(inp)
    got = axon_ssm.dt_sum(d["dt_raw"], d["dt_bias"]).cpu().double().numpy()
    v = inp["dt_raw"].double().numpy() + inp["dt_bias"].double().numpy()
    ref = np.clip(np.logaddexp(0.0, v), 1e-4, 100.0).sum(axis=1)
    np.testing.assert_allclose(got, ref, rtol=2e-5)


def test_carry_fold_matches_numpy(cuda_lib):
    from selective_state_space_52_b200 import axon_ssm
    rng = np.random.default_rng(96)
    P, B, E, N = 5, 2, 40, 16
    h_all = rng.standard_normal((P, B, E, N)).astype(np.float32)
    dts = rng.uniform(0.0, 3.0, (P, B, E)).astype(np.float32)
    A_log = np.log(np.tile(np.arange(1, N + 1, dtype=np.float64), (E, 1))).astype(np.float32)
    for r in range(1, P):
        got = axon_ssm.carry_fold(r, torch.from_numpy(A_log).cuda(), torch.from_numpy(h_all).cuda(),
                                  torch.from_numpy(dts).cuda()).cpu().double().numpy()
        A = -np.exp(A_log.astype(np.float64))
        h = h_all[0].astype(np.float64)
        for j in range(1, r):
            h = np.exp(A * dts[j].astype(np.float64)[..., None]) * h + h_all[j]
        np.testing.assert_allclose(got, h, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E,L,P", [(2, 40, 301, 2), (1, 264, 1000, 3), (1, 7680, 400, 4), (1, 2048, 4096, 4)])
@pytest.mark.parametrize("with_state", [False, True])
def test_time_split_over_slices(cuda_lib, io, B, E, L, P, with_state):
    from selective_state_space_52_b200.shard import sliced_scan_local
    inp = W.make_inputs(W.custom(B, L, E, io=io, seed=9000 + E + P), with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in ("conv_w", "conv_b", "dt_bias", "A_log", "D")}
    cut = [L * r // P for r in range(P + 1)]
    slices = [{k: d[k][:, cut[r]:cut[r + 1]].contiguous() for k in ("x", "z", "dt_raw", "B", "C")}
              for r in range(P)]
    cache = (d["conv_cache"], d["ssm_state"]) if with_state else None
    out = sliced_scan_local(slices, params, cache)
    torch.cuda.synchronize()
    y = np.concatenate([o[0].float().cpu().numpy() for o in out], axis=1)
    cc, ss = out[-1][1]
    y_ref, cc_ref, ss_ref = oracle.scan_fwd(
        inp["x"], inp["z"], inp["dt_raw"], inp["B"], inp["C"], inp["conv_w"], inp["conv_b"],
        inp["dt_bias"], inp["A_log"], inp["D"],
        inp["conv_cache"] if with_state else None, inp["ssm_state"] if with_state else None)
    check_close(y, y_ref, tol_for(io, y_ref), f"slices y B{B} E{E} L{L} P{P} {io}")
    check_close(ss.cpu().numpy(), ss_ref, state_tol(ss_ref), "slices state")
    assert torch.equal(cc.cpu(), torch.from_numpy(cc_ref).to(cc.dtype))


# The state-only first pass (axon_ssm_scan_state): the oracle's final caches
# and the sum of the step sizes, on shapes that take each run count of the
# split-chunk scan (few channels: 8 runs per chunk, many: 1), ragged lengths,
# with and without initial caches, in place, and an empty sequence.
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E,L", [(1, 64, 1), (2, 40, 301), (1, 2048, 1000), (3, 264, 77), (2, 7680, 129),
                                   (64, 7680, 33)])
@pytest.mark.parametrize("with_state", [False, True])
def test_scan_state_matches_oracle(cuda_lib, io, B, E, L, with_state):
    from selective_state_space_52_b200 import axon_ssm
    inp = W.make_inputs(W.custom(B, L, E, io=io, seed=9400 + E + L), with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in ("conv_w", "conv_b", "dt_bias", "A_log", "D")}
    cache = (d["conv_cache"], d["ssm_state"]) if with_state else None
    (cc, ss), dts = axon_ssm.scan_state(d["x"], d["dt_raw"], d["B"], params, cache)
    torch.cuda.synchronize()
    _, cc_ref, ss_ref = oracle.scan_fwd(inp["x"], inp["z"], inp["dt_raw"], inp["B"], inp["C"], inp["conv_w"],
                                        inp["conv_b"], inp["dt_bias"], inp["A_log"], inp["D"],
                                        inp["conv_cache"] if with_state else None,
                                        inp["ssm_state"] if with_state else None, parallel=True)
    check_close(ss.cpu().numpy(), ss_ref, state_tol(ss_ref), "scan_state state")
    assert torch.equal(cc.cpu(), torch.from_numpy(cc_ref).to(cc.dtype))
    v = inp["dt_raw"].double().numpy() + inp["dt_bias"].double().numpy()
    ref = np.clip(np.logaddexp(0.0, v), 1e-4, 100.0).sum(axis=1)
    np.testing.assert_allclose(dts.cpu().double().numpy(), ref, rtol=2e-5)
    # the same bits on a second run (a fixed summation order), and in place
    (cc2, ss2), dts2 = axon_ssm.scan_state(d["x"], d["dt_raw"], d["B"], params, cache)
    assert torch.equal(dts, dts2) and torch.equal(ss, ss2)
    if with_state:
        cci, ssi = d["conv_cache"].clone(), d["ssm_state"].clone()
        Bsz, K, N = B, inp["conv_w"].shape[1], inp["A_log"].shape[1]
        dt3 = torch.empty(B, E, dtype=torch.float32, device="cuda")
        axon_ssm.axon_ssm_scan_state(B, L, E, N, K, 1 if io == "bf16" else 0, d["x"], d["dt_raw"], d["B"],
                                     params["conv_w"], params["conv_b"], params["dt_bias"], params["A_log"],
                                     cci, ssi, cci, ssi, dt3)
        torch.cuda.synchronize()
        assert torch.equal(cci, cc) and torch.equal(ssi, ss) and torch.equal(dt3, dts)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_scan_state_empty_sequence(cuda_lib, io):
    from selective_state_space_52_b200 import axon_ssm
    inp = W.make_inputs(W.custom(2, 0, 40, io=io, seed=9500), with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in ("conv_w", "conv_b", "dt_bias", "A_log", "D")}
    (cc, ss), dts = axon_ssm.scan_state(d["x"], d["dt_raw"], d["B"], params, (d["conv_cache"], d["ssm_state"]))
    torch.cuda.synchronize()
    assert torch.equal(cc, d["conv_cache"]) and torch.equal(ss, d["ssm_state"])
    assert torch.count_nonzero(dts).item() == 0
