"""axon_ssm_scan_fwd_noalloc: the prefill whose time-split scratch lives in the
library's own 16 MiB device array instead of a caller workspace.

It exists for callers that cannot allocate device memory themselves -- a
serving process whose pool already reserved nearly all of HBM, or a host loop
that must not call cudaMalloc/cudaFree (they can synchronise the device).
Here it is called through the C ABI three times in a row, on different
inputs, and each result is compared with the existing workspace entry point
(axon_ssm_scan_fwd_segments) and with the fp64 oracle, within the parity
tolerances of the other tests; the later calls also show that the scratch left
behind by an earlier one does not leak into them.  The third call lets the
library choose the split (num_segments = 0) on a shape it splits in time.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from selective_state_space_52_b200 import workloads as W

from gpu_util import check_close, oracle_scan, state_tol, to_dev, tol_for

pytestmark = pytest.mark.gpu


def _run_pair(axon_ssm, inp, num_segments):
    d = to_dev(inp)
    Bsz, L, E = d["x"].shape
    N, K = 16, 4
    io = axon_ssm.AXON_BF16 if d["x"].dtype == torch.bfloat16 else axon_ssm.AXON_F32
    params = [d[k] for k in axon_ssm.PARAM_KEYS]
    seq = [d[k] for k in ("x", "z", "dt_raw", "B", "C")]

    def outs():
        return (torch.empty_like(d["x"]), torch.empty(Bsz, K - 1, E, dtype=d["x"].dtype, device="cuda"),
                torch.empty(Bsz, E, N, dtype=torch.float32, device="cuda"))

    ref = outs()
    ws_bytes = max(num_segments - 1, 0) * Bsz * E * (N + 1) * 4
    if num_segments == 0:
        ws_bytes = axon_ssm.axon_ssm_scan_workspace_bytes(Bsz, L, E, N, K, io)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    axon_ssm.axon_ssm_scan_fwd_segments(Bsz, L, E, N, K, io, *seq, *params,
                                        d["conv_cache"], d["ssm_state"], *ref, ws, ws_bytes,
                                        num_segments)
    got = outs()
    axon_ssm.axon_ssm_scan_fwd_noalloc(Bsz, L, E, N, K, io, *seq, *params,
                                       d["conv_cache"], d["ssm_state"], *got, num_segments)
    torch.cuda.synchronize()
    return ref, got


def _compare(io, ref, got, what, inp):
    y_ref = ref[0].float().cpu().numpy()
    check_close(got[0].float().cpu().numpy(), y_ref, tol_for(io, y_ref), what + " y")
    s_ref = ref[2].cpu().numpy()
    check_close(got[2].cpu().numpy(), s_ref, state_tol(s_ref), what + " ssm_state")
    assert torch.equal(got[1].cpu(), ref[1].cpu()), what + " conv_cache"
    # and against the fp64 oracle on the same inputs
    y_o, cc_o, ss_o = oracle_scan(inp)
    check_close(got[0].float().cpu().numpy(), y_o, tol_for(io, y_o), what + " y vs oracle")
    check_close(got[2].cpu().numpy(), ss_o, state_tol(ss_o), what + " ssm_state vs oracle")
    assert torch.equal(got[1].cpu(), torch.from_numpy(cc_o).to(got[1].dtype)), what + " conv_cache vs oracle"


def test_noalloc_matches_workspace_entry_point_and_oracle_calls_in_a_row(cuda_lib):
    axon_ssm = cuda_lib
    # first call: a long split (16 segments) that fills much of the scratch
    first = W.make_inputs(W.custom(2, 2048, 256, io="bf16", seed=901), with_state=True)
    ref, got = _run_pair(axon_ssm, first, num_segments=16)
    _compare("bf16", ref, got, "no-alloc call 1", first)
    # second call, straight after: other inputs, other split, fp32 io
    second = W.make_inputs(W.custom(1, 1000, 64, io="f32", seed=902), with_state=True)
    ref, got = _run_pair(axon_ssm, second, num_segments=7)
    _compare("f32", ref, got, "no-alloc call 2", second)
    # third call: the library's own plan; 256 channels and 4096 tokens are cut
    # into segments (fewer than four channels per SM, a long sequence)
    assert axon_ssm.axon_ssm_scan_launch_count(1, 4096, 256, 16, 4, axon_ssm.AXON_BF16) == 2
    third = W.make_inputs(W.custom(1, 4096, 256, io="bf16", seed=903), with_state=True)
    ref, got = _run_pair(axon_ssm, third, num_segments=0)
    _compare("bf16", ref, got, "no-alloc call 3 (library split)", third)


def test_noalloc_rejects_scratch_beyond_its_limit(cuda_lib):
    """(64 - 1) * 1 * 4096 * 17 * 4 bytes > 16 MiB: rejected on the host, nothing launched."""
    axon_ssm = cuda_lib
    fake = 1 << 40                        # never dereferenced: the call is rejected first
    ptrs = [fake + 0x100000 * i for i in range(15)]
    rc = axon_ssm._lib.axon_ssm_scan_fwd_noalloc(1, 65536, 4096, 16, 4, axon_ssm.AXON_BF16,
                                                 *ptrs, ctypes.c_int(64), None)
    assert rc == 2                        # AXON_ERR_UNSUPPORTED
    assert axon_ssm.axon_status_string(rc) == "AXON_ERR_UNSUPPORTED"
