"""GPU parity of the Mamba-2 (SSD) layer core (axon_ssd_scan_fwd: per-chunk
decays, then chunk walks per (batch row, head, segment of the sequence) with
the products on tcgen05 tensor-core MMAs into tensor memory) against the fp64
oracle's ``ssd_scan`` on the same bf16 inputs, for one segment, forced
segment counts and the automatic plan.

Tolerance: the bf16 output bound, elementwise |got - ref| <= 2e-2 *
max(1, |ref|) per head, and normwise ||got - ref|| / ||ref|| <= 1e-2, for y
and for the final state.  The tensor-core products take bf16 operands: the
decayed chunk Gram matrix M = G_ij exp(acum_i - acum_j) dt_j (plus D on its
diagonal) and the carried state each enter as a hi + lo pair of bf16 parts
(about 16 significant bits), the weighted x rows w_j x_j as one bf16 value,
x itself is exact; accumulation and the carried state are float32.  The
float64 model of these roundings (tests/test_ssd_rounding_model.py) stays
within 0.6 of the bound on the Mamba-2 workload's most cancelling heads.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import workloads as W

pytestmark = pytest.mark.gpu


def close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what + ": non-finite"
    err = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= 2e-2, f"{what}: worst {err.max():.3g} of max(1, |ref|), {int((err > 2e-2).sum())} elements; normwise {rel:.3g}"
    assert rel <= 1e-2, f"{what}: normwise {rel:.3g}"


def run(inp, with_state, segments=0, in_place=False):
    from selective_state_space_52_b200 import axon_ssm
    d = {k: v.cuda() for k, v in inp.items()}
    params = {k: d[k] for k in ("dt_bias", "A_log", "D")}
    h0 = d["h0"] if with_state else None
    out = (torch.empty_like(d["x"]), h0) if in_place else None
    y, h = axon_ssm.ssd_scan(d["x"], d["dt_raw"], d["B"], d["C"], params, h0, out=out, segments=segments)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), h.cpu().numpy()


def ref(inp, with_state):
    return oracle.ssd_scan(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A_log"], inp["B"], inp["C"],
                           inp["D"], inp["h0"] if with_state else None)


@pytest.mark.parametrize("L", [1, 64, 130, 1000])
@pytest.mark.parametrize("with_state", [False, True])
def test_ssd_small(cuda_lib, L, with_state):
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=L)
    y, h = run(inp, with_state)
    y_ref, h_ref = ref(inp, with_state)
    close(y, y_ref, f"ssd y L{L}")
    close(h, h_ref, f"ssd state L{L}")


@pytest.mark.parametrize("segments", [1, 2, 3, 16])
def test_ssd_segments(cuda_lib, segments):
    """The same answer for any cut of the sequence into segments (1000 tokens:
    16 chunks, the last one ragged)."""
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=1000)
    y, h = run(inp, True, segments=segments)
    y_ref, h_ref = ref(inp, True)
    close(y, y_ref, f"ssd y, {segments} segments")
    close(h, h_ref, f"ssd state, {segments} segments")


@pytest.mark.parametrize("segments", [1, 4])
def test_ssd_state_in_place(cuda_lib, segments):
    """h_out = h0: the final state overwrites the initial one, which the walks
    of the first segment read."""
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=520)
    y_ref, h_ref = ref(inp, True)
    y, h = run(inp, True, segments=segments, in_place=True)
    close(y, y_ref, f"ssd y in place, {segments} segments")
    close(h, h_ref, f"ssd state in place, {segments} segments")


def test_ssd_mamba2_heads(cuda_lib):
    """The Mamba-2 block's 64 heads on a sequence of several chunks."""
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["mamba2_ssd"], with_state=True, L=320)
    y, h = run(inp, True)
    y_ref, h_ref = ref(inp, True)
    close(y, y_ref, "mamba2 y")
    close(h, h_ref, "mamba2 state")


def test_ssd_empty_sequence_copies_state(cuda_lib):
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=0)
    y, h = run(inp, True)
    assert y.shape[1] == 0
    np.testing.assert_array_equal(h, inp["h0"].numpy())


def test_ssd_full_size(cuda_lib):
    """The benchmark's shape (B1 L4096, 64 heads, the automatic segment plan,
    as bench.py times it), every output against the oracle."""
    sw = W.SSD_WORKLOAD_BY_NAME["mamba2_ssd"]
    inp = W.make_ssd_inputs(sw, with_state=True)
    for with_state in (False, True):
        y, h = run(inp, with_state)
        y_ref, h_ref = ref(inp, with_state)
        close(y, y_ref, f"mamba2 full-size y, h0 {with_state}")
        close(h, h_ref, f"mamba2 full-size state, h0 {with_state}")


def test_ssd_wait_flag_stays_clear(cuda_lib):
    """The workspace's first 4 bytes are the walk's error flag: every wait for
    a tensor-core product completed, so it reads 0 after the call."""
    from selective_state_space_52_b200 import axon_ssm
    sw = W.SSD_WORKLOAD_BY_NAME["small_ssd"]
    inp = W.make_ssd_inputs(sw, with_state=True, L=1000)
    d = {k: v.cuda() for k, v in inp.items()}
    params = {k: d[k] for k in ("dt_bias", "A_log", "D")}
    nbytes = axon_ssm.axon_ssd_workspace_bytes(sw.B, 1000, sw.H, sw.P, sw.N, 3)
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device="cuda")   # a nonzero flag beforehand
    axon_ssm.ssd_scan(d["x"], d["dt_raw"], d["B"], d["C"], params, d["h0"], workspace=ws, segments=3)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0


def extreme_inputs(L=300):
    """Three heads at the edges of the dt clip: head 0 at the lower bound with
    A = -1 (a memory of ~10^4 tokens), head 1 at the upper bound with A = -16
    (exp(-1600): every token forgets the past), head 2 as drawn; D ~ N(0, 1)."""
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=L)
    g = torch.Generator().manual_seed(23)
    inp["dt_bias"] = torch.tensor([-30.0, 200.0, float(inp["dt_bias"][2])], dtype=torch.float32)
    inp["A_log"] = torch.tensor([0.0, math.log(16.0), float(inp["A_log"][2])], dtype=torch.float32)
    inp["D"] = torch.randn(3, generator=g, dtype=torch.float32)
    return inp


def test_ssd_extreme_decays_per_head(cuda_lib):
    """Both dt clip bounds and a random D, with an initial state, over three
    chunks (the last ragged) and the automatic segment plan; each head is held
    to its own scale."""
    inp = extreme_inputs()
    y, h = run(inp, True)
    y_ref, h_ref = ref(inp, True)
    for hd in range(3):
        close(y[:, :, hd], y_ref[:, :, hd], f"ssd y, extreme head {hd}")
        close(h[:, hd], h_ref[:, hd], f"ssd state, extreme head {hd}")


def test_ssd_wait_gives_up_and_reports(cuda_lib):
    """The walks' failure path: a wait on an mbarrier that nothing arrives on
    gives up after its bounded polls and reports it in the status word, and
    the device stays usable."""
    from selective_state_space_52_b200 import axon_ssm
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    axon_ssm.axon_ssd_wait_probe(status, 64)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    # the device still runs the SSD core afterwards
    test_ssd_small(cuda_lib, 130, True)


def test_ssd_back_to_back_calls_share_a_workspace(cuda_lib):
    """Three SSD calls enqueued back to back on one stream with one shared
    workspace and no synchronisation between them (inputs A, B, then A again;
    three segments, so the state-only walk and the carries run; the kernels
    chained by programmatic dependent launch): the two A results agree bit
    for bit and B's matches B run on its own."""
    import dataclasses
    from selective_state_space_52_b200 import axon_ssm
    sw = W.SSD_WORKLOAD_BY_NAME["small_ssd"]
    da = {k: v.cuda() for k, v in W.make_ssd_inputs(sw, with_state=True, L=1000).items()}
    db = {k: v.cuda() for k, v in W.make_ssd_inputs(dataclasses.replace(sw, seed=sw.seed + 77), with_state=True,
                                                   L=1000).items()}
    nbytes = axon_ssm.axon_ssd_workspace_bytes(sw.B, 1000, sw.H, sw.P, sw.N, 3)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")

    def call(d, w):
        params = {k: d[k] for k in ("dt_bias", "A_log", "D")}
        return axon_ssm.ssd_scan(d["x"], d["dt_raw"], d["B"], d["C"], params, d["h0"], workspace=w, segments=3,
                                 check=False)

    (ya1, ha1), (yb1, hb1), (ya2, ha2) = [call(d, ws) for d in (da, db, da)]
    torch.cuda.synchronize()
    assert axon_ssm.ssd_error_flag(ws) == 0
    assert torch.equal(ya1.view(torch.int16), ya2.view(torch.int16)) and torch.equal(ha1, ha2)
    yb2, hb2 = call(db, torch.empty_like(ws))
    torch.cuda.synchronize()
    assert torch.equal(yb1.view(torch.int16), yb2.view(torch.int16)) and torch.equal(hb1, hb2)
