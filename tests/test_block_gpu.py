"""GPU parity of the whole Axon-SSM layer (axon_ssm_block_fwd: input projection,
conv stage, projection to dt/B/C, fused scan, output projection) against the
fp64 oracle's ``block_fwd`` on the same bf16 inputs and weights.

Tolerance.  The layer stores its intermediates x, z, u, dt_raw, B, C and y in
bf16 between stages (relative rounding up to 2^-9); the plain fp64 oracle does
not round them.  Simulating those roundings in fp64 (the oracle's
``bf16_intermediates``) moves the output and state by 0.1-0.4% normwise but by
up to 9% of scale for isolated state elements (heavy-tailed: a rounded dt
changes a long-memory state's whole history).  So the GPU is checked two ways:
  * against the oracle with the same bf16 roundings, elementwise
    |got - ref| <= 1e-2 * max(rms(ref), |ref|): what remains is float32 against
    fp64 arithmetic and the rare intermediate whose bf16 rounding flips because
    the GEMM accumulated in float32;
  * against the plain fp64 oracle, normwise ||got - ref|| / ||ref|| <= 1e-2.
Applied to the output, the final state and the final conv cache (the last rows
of x, stored in bf16).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import workloads as W

from gpu_util import to_dev

pytestmark = pytest.mark.gpu


def block_close(got, ref_rounded, ref_plain, what, elem_tol=1e-2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref_rounded, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what + ": non-finite"
    scale = max(float(np.sqrt(np.mean(ref ** 2))), 1e-30)
    err = np.abs(got - ref) / np.maximum(scale, np.abs(ref))
    assert err.max() <= elem_tol, (f"{what}: {int((err > elem_tol).sum())} of {err.size} elements beyond "
                                   f"{elem_tol:.0%} of scale against the bf16-rounding oracle; "
                                   f"worst {float(err.max()):.3g}")
    plain = np.asarray(ref_plain, dtype=np.float64)
    rel = np.linalg.norm(got - plain) / max(np.linalg.norm(plain), 1e-30)
    assert rel <= 1e-2, f"{what}: normwise error {rel:.3g} against the plain fp64 oracle"
    return float(err.max()), rel


def run_block(inp, with_state):
    from selective_state_space_52_b200 import axon_ssm
    d = to_dev(inp)
    weights = {k: d[k] for k in axon_ssm.WEIGHT_KEYS}
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cache = (d["conv_cache"], d["ssm_state"]) if with_state else None
    out, (cc, ss) = axon_ssm.block_fwd(d["X"], weights, params, cache)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), cc.float().cpu().numpy(), ss.cpu().numpy()


def ref_block(inp, with_state, bf16_intermediates):
    return oracle.block_fwd(inp["X"], inp["W_in"], inp["W_x"], inp["W_out"], inp["conv_w"],
                            inp["conv_b"], inp["dt_bias"], inp["A_log"], inp["D"],
                            inp["conv_cache"] if with_state else None,
                            inp["ssm_state"] if with_state else None,
                            bf16_intermediates=bf16_intermediates)


def check_block(inp, with_state, what, elem_tol=1e-2):
    got = run_block(inp, with_state)
    rounded = ref_block(inp, with_state, True)
    plain = ref_block(inp, with_state, False)
    for name, g, r, p in zip(("out", "ssm_state", "conv_cache"), (got[0], got[2], got[1]),
                             (rounded[0], rounded[2], rounded[1]), (plain[0], plain[2], plain[1])):
        block_close(g, r, p, f"{what} {name}", elem_tol)


@pytest.mark.parametrize("with_state", [False, True])
def test_small_block(cuda_lib, with_state):
    bw = W.BLOCK_WORKLOAD_BY_NAME["small_block"]
    inp = W.make_block_inputs(bw, with_state=True)
    check_block(inp, with_state, "small block")


def test_block_on_cta_pairs_ragged_rows(cuda_lib):
    """A layer tall enough for the CTA-pair GEMM (M = B*L = 600: two full
    256-row tiles and a ragged one), with fewer tiles than pairs in every
    projection, so all three run the stream-K split (tiles shared by several
    pairs, partials added by their owners); small widths keep the oracle quick."""
    bw = W.BLOCK_WORKLOAD_BY_NAME["small_block"]
    inp = W.make_block_inputs(bw, with_state=True, L=300)
    check_block(inp, True, "small block, 600 rows")


def test_bit_axon_block_full_width(cuda_lib):
    """The Bit-Axon layer's widths (D 2560, E 7680) on a short sequence."""
    bw = W.BLOCK_WORKLOAD_BY_NAME["bit_axon_block"]
    inp = W.make_block_inputs(bw, with_state=True, L=48)
    check_block(inp, True, "bit-axon block")


def test_bit_axon_block_full_size(cuda_lib):
    """The Bit-Axon layer at the measured size (B1 L2048 D2560 E7680): every
    projection runs several waves of persistent tiles, with a partial last
    wave.  Elementwise bound 2% of scale against the bf16-rounding oracle:
    over 2048 x 7680 stored intermediates a few land, in float32, on the other
    side of a bf16 rounding boundary than in fp64 (one bf16 ulp each), and one
    such flip in a long-memory channel moves that token's y, which the output
    projection spreads over the whole output row -- measured: 11 of 5.2 M
    outputs above 1%, worst 1.37%, all in one token row, the same whether or
    not the projections' last wave was split over the SMs.  The normwise bound
    against the plain fp64 oracle stays 1%."""
    bw = W.BLOCK_WORKLOAD_BY_NAME["bit_axon_block"]
    inp = W.make_block_inputs(bw, with_state=True)
    check_block(inp, True, "bit-axon block, full size", elem_tol=2e-2)


def test_block_empty_sequence_copies_caches(cuda_lib):
    bw = W.BLOCK_WORKLOAD_BY_NAME["small_block"]
    inp = W.make_block_inputs(bw, with_state=True, L=0)
    out, cc, ss = run_block(inp, True)
    assert out.shape == (bw.B, 0, bw.Dm)
    np.testing.assert_array_equal(cc, inp["conv_cache"].float().numpy())
    np.testing.assert_array_equal(ss, inp["ssm_state"].numpy())


def test_back_to_back_layer_calls_share_a_workspace(cuda_lib):
    """Three layer calls enqueued back to back on one stream with one shared
    workspace and no synchronisation between them (inputs A, B, then A again;
    CTA-pair projections with the stream-K split, kernels chained by
    programmatic dependent launch): the two A outputs agree bit for bit and
    B's matches B run on its own, so no kernel reads its inputs early or sees
    flags or partial sums left by the call before."""
    from selective_state_space_52_b200 import axon_ssm
    bw = W.BLOCK_WORKLOAD_BY_NAME["small_block"]
    ia = to_dev(W.make_block_inputs(bw, with_state=True, L=300))
    ib = to_dev(W.make_block_inputs(dataclasses.replace(bw, seed=bw.seed + 101), with_state=True, L=300))

    def call(d, ws):
        weights = {k: d[k] for k in axon_ssm.WEIGHT_KEYS}
        params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
        return axon_ssm.block_fwd(d["X"], weights, params, (d["conv_cache"], d["ssm_state"]), workspace=ws,
                                  check=False)

    E, N, K, Dm = bw.E, bw.N, bw.K, bw.Dm
    ws = torch.empty(axon_ssm.axon_ssm_block_workspace_bytes(bw.B, 300, Dm, E, N, K), dtype=torch.uint8,
                     device="cuda")
    outs = [call(d, ws) for d in (ia, ib, ia)]
    torch.cuda.synchronize()
    assert axon_ssm.block_error_flag(ws) == 0
    (a1, (ca1, sa1)), (b1, (cb1, sb1)), (a2, (ca2, sa2)) = outs
    assert torch.equal(a1.view(torch.int16), a2.view(torch.int16))
    assert torch.equal(sa1, sa2) and torch.equal(ca1.view(torch.int16), ca2.view(torch.int16))
    ws2 = torch.empty_like(ws)
    b2, (cb2, sb2) = call(ib, ws2)
    torch.cuda.synchronize()
    assert torch.equal(b1.view(torch.int16), b2.view(torch.int16))
    assert torch.equal(sb1, sb2) and torch.equal(cb1.view(torch.int16), cb2.view(torch.int16))
