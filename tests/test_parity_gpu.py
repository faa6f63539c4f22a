"""GPU parity: the CUDA prefill and decode step (through the C ABI) against the
fp64 oracle, element by element, on seeded inputs.

Small cases span several CUDA blocks and ragged tails; full-size workloads are
checked on sampled channels (channels are independent, so the oracle can
compute any one of them alone).  Tolerances are in tests/gpu_util.py.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import workloads as W

from gpu_util import (Guarded, check_close, compare_scan, oracle_scan, run_gpu_scan, state_tol,
                      to_dev, tol_for)

pytestmark = pytest.mark.gpu

SWEEP_L = [1, 2, 3, 4, 5, 63, 64, 65, 127, 257, 1000]
SWEEP_BE = [(1, 8), (3, 40), (2, 264)]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E", SWEEP_BE)
@pytest.mark.parametrize("L", SWEEP_L)
def test_sweep_small_shapes(cuda_lib, io, B, E, L):
    wl = W.custom(B, L, E, io=io, seed=1000 + 7 * L + E + B)
    with_state = (L + E) % 2 == 0
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, with_state=with_state, what=f"B{B} L{L} E{E} {io}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E", SWEEP_BE)
@pytest.mark.parametrize("L", [1, 5, 63, 257, 1000, 3001])
def test_chunked_kernel_small_shapes(cuda_lib, io, B, E, L):
    """The unsplit chunked kernel (num_segments=1) on tiny channel tiles with
    16-byte windows that start mid-chunk, several chunks and ragged tails."""
    wl = W.custom(B, L, E, io=io, seed=3000 + L + E + B)
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, num_segments=1, with_state=(L % 2 == 1), what=f"chunked B{B} L{L} E{E} {io}")


# Shapes that steer the first-order planner to each unsplit kernel on a
# 148-SM B200: the split-chunk quadrant scan with 8 runs per chunk below 20
# channels per SM, the eighths scan from 20 to 47, the split-chunk scan with
# one run per chunk from 48 to 511, the direct walk (one thread per channel)
# above.  (The exact-ZOH planner keeps the eighths / quadrant / run-split
# chunked kernels; tests/test_zoh_gpu.py covers it.)
PLANNER_SHAPES = [
    (1, 1000, 300),     # 6.8 channels per SM, fp32 tail tile: split-chunk, 8 runs
    (1, 7680, 200),     # 52 channels per SM: split-chunk, 1 run
    (2, 2048, 300),     # 28 channels per SM: eighths scan
    (1, 1096, 200),     # 7.4 channels per SM: split-chunk, 8 runs
    (1, 1600, 200),     # 10.8 channels per SM: split-chunk, 8 runs
    (1, 14800, 100),    # 100 channels per SM: split-chunk, 1 run
    (1, 29600, 40),     # 200 channels per SM: split-chunk, 1 run
    (8, 4800, 40),      # 259 channels per SM: split-chunk, 1 run
    (16, 4800, 24),     # 519 channels per SM: direct walk
]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E,L", PLANNER_SHAPES)
def test_chunked_kernel_planner_shapes(cuda_lib, io, B, E, L):
    wl = W.custom(B, L, E, io=io, seed=4000 + E + L)
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, num_segments=1, with_state=True, what=f"planner B{B} E{E} L{L} {io}")


# The quadrant scan (one warp per 8 channels, chunks of 32 tokens): single
# tokens, ragged last chunks, several batch rows, both ends of its planner range.
QUAD_SHAPES = [
    (1, 7680, 1), (1, 7680, 33), (1, 7680, 257), (2, 3584, 100), (3, 2400, 65), (1, 37000, 40),
    (8, 9440, 20),
]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E,L", QUAD_SHAPES)
def test_quadrant_scan_shapes(cuda_lib, io, B, E, L):
    wl = W.custom(B, L, E, io=io, seed=4500 + E + L)
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, with_state=(L % 2 == 1), what=f"quad B{B} E{E} L{L} {io}")


# The eighths scan (one warp per 4 channels, two states per lane).
OCTO_SHAPES = [(1, 4096, 1), (1, 4096, 33), (1, 4096, 257), (2, 2048, 100), (1, 3072, 65), (3, 2000, 40),
               (1, 1800, 130)]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E,L", OCTO_SHAPES)
def test_eighths_scan_shapes(cuda_lib, io, B, E, L):
    wl = W.custom(B, L, E, io=io, seed=4800 + E + L)
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, with_state=(L % 2 == 1), what=f"octo B{B} E{E} L{L} {io}")


@pytest.mark.parametrize("B,E,L", [(1, 7684, 97), (2, 3596, 40)])
def test_quadrant_scan_fp32_tail_tile(cuda_lib, B, E, L):
    """E % 8 == 4 (fp32 only): the last warp of every batch row owns 4 channels."""
    inp = W.make_inputs(W.custom(B, L, E, io="f32", seed=4600 + E), with_state=True)
    compare_scan(inp, "f32", what=f"quad tail B{B} E{E} L{L}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("E", [7680, 4096])
def test_warp_scans_continue_in_place(cuda_lib, io, E):
    """Streaming prefill on a quadrant-scan (E 7680) and an eighths-scan (E
    4096) shape with the caches updated in place: scan(0:1), scan(1:3),
    scan(3:40), scan(40:100) == one scan."""
    from selective_state_space_52_b200 import axon_ssm
    wl = W.custom(1, 100, E, io=io, seed=4700 + E)
    inp = W.make_inputs(wl, with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cc, ss = d["conv_cache"].clone(), d["ssm_state"].clone()
    ys = []
    for lo, hi in [(0, 1), (1, 3), (3, 40), (40, 100)]:
        sl = {k: d[k][:, lo:hi].contiguous() for k in ("x", "z", "dt_raw", "B", "C")}
        y = torch.empty_like(sl["x"])
        axon_ssm.scan_fwd(sl["x"], sl["z"], sl["dt_raw"], sl["B"], sl["C"], params, (cc, ss), out=(y, cc, ss))
        ys.append(y)
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1).float().cpu().numpy()
    y_ref, cc_ref, ss_ref = oracle_scan(inp)
    check_close(y, y_ref, tol_for(io, y_ref), "quad streamed y")
    check_close(ss.cpu().numpy(), ss_ref, state_tol(ss_ref), "quad streamed state")
    assert torch.equal(cc.cpu(), torch.from_numpy(cc_ref).to(cc.dtype))


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("L,P", [(64, 2), (257, 3), (1000, 7), (2048, 16), (300, 60), (4096, 64)])
def test_forced_time_split(cuda_lib, io, L, P):
    """The segment-carry path (phase 1 summaries + carry fold + second walk)."""
    if (L + P - 1) // P < 4:
        pytest.skip("segment shorter than the conv window")
    wl = W.custom(2, L, 24 if io == "f32" else 48, io=io, seed=77 + L + P)
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, num_segments=P, what=f"split P={P} L={L} {io}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_split_equals_unsplit_closely(cuda_lib, io):
    wl = W.custom(1, 1024, 64, io=io, seed=5)
    inp = W.make_inputs(wl, with_state=True)
    y1, cc1, ss1 = run_gpu_scan(inp, num_segments=1)
    y8, cc8, ss8 = run_gpu_scan(inp, num_segments=8)
    assert torch.equal(cc1, cc8)
    check_close(y8, y1, tol_for(io, y1), "split vs unsplit")
    check_close(ss8, ss1, state_tol(ss1), "split vs unsplit state")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shift", [-200.0, 200.0, -9.21, 0.0, 4.0, 20.0, 21.0])
def test_dt_clip_edges(cuda_lib, io, shift):
    wl = W.custom(1, 96, 32, io=io, seed=int(abs(shift) * 10) + 3)
    inp = W.make_inputs(wl, with_state=True)
    inp["dt_raw"] = (inp["dt_raw"].float() * 0.01 + shift).to(inp["dt_raw"].dtype)
    compare_scan(inp, io, what=f"dt shift {shift}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_bimodal_dt_long_and_fast_memory(cuda_lib, io):
    wl = W.Workload("bimodal_small", 2, 777, 40, io, 9, dt_mode="bimodal", params="random")
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, what="bimodal")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_empty_sequence_copies_caches(cuda_lib, io):
    wl = W.custom(2, 0, 16, io=io, seed=3)
    inp = W.make_inputs(wl, with_state=True)
    y, cc, ss = run_gpu_scan(inp)
    assert y.shape == (2, 0, 16)
    assert torch.equal(cc, inp["conv_cache"])
    np.testing.assert_array_equal(ss, inp["ssm_state"].numpy())
    y, cc, ss = run_gpu_scan(inp, with_state=False)
    assert torch.all(cc.float() == 0) and np.all(ss == 0)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("P", [1, 4])
def test_in_place_caches(cuda_lib, io, P):
    """conv_cache_out / ssm_state_out may be the input buffers themselves."""
    from selective_state_space_52_b200 import axon_ssm
    wl = W.custom(2, 512, 40, io=io, seed=41 + P)
    inp = W.make_inputs(wl, with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cc, ss = d["conv_cache"].clone(), d["ssm_state"].clone()
    y = torch.empty_like(d["x"])
    axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, (cc, ss),
                      num_segments=P, out=(y, cc, ss))
    torch.cuda.synchronize()
    y_ref, cc_ref, ss_ref = oracle_scan(inp)
    check_close(y.float().cpu().numpy(), y_ref, tol_for(io, y_ref), "in-place y")
    check_close(ss.cpu().numpy(), ss_ref, state_tol(ss_ref), "in-place state")
    assert torch.equal(cc.cpu(), torch.from_numpy(cc_ref).to(cc.dtype))


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_chunked_prefill_continues_exactly(cuda_lib, io):
    """scan(L1) then scan(L - L1) with the returned caches == one scan over L
    (the streaming pattern of the wiki page "Selective State Space Models")."""
    from selective_state_space_52_b200 import axon_ssm
    wl = W.custom(2, 700, 32, io=io, seed=61)
    inp = W.make_inputs(wl, with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cache = (d["conv_cache"], d["ssm_state"])
    ys = []
    for lo, hi in [(0, 1), (1, 3), (3, 300), (300, 700)]:
        sl = {k: d[k][:, lo:hi].contiguous() for k in ("x", "z", "dt_raw", "B", "C")}
        y, cache = axon_ssm.scan_fwd(sl["x"], sl["z"], sl["dt_raw"], sl["B"], sl["C"], params, cache)
        ys.append(y)
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1).float().cpu().numpy()
    y_ref, cc_ref, ss_ref = oracle_scan(inp)
    check_close(y, y_ref, tol_for(io, y_ref), "chunked y")
    check_close(cache[1].cpu().numpy(), ss_ref, state_tol(ss_ref), "chunked state")
    assert torch.equal(cache[0].cpu(), torch.from_numpy(cc_ref).to(cache[0].dtype))


def _run_steps(d, params, cache, steps_inp, guarded_y=True):
    from selective_state_space_52_b200 import axon_ssm
    ys = []
    S = steps_inp["x"].shape[0]
    for s in range(S):
        xs = {k: steps_inp[k][s] for k in ("x", "z", "dt_raw", "B", "C")}
        if guarded_y:
            g = Guarded(tuple(xs["x"].shape), xs["x"].dtype)
            y = axon_ssm.step(xs["x"], xs["z"], xs["dt_raw"], xs["B"], xs["C"], params, cache, y=g.t)
            torch.cuda.synchronize()
            assert g.canaries_intact()
        else:
            y = axon_ssm.step(xs["x"], xs["z"], xs["dt_raw"], xs["B"], xs["C"], params, cache)
        ys.append(y.float().cpu().numpy())
    return np.stack(ys)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E", [(1, 8), (3, 40), (5, 264)])
def test_decode_steps_equal_full_prefill(cuda_lib, io, B, E):
    """prefill(L0) + (L - L0) cached steps on the GPU == oracle prefill over L."""
    from selective_state_space_52_b200 import axon_ssm
    L0, L = 13, 29
    wl = W.custom(B, L, E, io=io, seed=500 + E)
    inp = W.make_inputs(wl, with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    y0, cache = axon_ssm.scan_fwd(*(d[k][:, :L0].contiguous() for k in ("x", "z", "dt_raw", "B", "C")),
                                  params, (d["conv_cache"], d["ssm_state"]))
    steps = {k: d[k][:, L0:].transpose(0, 1).contiguous() for k in ("x", "z", "dt_raw", "B", "C")}
    ys = _run_steps(d, params, cache, steps)
    y_gpu = np.concatenate([y0.float().cpu().numpy(), ys.transpose(1, 0, 2)], axis=1)
    y_ref, cc_ref, ss_ref = oracle_scan(inp)
    check_close(y_gpu, y_ref, tol_for(io, y_ref), "decode y")
    check_close(cache[1].cpu().numpy(), ss_ref, state_tol(ss_ref), "decode state")
    assert torch.equal(cache[0].cpu(), torch.from_numpy(cc_ref).to(cache[0].dtype))


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_step_matches_oracle_step(cuda_lib, io):
    from selective_state_space_52_b200 import axon_ssm
    wl = W.custom(7, 1, 136, io=io, seed=88)
    inp = W.make_inputs(wl, with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cc, ss = d["conv_cache"].clone(), d["ssm_state"].clone()
    y = axon_ssm.step(d["x"][:, 0].contiguous(), d["z"][:, 0].contiguous(),
                      d["dt_raw"][:, 0].contiguous(), d["B"][:, 0].contiguous(),
                      d["C"][:, 0].contiguous(), params, (cc, ss))
    torch.cuda.synchronize()
    y_ref, cc_ref, ss_ref = oracle.step(inp["x"][:, 0], inp["z"][:, 0], inp["dt_raw"][:, 0],
                                        inp["B"][:, 0], inp["C"][:, 0], inp["conv_w"],
                                        inp["conv_b"], inp["dt_bias"], inp["A_log"], inp["D"],
                                        inp["conv_cache"], inp["ssm_state"])
    check_close(y.float().cpu().numpy(), y_ref, tol_for(io, y_ref), "step y")
    check_close(ss.cpu().numpy(), ss_ref, state_tol(ss_ref), "step state")
    assert torch.equal(cc.cpu(), torch.from_numpy(cc_ref).to(cc.dtype))


# Decode blocks that walk several rounds of four rows and end on a partial one
# (B = 30: blocks of 12 rows, the last with 6; B = 50 with E % 32 == 8: a
# channel tail in every round), through the occupancy-sized row plan.
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("B,E", [(30, 4096), (50, 2056)])
def test_step_multi_round_blocks(cuda_lib, io, B, E):
    from selective_state_space_52_b200 import axon_ssm
    wl = W.custom(B, 1, E, io=io, seed=91 + B)
    inp = W.make_inputs(wl, with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cc, ss = d["conv_cache"].clone(), d["ssm_state"].clone()
    y = axon_ssm.step(*(d[k][:, 0].contiguous() for k in ("x", "z", "dt_raw", "B", "C")), params, (cc, ss))
    torch.cuda.synchronize()
    y_ref, cc_ref, ss_ref = oracle.step(inp["x"][:, 0], inp["z"][:, 0], inp["dt_raw"][:, 0],
                                        inp["B"][:, 0], inp["C"][:, 0], inp["conv_w"],
                                        inp["conv_b"], inp["dt_bias"], inp["A_log"], inp["D"],
                                        inp["conv_cache"], inp["ssm_state"])
    check_close(y.float().cpu().numpy(), y_ref, tol_for(io, y_ref), "step y")
    check_close(ss.cpu().numpy(), ss_ref, state_tol(ss_ref), "step state")
    assert torch.equal(cc.cpu(), torch.from_numpy(cc_ref).to(cc.dtype))


# The split-chunk quadrant scan with each number of runs per chunk (W warps per
# 8 channels; W = 1: runs of 32 tokens, else 16): single tokens, ragged runs
# and chunks, chunks whose last runs lie wholly past L, several batch rows, an
# fp32 tail tile (E % 8 == 4), both discretisations.
QSPLIT_SHAPES = [(1, 64, 1), (1, 64, 17), (2, 40, 100), (1, 2048, 300), (3, 24, 515), (1, 16, 2049)]


@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("runs", [1, 2, 4, 8])
@pytest.mark.parametrize("B,E,L", QSPLIT_SHAPES)
def test_split_chunk_scan_shapes(cuda_lib, runs, io, zoh, B, E, L):
    wl = W.custom(B, L, E, io=io, seed=5100 + 3 * E + L + runs)
    inp = W.make_inputs(wl, with_state=True)
    compare_scan(inp, io, with_state=(L % 2 == 1), runs=runs, zoh=zoh,
                 what=f"qsplit W{runs} B{B} E{E} L{L} {io} zoh={zoh}")


@pytest.mark.parametrize("runs", [1, 2, 8])
def test_split_chunk_scan_fp32_tail_tile(cuda_lib, runs):
    inp = W.make_inputs(W.custom(2, 77, 36, io="f32", seed=5200 + runs), with_state=True)
    compare_scan(inp, "f32", runs=runs, what=f"qsplit tail W{runs}")


@pytest.mark.parametrize("runs", [1, 4])
def test_split_chunk_scan_in_place_caches(cuda_lib, runs):
    from selective_state_space_52_b200 import axon_ssm
    inp = W.make_inputs(W.custom(1, 333, 64, io="bf16", seed=5300 + runs), with_state=True)
    d = to_dev(inp)
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cc, ss = d["conv_cache"].clone(), d["ssm_state"].clone()
    y = torch.empty_like(d["x"])
    axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, (cc, ss), out=(y, cc, ss),
                      runs=runs)
    torch.cuda.synchronize()
    y_ref, cc_ref, ss_ref = oracle_scan(inp)
    check_close(y.float().cpu().numpy(), y_ref, tol_for("bf16", y_ref), "qsplit in-place y")
    check_close(ss.cpu().numpy(), ss_ref, state_tol(ss_ref), "qsplit in-place state")
    assert torch.equal(cc.cpu(), torch.from_numpy(cc_ref).to(cc.dtype))
