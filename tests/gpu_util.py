"""Helpers shared by the GPU parity tests: device copies, canary-guarded output
buffers, oracle comparison with the stated tolerances.

Tolerances (stated in the measurement plan, read elementwise against the fp64
oracle run on the same bf16-rounded inputs):
  fp32 outputs:  |y_gpu - y_ref| <= 1e-4 * (1 + |y_ref|)
  bf16 outputs:  |y_gpu - y_ref| <= 2e-2 * max(1, |y_ref|)
  ssm_state (always fp32): 1e-4 * (1 + |h_ref|)
  conv_cache: bit-exact (it is a copy of raw inputs)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from selective_state_space_52_b200 import axon_ssm
from selective_state_space_52_b200 import workloads as W

CANARY_BYTES = 256
CANARY_BYTE = 0xA5


def tol_for(io: str, ref: np.ndarray) -> np.ndarray:
    if io == "f32":
        return 1e-4 * (1.0 + np.abs(ref))
    return 2e-2 * np.maximum(1.0, np.abs(ref))


def state_tol(ref: np.ndarray) -> np.ndarray:
    return 1e-4 * (1.0 + np.abs(ref))


def check_close(got, ref, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bad = err > tol
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} elements out of tolerance; "
                             f"worst at {i}: got {got[i]!r} ref {ref[i]!r} tol {tol[i]!r}")
    denom = np.linalg.norm(ref) or 1.0
    return {"max_abs": float(err.max(initial=0.0)), "rel_norm": float(np.linalg.norm(got - ref) / denom)}


class Guarded:
    """A device tensor with canary bytes before and after it (out-of-bounds write check)."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        n = int(np.prod(shape)) if len(shape) else 1
        esize = torch.empty((), dtype=dtype).element_size()
        self.nbytes = n * esize
        self.raw = torch.full((CANARY_BYTES * 2 + self.nbytes,), CANARY_BYTE, dtype=torch.uint8,
                              device=device)
        self.t = self.raw[CANARY_BYTES:CANARY_BYTES + self.nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)
        else:
            self.t.fill_(float("nan"))

    def canaries_intact(self) -> bool:
        head = self.raw[:CANARY_BYTES]
        tail = self.raw[CANARY_BYTES + self.nbytes:]
        return bool(torch.all(head == CANARY_BYTE).item() and torch.all(tail == CANARY_BYTE).item())


def to_dev(inp: dict, device="cuda") -> dict:
    return {k: (v.to(device).contiguous() if v is not None else None) for k, v in inp.items()}


def run_gpu_scan(inp_cpu: dict, num_segments=None, with_state=True, guarded=True, runs=None,
                 discretization="first_order"):
    """Run the CUDA prefill on `inp_cpu` (a workloads dict); returns numpy outputs."""
    d = to_dev(inp_cpu)
    x = d["x"]
    Bsz, L, E = x.shape
    K = d["conv_w"].shape[1]
    N = d["A_log"].shape[1]
    params = {k: d[k] for k in axon_ssm.PARAM_KEYS}
    cache = (d["conv_cache"], d["ssm_state"]) if with_state and "conv_cache" in d else None
    gy = Guarded((Bsz, L, E), x.dtype)
    gcc = Guarded((Bsz, K - 1, E), x.dtype)
    gss = Guarded((Bsz, E, N), torch.float32)
    y, (cc, ss) = axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, cache,
                                    num_segments=num_segments, out=(gy.t, gcc.t, gss.t), runs=runs,
                                    discretization=discretization)
    torch.cuda.synchronize()
    if guarded:
        for g, name in ((gy, "y"), (gcc, "conv_cache"), (gss, "ssm_state")):
            assert g.canaries_intact(), f"out-of-bounds write next to {name}"
    return (y.float().cpu().numpy(), cc.cpu(), ss.cpu().numpy())


def oracle_scan(inp_cpu: dict, with_state=True, zoh=False):
    cc = inp_cpu.get("conv_cache") if with_state else None
    ss = inp_cpu.get("ssm_state") if with_state else None
    return oracle.scan_fwd(inp_cpu["x"], inp_cpu["z"], inp_cpu["dt_raw"], inp_cpu["B"],
                           inp_cpu["C"], inp_cpu["conv_w"], inp_cpu["conv_b"],
                           inp_cpu["dt_bias"], inp_cpu["A_log"], inp_cpu["D"], cc, ss, zoh=zoh)


def compare_scan(inp_cpu: dict, io: str, num_segments=None, with_state=True, what="", runs=None,
                 zoh=False):
    y, cc, ss = run_gpu_scan(inp_cpu, num_segments=num_segments, with_state=with_state, runs=runs,
                             discretization="zoh" if zoh else "first_order")
    y_ref, cc_ref, ss_ref = oracle_scan(inp_cpu, with_state=with_state, zoh=zoh)
    stats = check_close(y, y_ref, tol_for(io, y_ref), what + " y")
    check_close(ss, ss_ref, state_tol(ss_ref), what + " ssm_state")
    # conv cache: bit-exact copy of raw inputs
    cc_ref_t = torch.from_numpy(cc_ref).to(cc.dtype)
    assert torch.equal(cc, cc_ref_t), what + " conv_cache not bit-exact"
    return stats
