"""A sequence split by time across ranks, with one exchange of per-slice
summaries (the chunked associative scan of the SSD article, with devices as
the blocks; the Axon-SSM recurrence decays a run of tokens by exp(A * sum dt)).

Rank r holds tokens [r*L/P, (r+1)*L/P) of every input: x, z, dt_raw (B,Ls,E)
and B, C (B,Ls,N), with Ls >= K-1.  The protocol (include/axon_ssm.h describes
the same steps at the C level):

  1. all-gather every slice's last K-1 inputs: slice r's conv cache is slice
     r-1's tail (slice 0 uses the sequence's own conv cache);
  2. first pass: slice 0 scans from the sequence's initial state -- its y and
     end state are final; slice r >= 1 runs a state-only scan from a zero
     state for its end state h_loc_r and the sum of its dt
     (axon_ssm_scan_state; or a full scan and axon_ssm_dt_sum);
  3. all-gather the (h_loc, dt_sum) pairs;
  4. slice r >= 1 folds them into its entering state (axon_ssm_carry_fold) and
     scans again from it: its y and end caches are final.

The same phases run either across ranks of a torch.distributed process group
(``sharded_scan_fwd``, one all-gather per exchange, the same collective steps
in the same order on every rank) or one after another on one device
(``sliced_scan_local``).  The per-slice operations are this package's CUDA entry
points unless ``ops`` supplies others.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch


@dataclass
class SliceOps:
    """The per-slice operations: scan(x, z, dt_raw, B, C, params, cache) ->
    (y, (conv_cache, ssm_state)); dt_sum(dt_raw, dt_bias) -> (B,E); fold(r,
    A_log, h_loc_all (P,B,E,N), dt_sum_all (P,B,E)) -> (B,E,N); optionally
    scan_state(x, dt_raw, B, params, cache) -> ((conv_cache, ssm_state),
    dt_sum), the first pass of a slice r >= 1 in one state-only scan."""
    scan: Callable
    dt_sum: Callable
    fold: Callable
    scan_state: Callable | None = None


def cuda_ops() -> SliceOps:
    from . import axon_ssm
    return SliceOps(scan=axon_ssm.scan_fwd, dt_sum=axon_ssm.dt_sum, fold=axon_ssm.carry_fold,
                    scan_state=axon_ssm.scan_state)


def slice_tail(x: torch.Tensor, K: int) -> torch.Tensor:
    """The last K-1 inputs of a slice: the next slice's conv cache."""
    Ls = x.shape[1]
    if Ls < K - 1:
        raise ValueError(f"a slice must hold at least K-1 = {K - 1} tokens, got {Ls}")
    return x[:, Ls - (K - 1):, :].contiguous()


def first_pass(r: int, sl: dict, params: dict, halo, cache0, ops: SliceOps):
    """Phase 2 for slice r: returns (y, caches, h_loc, dt_sum); y is None for
    r >= 1 with a state-only scan (only slice 0's first-pass y is final)."""
    if r == 0:
        y, caches = ops.scan(sl["x"], sl["z"], sl["dt_raw"], sl["B"], sl["C"], params, cache0)
        # the same dtype as every other slice's sum: the exchange gathers equal buffers
        dts = torch.zeros(caches[1].shape[:2], dtype=caches[1].dtype, device=caches[1].device)
        return y, caches, caches[1], dts
    if ops.scan_state is not None:
        try:
            caches, dts = ops.scan_state(sl["x"], sl["dt_raw"], sl["B"], params, (halo, None))
            return None, caches, caches[1], dts
        except Exception as ex:                      # a shape the state-only scan does not take
            if getattr(ex, "status", None) != 2:     # AXON_ERR_UNSUPPORTED
                raise
    y, caches = ops.scan(sl["x"], sl["z"], sl["dt_raw"], sl["B"], sl["C"], params, (halo, None))
    return y, caches, caches[1], ops.dt_sum(sl["dt_raw"], params["dt_bias"])


def second_pass(r: int, sl: dict, params: dict, halo, h_all: torch.Tensor, dts_all: torch.Tensor,
                ops: SliceOps):
    """Phase 4 for slice r >= 1: returns (y, caches)."""
    h_in = ops.fold(r, params["A_log"], h_all, dts_all)
    return ops.scan(sl["x"], sl["z"], sl["dt_raw"], sl["B"], sl["C"], params, (halo, h_in))


def sharded_scan_fwd(sl: dict, params: dict, cache=None, *, group=None, ops: SliceOps | None = None):
    """This rank's slice of a time-split prefill.  ``sl`` holds the slice's x,
    z, dt_raw, B, C; ``cache`` the sequence's initial (conv_cache, ssm_state)
    (read on rank 0 only; None means zeros).  Returns (y, (conv_cache,
    ssm_state)) of the slice; on the last rank the caches are the sequence's."""
    import torch.distributed as dist
    ops = ops or cuda_ops()
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    K = params["conv_w"].shape[1]
    tail = slice_tail(sl["x"], K)
    tails = [torch.empty_like(tail) for _ in range(P)]
    dist.all_gather(tails, tail, group=group)
    halo = tails[r - 1] if r > 0 else None
    y, caches, h_loc, dts = first_pass(r, sl, params, halo, cache, ops)
    h_all = [torch.empty_like(h_loc) for _ in range(P)]
    dts_all = [torch.empty_like(dts) for _ in range(P)]
    dist.all_gather(h_all, h_loc.contiguous(), group=group)
    dist.all_gather(dts_all, dts.contiguous(), group=group)
    if r == 0:
        return y, caches
    return second_pass(r, sl, params, halo, torch.stack(h_all), torch.stack(dts_all), ops)


def sliced_scan_local(slices: list, params: dict, cache=None, ops: SliceOps | None = None):
    """The same protocol over a list of slices on one device, phase by phase.
    Returns the list of (y, caches) per slice."""
    ops = ops or cuda_ops()
    K = params["conv_w"].shape[1]
    tails = [slice_tail(sl["x"], K) for sl in slices]
    firsts = [first_pass(r, sl, params, tails[r - 1] if r > 0 else None, cache, ops)
              for r, sl in enumerate(slices)]
    h_all = torch.stack([f[2] for f in firsts])
    dts_all = torch.stack([f[3] for f in firsts])
    out = [(firsts[0][0], firsts[0][1])]
    for r in range(1, len(slices)):
        out.append(second_pass(r, slices[r], params, tails[r - 1], h_all, dts_all, ops))
    return out
