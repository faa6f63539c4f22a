"""The error budget behind the SSD GPU tests' tolerance, made checkable on CPU.

A float32 / bf16 model of the arithmetic the SSD walk performs (not its code):
128-token chunks; the decayed Gram matrix M, with D on its diagonal and, below
the diagonal 32-token blocks, the decay factorised as
2^(acum_i - acum_r) * dt_j 2^(acum_r - acum_j) (r the block's last token),
entering M x as a bf16 pair (hi = M rounded, lo = the residual rounded); the
state weights w_j x_j rounded to bf16; the carried state float32, entering
C S^T as a bf16 pair (hi = its top 16 bits, lo = the rest rounded); products
accumulated exactly (float64 here, float32 on the GPU); y rounded to bf16.
Against the fp64 oracle on the GPU tests' inputs this model stays within
half of the bf16 output bound |got - ref| <= 2e-2 max(1, |ref|) elementwise
(0.6 of it on the Mamba-2 workload's most cancelling heads) and 0.5%
normwise per head, so the GPU tests' bound leaves room for float32
accumulation order.  With a single bf16 copy of M, heads of the Mamba-2
workload exceed that bound; with a single bf16 copy of the state instead of
the pair, one small case exceeds 3% of max(rms, |ref|): that is why the
kernel splits both.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_52_b200 import workloads as W

Q, BLK = 128, 32
LOG2E = 1.0 / math.log(2.0)


def bf(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def f32(a):
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def hi_part(a):
    """The top 16 bits of each float32 value (truncation to a bf16 pattern)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return u.view(np.float32).astype(np.float64)


def dt_of(v):
    sp = np.where(v > 20, v, np.log1p(np.exp(np.minimum(v, 20))))
    return np.clip(sp, 1e-4, 100.0)


def model(inp, with_state, split_state=True, split_m=True, heads=None):
    x = inp["x"].float().numpy().astype(np.float64)
    dtr = inp["dt_raw"].float().numpy().astype(np.float64)
    Bm = inp["B"].float().numpy().astype(np.float64)
    Cm = inp["C"].float().numpy().astype(np.float64)
    bias = inp["dt_bias"].numpy().astype(np.float64)
    Alog = inp["A_log"].numpy().astype(np.float64)
    D = inp["D"].numpy().astype(np.float64)
    Bs, L, H, P = x.shape
    N = Bm.shape[2]
    y = np.zeros_like(x)
    hout = np.zeros((Bs, H, P, N))
    for b in range(Bs):
        for h in (range(H) if heads is None else heads):
            A2 = f32(-math.exp(Alog[h]) * LOG2E)
            S = f32(inp["h0"][b, h].numpy()) if with_state else np.zeros((P, N))
            for t0 in range(0, L, Q):
                n = min(Q, L - t0)
                dt = np.zeros(Q)
                dt[:n] = f32(dt_of(dtr[b, t0:t0 + n, h] + bias[h]))
                a = f32(np.cumsum(dt * A2))                       # acum, log2 units
                C = np.zeros((Q, N)); C[:n] = Cm[b, t0:t0 + n]
                Bc = np.zeros((Q, N)); Bc[:n] = Bm[b, t0:t0 + n]
                X = np.zeros((Q, P)); X[:n] = x[b, t0:t0 + n, h]
                G = f32(C @ Bc.T)
                M = np.zeros((Q, Q))
                for ib in range(Q // BLK):
                    rows = slice(BLK * ib, BLK * ib + BLK)
                    i = np.arange(BLK * ib, BLK * ib + BLK)
                    for jb in range(ib + 1):
                        cols = slice(BLK * jb, BLK * jb + BLK)
                        j = np.arange(BLK * jb, BLK * jb + BLK)
                        if jb < ib:
                            r = BLK * jb + BLK - 1
                            u = np.exp2(a[i] - a[r])
                            v = dt[j] * np.exp2(a[r] - a[j])
                            M[rows, cols] = G[rows, cols] * u[:, None] * v[None, :]
                        else:
                            d = np.where(j[None, :] <= i[:, None], np.exp2(np.minimum(a[i][:, None] - a[j][None, :], 0)), 0.0)
                            blk = G[rows, cols] * d * dt[j][None, :]
                            blk[np.arange(BLK), np.arange(BLK)] += D[h]
                            M[rows, cols] = blk
                if split_m:
                    Mh = bf(M)
                    M = Mh + bf(M - Mh)
                else:
                    M = bf(M)
                if split_state:
                    Sh = hi_part(S)
                    Sb = Sh + bf(S - Sh)
                else:
                    Sb = bf(S)
                yq = np.exp2(a)[:, None] * (C @ Sb.T) + M @ X
                y[b, t0:t0 + n, h] = bf(yq[:n])
                w = dt * np.exp2(a[-1] - a)
                S = f32(np.exp2(a[-1]) * S + bf(w[:, None] * X).T @ Bc)
            hout[b, h] = S
    return y, hout


def errors(got, ref):
    """(worst |got - ref| / max(1, |ref|), normwise relative error)"""
    err = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    return float(err.max()), float(rel)


def errors_of_scale(got, ref):
    """worst |got - ref| / max(rms(ref), |ref|)"""
    scale = max(float(np.sqrt(np.mean(ref ** 2))), 1e-30)
    return float((np.abs(got - ref) / np.maximum(scale, np.abs(ref))).max())


def oracle_ref(inp, with_state):
    return oracle.ssd_scan(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A_log"], inp["B"], inp["C"], inp["D"],
                           inp["h0"] if with_state else None)


CASES = [(L, ws) for L in (130, 1000) for ws in (False, True)]


@pytest.mark.parametrize("L,with_state", CASES)
def test_rounding_model_within_budget(L, with_state):
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=L)
    y, h = model(inp, with_state)
    y_ref, h_ref = oracle_ref(inp, with_state)
    for hd in range(y.shape[2]):
        ey, ry = errors(y[:, :, hd], y_ref[:, :, hd])
        eh, rh = errors(h[:, hd], h_ref[:, hd])
        assert ey <= 1e-2 and ry <= 5e-3, (L, with_state, hd, ey, ry)
        assert eh <= 1e-2 and rh <= 5e-3, (L, with_state, hd, eh, rh)


def test_rounding_model_at_the_clip_bounds():
    """The inputs of the GPU test at both dt clip bounds with a random D."""
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=300)
    g = torch.Generator().manual_seed(23)
    inp["dt_bias"] = torch.tensor([-30.0, 200.0, float(inp["dt_bias"][2])], dtype=torch.float32)
    inp["A_log"] = torch.tensor([0.0, math.log(16.0), float(inp["A_log"][2])], dtype=torch.float32)
    inp["D"] = torch.randn(3, generator=g, dtype=torch.float32)
    y, h = model(inp, True)
    y_ref, h_ref = oracle_ref(inp, True)
    for hd in range(3):
        ey, ry = errors(y[:, :, hd], y_ref[:, :, hd])
        eh, rh = errors(h[:, hd], h_ref[:, hd])
        assert ey <= 1e-2 and ry <= 5e-3, (hd, ey, ry)
        assert eh <= 1e-2 and rh <= 5e-3, (hd, eh, rh)


def test_single_bf16_state_copy_would_break_the_bound():
    """Why the walk splits the carried state: with one bf16 copy in C S^T the
    model's worst element, over 1000 tokens from an initial state, is beyond
    the 3% the GPU tests allow."""
    inp = W.make_ssd_inputs(W.SSD_WORKLOAD_BY_NAME["small_ssd"], with_state=True, L=1000)
    y, _ = model(inp, True, split_state=False)
    y_ref, _ = oracle_ref(inp, True)
    worst = max(errors_of_scale(y[:, :, hd], y_ref[:, :, hd]) for hd in range(y.shape[2]))
    assert worst > 3e-2, worst


# heads of the Mamba-2 workload (B1 L4096, 64 heads) whose outputs cancel most
MAMBA2_HEADS = (22, 31, 41)


def test_m_split_keeps_the_mamba2_heads_within_the_bound():
    """Why the walk splits M: on the Mamba-2 workload's most cancelling heads,
    a single bf16 copy of M puts elements beyond 2e-2 max(1, |ref|); the
    hi + lo pair keeps them within 0.6 of it (what remains is the rounding of
    w x to bf16 and of y itself)."""
    sw = W.SSD_WORKLOAD_BY_NAME["mamba2_ssd"]
    inp = W.make_ssd_inputs(sw, with_state=True)
    heads = list(MAMBA2_HEADS)
    sub = {k: v for k, v in inp.items()}
    sub["x"], sub["dt_raw"] = inp["x"][:, :, heads], inp["dt_raw"][:, :, heads]
    for k in ("dt_bias", "A_log", "D"):
        sub[k] = inp[k][heads]
    sub["h0"] = inp["h0"][:, heads]
    y_ref, _ = oracle_ref(sub, True)
    y1, _ = model(sub, True, split_m=False)
    y2, _ = model(sub, True, split_m=True)
    single = max(errors(y1[:, :, hd], y_ref[:, :, hd])[0] for hd in range(len(heads)))
    pair = max(errors(y2[:, :, hd], y_ref[:, :, hd])[0] for hd in range(len(heads)))
    assert single > 2e-2, single
    assert pair <= 1.2e-2, pair
