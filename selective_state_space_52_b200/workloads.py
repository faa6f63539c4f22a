"""Seeded synthetic inputs for the selective-scan layer core.

This module only draws random numbers and shapes them; it holds none of the
layer's arithmetic.  Both sides of every parity check (the CUDA library and the
fp64 oracle) receive tensors made here, so they see identical bits: bf16 inputs
are drawn in fp32 on the CPU generator and rounded to bf16 once
(round-to-nearest-even), and the oracle upcasts those exact bf16 values.

Distributions ("config-0 distributions"), for every workload below:
  x, z ~ N(0, 1);  B, C ~ N(0, 1)          (B, C shared by all channels, (B,L,N))
  conv_w ~ N(0, 1/4) (variance), conv_b = 0
  dt_raw ~ N(0, 0.5) (variance)
  dt_bias = log(expm1(u)), u ~ logUniform[1e-3, 1e-1] per channel
            (the inverse-softplus initialisation: softplus(dt_bias) = u)
  A_log[e, n] = log(n + 1)   (so the diagonal of A is -1, -2, ..., -N)
  D = 1
The Mamba-block workload adds a bimodal dt: even channels u = 1e-4 (long
memory), odd channels u = 1.0 (fast forgetting), same dt_raw noise.

Test inputs (``params="random"``, the default of ``custom``) make every
per-channel parameter differ from one channel to the next, as a trained layer's
do (A_log is a learned per-state parameter that log(1..N) only initialises):
  conv_b ~ N(0, 0.1^2) per channel;  D ~ N(0, 1) per channel;
  A_log[e, n] = log(n + 1) + N(0, 0.1^2) per (channel, state).
The five measured workloads keep the initialisation above.

The Mamba-2 (SSD) workloads (``SSD_WORKLOADS``): x ~ N(0, 1) (B,L,H,64),
dt_raw ~ N(0, 0.5), B, C ~ N(0, 1) (B,L,128) in bf16; per head dt_bias =
log(expm1(u)), u ~ logUniform[1e-3, 1e-1], A_log = log(Uniform[1, 16]) and
D = 1; an initial state h0 ~ N(0, 1/4).

The whole-layer workloads (``BLOCK_WORKLOADS``) draw the layer input
X ~ N(0, 1) and the projection weights with fan-in scaling, W_in ~ N(0, 1/Dm),
W_x ~ N(0, 1/E), W_out ~ N(0, 1/E), all rounded to bf16 once; the per-channel
parameters are those above (drawn for E channels).  dt_raw, B and C then come
out of the projection with standard deviation about 0.6.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

N_STATE = 16
K_CONV = 4


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    E: int
    io: str                      # "f32" or "bf16"
    seed: int
    dt_mode: str = "logu"        # "logu" or "bimodal"
    decode_steps: int = 0        # cached single-token steps after the prefill
    note: str = ""
    params: str = "init"         # "init": conv_b 0, D 1, A_log log(1..N); "random": per-channel draws
    N: int = N_STATE
    K: int = K_CONV

    @property
    def torch_io(self):
        return torch.float32 if self.io == "f32" else torch.bfloat16

    @property
    def token_channels(self) -> int:
        return self.B * self.L * self.E


# The five workloads of the measurement plan.  Index = seed.
WORKLOADS = [
    Workload("tiny_f32", 1, 64, 32, "f32", 0,
             note="tiny fp32 scan, B1 L64 E32"),
    Workload("bit_axon_layer", 1, 2048, 7680, "bf16", 1,
             note="Bit-Axon layer shape: D=2560, expand 3 -> E=7680; bf16 io, fp32 state"),
    Workload("mamba_block", 2, 4096, 2048, "f32", 2, dt_mode="bimodal",
             note="Mamba block shape: d_model 1024, expand 2 -> E=2048; fp32 io; bimodal dt"),
    Workload("long_seq", 1, 65536, 2048, "bf16", 3,
             note="long sequence, multi-chunk carry; returns final ssm_state and conv_cache"),
    Workload("decode", 64, 128, 7680, "bf16", 4, decode_steps=512,
             note="64 sequences prefilled with 128 tokens, then 512 cached decode steps"),
]
WORKLOAD_BY_NAME = {w.name: w for w in WORKLOADS}


def custom(B, L, E, io="f32", seed=0, dt_mode="logu", name="custom", params="random") -> Workload:
    return Workload(name, B, L, E, io, seed, dt_mode=dt_mode, params=params)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def make_params(wl: Workload, g: torch.Generator | None = None) -> dict:
    """fp32 per-channel parameters: conv_w (E,K), conv_b (E), dt_bias (E), A_log (E,N), D (E)."""
    g = g or _gen(wl.seed)
    E, N, K = wl.E, wl.N, wl.K
    conv_w = torch.randn(E, K, generator=g, dtype=torch.float32) * 0.5      # variance 1/4
    conv_b = torch.zeros(E, dtype=torch.float32)
    if wl.dt_mode == "bimodal":
        u = torch.where(torch.arange(E) % 2 == 0,
                        torch.tensor(1e-4, dtype=torch.float64),
                        torch.tensor(1.0, dtype=torch.float64))
    else:
        lo, hi = math.log(1e-3), math.log(1e-1)
        u = torch.exp(lo + (hi - lo) * torch.rand(E, generator=g, dtype=torch.float64))
    dt_bias = torch.log(torch.expm1(u)).to(torch.float32)
    A_log = torch.log(torch.arange(1, N + 1, dtype=torch.float64))
    A_log = A_log.unsqueeze(0).expand(E, N).contiguous()
    D = torch.ones(E, dtype=torch.float32)
    if wl.params == "random":
        conv_b = torch.randn(E, generator=g, dtype=torch.float32) * 0.1
        D = torch.randn(E, generator=g, dtype=torch.float32)
        A_log = A_log + torch.randn(E, N, generator=g, dtype=torch.float64) * 0.1
    elif wl.params != "init":
        raise ValueError(f"params must be 'init' or 'random', not {wl.params!r}")
    A_log = A_log.to(torch.float32)
    return {"conv_w": conv_w, "conv_b": conv_b, "dt_bias": dt_bias, "A_log": A_log, "D": D}


def make_sequence(wl: Workload, L: int | None = None, g: torch.Generator | None = None,
                  B: int | None = None) -> dict:
    """x, z, dt_raw (B,L,E) and B, C (B,L,N) in the workload's io dtype."""
    g = g or _gen(wl.seed + 1000)
    Bsz = wl.B if B is None else B
    L = wl.L if L is None else L
    E, N = wl.E, wl.N
    io = wl.torch_io
    x = torch.randn(Bsz, L, E, generator=g, dtype=torch.float32).to(io)
    z = torch.randn(Bsz, L, E, generator=g, dtype=torch.float32).to(io)
    dt_raw = (torch.randn(Bsz, L, E, generator=g, dtype=torch.float32) * math.sqrt(0.5)).to(io)
    Bm = torch.randn(Bsz, L, N, generator=g, dtype=torch.float32).to(io)
    Cm = torch.randn(Bsz, L, N, generator=g, dtype=torch.float32).to(io)
    return {"x": x, "z": z, "dt_raw": dt_raw, "B": Bm, "C": Cm}


def make_state(wl: Workload, g: torch.Generator | None = None, B: int | None = None,
               zero: bool = False) -> dict:
    """An initial (conv_cache (B,K-1,E) io, ssm_state (B,E,N) fp32) pair."""
    Bsz = wl.B if B is None else B
    if zero:
        return {"conv_cache": torch.zeros(Bsz, wl.K - 1, wl.E, dtype=wl.torch_io),
                "ssm_state": torch.zeros(Bsz, wl.E, wl.N, dtype=torch.float32)}
    g = g or _gen(wl.seed + 2000)
    cc = torch.randn(Bsz, wl.K - 1, wl.E, generator=g, dtype=torch.float32).to(wl.torch_io)
    ss = torch.randn(Bsz, wl.E, wl.N, generator=g, dtype=torch.float32) * 0.5
    return {"conv_cache": cc, "ssm_state": ss}


def make_inputs(wl: Workload, with_state: bool = False, L: int | None = None) -> dict:
    """Everything one prefill call needs, on the CPU, seeded by the workload."""
    out = make_params(wl)
    out.update(make_sequence(wl, L=L))
    if with_state:
        out.update(make_state(wl))
    return out


def make_decode_inputs(wl: Workload, steps: int, g: torch.Generator | None = None) -> dict:
    """Per-step inputs for `steps` cached decode steps: x, z, dt_raw (S,B,E), B, C (S,B,N)."""
    g = g or _gen(wl.seed + 3000)
    io = wl.torch_io
    S, Bsz, E, N = steps, wl.B, wl.E, wl.N
    return {
        "x": torch.randn(S, Bsz, E, generator=g, dtype=torch.float32).to(io),
        "z": torch.randn(S, Bsz, E, generator=g, dtype=torch.float32).to(io),
        "dt_raw": (torch.randn(S, Bsz, E, generator=g, dtype=torch.float32) * math.sqrt(0.5)).to(io),
        "B": torch.randn(S, Bsz, N, generator=g, dtype=torch.float32).to(io),
        "C": torch.randn(S, Bsz, N, generator=g, dtype=torch.float32).to(io),
    }


# ------------------------------------------------------------ whole layer
@dataclass(frozen=True)
class BlockWorkload:
    name: str
    B: int
    L: int
    Dm: int          # hidden size D of the layer configuration table
    E: int           # d_inner = expand * D
    seed: int
    note: str = ""
    N: int = N_STATE
    K: int = K_CONV
    params: str = "init"

    def core(self) -> Workload:
        """The layer-core workload with the same per-channel parameters."""
        return Workload(self.name, self.B, self.L, self.E, "bf16", self.seed, params=self.params)


BLOCK_WORKLOADS = [
    BlockWorkload("bit_axon_block", 1, 2048, 2560, 7680, 11,
                  note="the Bit-Axon layer: D=2560, expand 3 -> E=7680, bf16"),
    BlockWorkload("small_block", 2, 100, 256, 768, 12, note="small layer for parity tests",
                  params="random"),
]
BLOCK_WORKLOAD_BY_NAME = {w.name: w for w in BLOCK_WORKLOADS}


def make_block_inputs(bw: BlockWorkload, with_state: bool = False, L: int | None = None,
                      B: int | None = None) -> dict:
    """X (B,L,Dm), W_in (Dm,2E), W_x (E,E+2N), W_out (E,Dm) in bf16, plus the
    per-channel parameters (and an initial cache pair with ``with_state``)."""
    g = _gen(bw.seed + 5000)
    Bsz = bw.B if B is None else B
    L = bw.L if L is None else L
    Dm, E, N = bw.Dm, bw.E, bw.N
    out = make_params(bw.core())
    out["X"] = torch.randn(Bsz, L, Dm, generator=g, dtype=torch.float32).to(torch.bfloat16)
    out["W_in"] = (torch.randn(Dm, 2 * E, generator=g, dtype=torch.float32) / math.sqrt(Dm)).to(torch.bfloat16)
    out["W_x"] = (torch.randn(E, E + 2 * N, generator=g, dtype=torch.float32) / math.sqrt(E)).to(torch.bfloat16)
    out["W_out"] = (torch.randn(E, Dm, generator=g, dtype=torch.float32) / math.sqrt(E)).to(torch.bfloat16)
    if with_state:
        out.update(make_state(bw.core(), B=Bsz))
    return out


# ------------------------------------------------------------ Mamba-2 (SSD) core
@dataclass(frozen=True)
class SsdWorkload:
    name: str
    B: int
    L: int
    H: int
    seed: int
    P: int = 64
    N: int = 128
    note: str = ""


SSD_WORKLOADS = [
    SsdWorkload("mamba2_ssd", 1, 4096, 64, 21,
                note="Mamba-2 block: d_model 2048, expand 2 -> 64 heads of 64, d_state 128, bf16"),
    SsdWorkload("small_ssd", 2, 130, 3, 22, note="small SSD case for parity tests"),
]
SSD_WORKLOAD_BY_NAME = {w.name: w for w in SSD_WORKLOADS}


def make_ssd_inputs(sw: SsdWorkload, with_state: bool = False, L: int | None = None) -> dict:
    g = _gen(sw.seed + 7000)
    L = sw.L if L is None else L
    B, H, P, N = sw.B, sw.H, sw.P, sw.N
    bf = torch.bfloat16
    lo, hi = math.log(1e-3), math.log(1e-1)
    u = torch.exp(lo + (hi - lo) * torch.rand(H, generator=g, dtype=torch.float64))
    out = {
        "x": torch.randn(B, L, H, P, generator=g, dtype=torch.float32).to(bf),
        "dt_raw": (torch.randn(B, L, H, generator=g, dtype=torch.float32) * math.sqrt(0.5)).to(bf),
        "B": torch.randn(B, L, N, generator=g, dtype=torch.float32).to(bf),
        "C": torch.randn(B, L, N, generator=g, dtype=torch.float32).to(bf),
        "dt_bias": torch.log(torch.expm1(u)).to(torch.float32),
        "A_log": torch.log(1.0 + 15.0 * torch.rand(H, generator=g, dtype=torch.float64)).to(torch.float32),
        "D": torch.ones(H, dtype=torch.float32),
    }
    if with_state:
        out["h0"] = torch.randn(B, H, P, N, generator=g, dtype=torch.float32) * 0.5
    return out
