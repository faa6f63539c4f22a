"""The seeded input generators (CPU): the test inputs vary every per-channel
parameter from one channel to the next, so that a kernel reading a parameter
of the wrong channel (or a constant in its place) fails the GPU parity tests;
the five measured workloads keep the layer's initialisation."""
import math

import numpy as np
import torch

from selective_state_space_52_b200 import workloads as W


def test_random_params_differ_per_channel_and_state():
    p = W.make_params(W.custom(1, 8, 64, io="bf16", seed=5))
    for k in ("conv_b", "D", "dt_bias"):
        v = p[k].numpy()
        assert len(np.unique(v)) == v.size, k
    a = p["A_log"].numpy()
    assert len(np.unique(a)) >= 0.99 * a.size               # (channel, state) values differ
    assert len(np.unique(a, axis=0)) == a.shape[0]          # no two channels share their A_log row
    base = np.log(np.arange(1, 17, dtype=np.float64))
    dev = a - base[None, :]
    assert 0.05 < dev.std() < 0.2 and abs(dev.mean()) < 0.05   # log(1..N) + N(0, 0.1^2)
    assert 0.5 < p["D"].std().item() < 1.5 and (p["D"] < 0).any()
    assert 0.05 < p["conv_b"].std().item() < 0.2


def test_measured_workloads_keep_the_initialisation():
    for wl in W.WORKLOADS:
        assert wl.params == "init"
        p = W.make_params(W.Workload(wl.name, 1, 1, 16, wl.io, wl.seed, dt_mode=wl.dt_mode))
        assert torch.all(p["conv_b"] == 0) and torch.all(p["D"] == 1)
        ref = torch.log(torch.arange(1, 17, dtype=torch.float64)).to(torch.float32)
        assert torch.equal(p["A_log"], ref.expand(16, 16))


def test_block_test_layer_uses_random_params():
    bw = W.BLOCK_WORKLOAD_BY_NAME["small_block"]
    assert bw.params == "random" and bw.core().params == "random"
    assert W.BLOCK_WORKLOAD_BY_NAME["bit_axon_block"].params == "init"


def test_unknown_param_mode_is_rejected():
    try:
        W.make_params(W.custom(1, 1, 8, params="trained"))
    except ValueError:
        return
    raise AssertionError("an unknown parameter mode was accepted")
