"""The FMA-pipe exp2 on the device (axon_exp2_fma), against float64 exp2.

Bound: relative error within 1.5 * 2^-24 for every x in [-126, 0] (the
degree-6 minimax polynomial's float32 evaluation stays within 1.3 * 2^-24 and
adding n to the exponent is exact) -- tighter than the 2-ulp bound of the
library's exp2f; exactly 1 at 0, exact powers of two at the integers, 2^-126
below -126.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ULP = 2.0 ** -24


def run(x_np):
    from selective_state_space_52_b200 import axon_ssm
    x = torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).cuda()
    y = axon_ssm.exp2_fma(x)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_exp2_fma_relative_error(cuda_lib):
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-126.0, 0.0, 4_000_001), -rng.exponential(3.0, 1_000_001),
                        -np.ldexp(rng.random(200_001), -rng.integers(1, 60, 200_001))]).astype(np.float32)
    x = x[x >= -126.0]
    got = run(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= 1.5 * ULP, (rel.max() / ULP, float(x[np.argmax(rel)]))


def test_exp2_fma_special_values(cuda_lib):
    ints = -np.arange(0, 127, dtype=np.float32)
    got = run(ints)
    assert np.array_equal(got, np.exp2(ints.astype(np.float64)).astype(np.float32))
    assert run(np.array([0.0], dtype=np.float32))[0] == 1.0
    low = run(np.array([-126.0, -300.0, -1e30], dtype=np.float32))
    assert np.all(low == np.float32(2.0 ** -126))


def test_exp2_fma_odd_count_and_in_place(cuda_lib):
    from selective_state_space_52_b200 import axon_ssm
    x = -torch.rand(1001, device="cuda") * 20.0
    ref = torch.exp2(x.double())
    y = axon_ssm.exp2_fma(x.clone())
    axon_ssm.exp2_fma(x, out=x)                    # y may be x itself
    torch.cuda.synchronize()
    assert torch.equal(x, y)
    assert float((y.double() / ref - 1.0).abs().max()) <= 1.5 * ULP
