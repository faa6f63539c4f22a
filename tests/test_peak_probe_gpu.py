"""The throughput probes behind bench.py's in-run roofline (axon_peak_probe):
the MUFU exp2 and float32 FMA rates they measure lie between 60% and 110% of
the SM count x lanes per clock x the SM clock the device reports (16 MUFU
and 128 FMA lanes per SM per clock on B200), and the probes' sums are finite.
"""
import math

import pytest
import torch

pytestmark = pytest.mark.gpu


def max_sm_clock_hz() -> float:
    """The device's maximum SM clock from NVML (1965 MHz, B200's, without NVML)."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
        return pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM) * 1e6
    except Exception:
        return 1.965e9


@pytest.mark.parametrize("kind,lanes", [(0, 16), (1, 128)])
def test_peak_probe_rate(cuda_lib, kind, lanes):
    props = torch.cuda.get_device_properties(0)
    sms = props.multi_processor_count
    blocks = sms * 8
    out = torch.empty(blocks * 256, dtype=torch.float32, device="cuda")
    iters = 2048 if kind == 0 else 8192
    cuda_lib.axon_peak_probe(kind, out, blocks, iters)
    torch.cuda.synchronize()
    best = math.inf
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(); cuda_lib.axon_peak_probe(kind, out, blocks, iters); b.record()
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b) / 1e3)
    rate = blocks * 256 * 8 * iters / best
    nominal = sms * lanes * max_sm_clock_hz()
    assert 0.6 * nominal <= rate <= 1.1 * nominal, (rate / 1e9, nominal / 1e9)
    assert torch.isfinite(out).all()
