"""B200-native selective-scan (S6) layer core: causal conv1d(K=4)+SiLU, dt, the
diagonal selective recurrence, C contraction + D skip and the SiLU(z) gate,
behind the C ABI declared in include/axon_ssm.h.

Submodules are imported on demand: ``axon_ssm`` (the binding to the CUDA
library; it raises if the library is not built) and ``workloads`` (seeded
synthetic inputs).
"""
__all__ = ["axon_ssm", "workloads"]
