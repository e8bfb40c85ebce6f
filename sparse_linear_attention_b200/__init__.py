"""SLA2 / SLA sparse-linear attention forward on NVIDIA B200 (sm_100a).

The compute lives in libsla.so (hand-written CUDA behind the C ABI of
include/sla.h); `sla` is its ctypes binding and `inputs` draws seeded
synthetic workloads.
"""
from . import sla  # noqa: F401
