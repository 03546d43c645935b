"""B200-native (sm_100a) fused exact attention.

The compute path is the CUDA library ``libfa_sm100.so`` built from
``csrc/``; ``binding`` is a thin ctypes layer over its C ABI (``fa_fwd``,
``fa_bwd`` and friends, declared in ``include/fa.h``).  There is no CPU
fallback: calling into the binding without the built library raises.
"""
from .inputs import WORKLOADS, Workload, make_inputs, workload_inputs, sample_rows  # noqa: F401
