"""B200-native multi-head ReLU linear self-attention forward (Sana Linear DiT).

The compute path is the C-ABI library ``libsana_linattn.so`` (CUDA, sm_100a);
``ops`` marshals torch tensors into it. The library is loaded on first use and
a missing or unloadable library raises: there is no CPU fallback.
"""
from .workloads import WORKLOADS, Workload, make_inputs  # noqa: F401

__all__ = ["WORKLOADS", "Workload", "make_inputs"]
