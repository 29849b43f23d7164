"""B200-native (sm_100a) selective diagonal state-space scan.

The forward and backward scan of a linear-transition diagonal SSM
``h_t = A_t h_{t-1} + B_t u_t, y_t = C_t h_t + D u_t`` with HybridMamba's mix of
per-coordinate-decay real states and 2x2 rotation pairs, two-endpoint writes
and SSD-MIMO rank-R routing, as a C-ABI CUDA library (``include/ssm_scan.h``).

Modules:
  ``abi``        ctypes binding with the C entry-point names
  ``scan``       torch device-buffer helpers around the binding
  ``cp``         sequence sharding: segment scans joined through boundary values
  ``dist``       data-parallel plumbing (parameter-gradient all-reduce)
  ``synthetic``  seeded input generators (no scan arithmetic)
  ``build``      nvcc build of ``libssm_scan.so`` for sm_100a
"""
from .synthetic import WORKLOADS, WORKLOAD_ORDER, ScanShape  # noqa: F401

__all__ = ["WORKLOADS", "WORKLOAD_ORDER", "ScanShape"]
