"""Frame/block-sparse self-attention for long video DiT sequences on B200.

Submodules:
  binding    ctypes binding of libbsa.so (the CUDA path; raises on import if
             the library is missing - there is no fallback)
  build      nvcc build of libbsa.so for sm_100a
  workloads  workload shapes (data only)
  inputs     seeded synthetic q/k/v generators (no method arithmetic)
"""
