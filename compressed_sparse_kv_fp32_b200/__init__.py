"""B200-native ADAMAS sparse decode attention.

Submodules:
  synth       seeded synthetic workloads (no method arithmetic)
  accounting  byte accounting of the KV cache and of one decode step
  adamas      ctypes binding of the C-ABI library libadamas.so (CUDA, sm_100a)

The binding is imported lazily so that the generator and the accounting helpers
load on machines without a GPU.
"""
__all__ = ["synth", "accounting", "adamas"]
