"""B200-native Mixture-of-Experts layer (router, capacity-limited dispatch, grouped expert FFN
on tcgen05 tensor cores, combine; forward and backward) behind a C ABI (include/moe.h).

Submodules:
  configs  layer shapes (plain data)
  synth    seeded synthetic inputs (shared with the test oracle; no layer arithmetic)
  moe      ctypes binding of libmoe.so (imports fail loudly if the library is missing)
  layer    torch-allocated workspaces and views around the binding
  build    nvcc build of libmoe.so
"""
