"""DFlash block-diffusion draft step on B200 (sm_100a).

The CUDA library (libdflash.so) is loaded on first use by the `dflash`
binding; importing this package loads nothing.  Modules:
  dflash   - ctypes binding with the C ABI's names (include/dflash.h)
  drafter  - torch-memory convenience layer (Drafter, Cache)
  inputs   - seeded synthetic inputs and workload presets
  build    - nvcc build of libdflash.so for sm_100a
"""
