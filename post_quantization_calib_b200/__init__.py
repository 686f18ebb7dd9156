"""SmoothQuant smoothed W8A8 linear for NVIDIA B200 (sm_100a).

Modules:
  sq      ctypes binding of libsq (include/sq.h); importing it requires the built libsq.so.
  layer   SmoothedW8A8Linear: sequencing of the libsq calls for one smoothing group.
  dist    data-parallel plumbing (sharded calibration with an all-reduce(MAX)).
  synth   seeded synthetic inputs and the workload table.
  build   nvcc build of libsq.so.
"""
__version__ = "0.1.0"
