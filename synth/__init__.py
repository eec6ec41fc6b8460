"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the benchmark.

This package generates inputs only: fp16 keys, values and queries with the
shapes and value distributions of the workloads below, plus the raw samples a
per-layer codebook is fitted on. It holds none of the quantization or
attention arithmetic. Two implementations of one counter-based generator live
here and agree bit for bit:

* ``philox.py``: numpy, for the CPU side (oracle inputs, sampled checks);
* ``gen.cu`` (built into ``libkvqsynth.so``): the same generator as a CUDA
  kernel, for filling device buffers of any size (the 1M-token cache).

See ``philox.py`` for the definition of the generator.
"""
from .philox import (  # noqa: F401
    philox4x32_10,
    normals,
    Workload,
    WORKLOADS,
    workload,
    gen_k,
    gen_v,
    gen_q,
    heavy_channel_scale,
    student_t_channels,
    codebook_samples_k,
    codebook_samples_v,
)
