"""Seeded synthetic workloads for the tests and the benchmark.

This package holds the parameter-shape tables of the benchmark workloads
and a counter-based random generator.  It contains none of the optimizer's
arithmetic (no downcast-with-ECC, no companding, no update): it only says
which float32 masters and which 16-bit gradients exist, so that the CPU
oracle and the CUDA library can each encode and step them on their own.

The same generator exists twice, from one definition:
  * ``workloads.gen`` - numpy, host, random access by element index;
  * ``workloads/csrc/gen.cu`` - CUDA, device, for full-size inputs.
Every value is built from integer arithmetic and correctly rounded IEEE
binary32 operations (no transcendental functions), so both produce the
same bits; a GPU test checks that on sampled indices.
"""
from .shapes import CONFIGS, TensorSpec, Workload, workload  # noqa: F401
