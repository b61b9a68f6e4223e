"""Seeded synthetic inputs for the LSA hot path, shared by the oracle-based tests and the GPU runs.

Holds only random-number generation and storage encodings (BF16, FP8 e4m3); none of the
method's arithmetic.  ``gen`` is the host generator, ``workloads`` the workload shapes,
``device`` the GPU filler that writes the same bytes directly into device memory.
"""
from . import gen, workloads  # noqa: F401
