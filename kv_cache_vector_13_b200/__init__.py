"""TurboQuant KV-cache compression and decode attention for NVIDIA B200.

The compute path is the CUDA library libtq_b200.so (C ABI in include/tq.h);
``api`` is its thin torch binding and ``inputs`` holds the seeded synthetic
workloads.  Importing the package does not load the library; the first call
into ``api`` does, and fails loudly when it is missing.
"""

__all__ = ["api", "inputs", "build"]
