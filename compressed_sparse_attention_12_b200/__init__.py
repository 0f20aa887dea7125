"""C4 compressed sparse attention (DeepSeek-V4 style) on B200 / sm_100a.

The compute path is the C-ABI library ``libcsa.so`` built from ``csrc/``;
``csa`` is its thin ctypes binding and ``synth`` draws seeded synthetic
workloads.  Importing the package does not load the library; the first call
through ``csa`` does, and raises if it is missing.
"""
