"""Exact, IO-aware tiled attention for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libfa.so`` (CUDA kernels for sm_100a);
``exact_io_aware_45_b200.fa`` is its thin Python binding. ``inputs`` holds the
seeded synthetic workloads. Importing the package does not load the library;
the first call into ``fa`` does, and fails loudly if it is missing.
"""
