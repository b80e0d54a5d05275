"""B200-native split-KV decode attention over a paged, variable-length KV cache.

The compute path is the CUDA library ``libda.so`` (sources in ``csrc/``, C ABI in
``include/da.h``); ``variable_length_paged_b200.da`` is its thin ctypes binding
and ``variable_length_paged_b200.workloads`` the seeded input generator.
Importing this package loads nothing; the binding loads the library on first
use and raises if it is missing.
"""
