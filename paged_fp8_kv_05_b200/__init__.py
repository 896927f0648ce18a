"""Paged FP8 KV decode / MTP-verify attention for NVIDIA B200 (sm_100a).

The product is the C-ABI shared library ``libatlas_kv.so`` built from
``csrc/`` (entry points declared in ``include/atlas_kv.h``).  ``atlas_kv``
is its thin ctypes binding; ``workloads`` draws the seeded synthetic inputs.
Importing this package loads nothing; ``from paged_fp8_kv_05_b200 import
atlas_kv`` loads the library and fails loudly if it has not been built.
"""
