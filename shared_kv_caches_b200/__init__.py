"""B200-native decode attention over compressed / shared KV caches.

The compute path is the C-ABI CUDA library ``libkvattn.so`` (built from
``csrc/`` for sm_100a); ``kvattn`` is its thin ctypes binding and
``workloads`` draws seeded synthetic inputs.
"""
