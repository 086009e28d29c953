"""fp64 CPU oracle for decode attention over compressed / shared KV caches.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the cpu_baseline / reference leg of ``bench.py``, never by the library.
"""
