"""Host-side pieces of bench.py: the stored DRAM-traffic lookup and the
per-kernel source digests that decide whether a stored figure still applies."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_every_kernel_digest_covers_its_sources():
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files + bench.SHARED_SOURCES:
            assert os.path.exists(os.path.join(ROOT, "shared_kv_caches_b200", "csrc", f)), (kernel, f)
        d = bench.source_digest(kernel)
        assert len(d) == 16 and int(d, 16) >= 0
        assert d == bench.source_digest(kernel)          # stable


def test_digests_differ_between_kernels():
    ds = {k: bench.source_digest(k) for k in bench.KERNEL_SOURCES}
    assert len(set(ds.values())) == len(ds)


def test_stored_traffic_matches_only_current_digest():
    path = os.path.join(ROOT, "profiles", "ncu_traffic.md")
    rows = []
    for line in open(path):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 5 and cells[3].isdigit():
            rows.append(cells)
    assert rows, "no traffic rows"
    for wl, prob, _kname, nbytes, digest in (r[:5] for r in rows):
        assert bench.stored_traffic(wl, prob, digest) == float(nbytes)
        assert bench.stored_traffic(wl, prob, "0" * 16) is None
    assert bench.stored_traffic("no-such-workload", "x", rows[0][4]) is None
