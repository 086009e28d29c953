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


def test_line_keeps_the_timed_step_count():
    """"steps" in the JSON line is the timed step count K; the breakdown of
    the steps either side of attention goes under its own key."""
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert 'line["steps"] =' not in src
    assert 'line["steps_ops"] = measure_steps' in src


def test_cache_bytes_per_token_of_each_variant():
    """Algorithmic cache bytes per context token: K and V of every KV head in
    bf16 (one byte per element for the fp8 cache), one tied plane for GTA and
    MFA-KR, the 576-wide latent row for MLA, GLA-2 and MLRA-4."""
    from shared_kv_caches_b200 import benchutil as BU
    from shared_kv_caches_b200 import workloads as W
    want = {"gqa": 4096, "gqa_fp8": 2048, "gta": 2048, "mfa": 1024, "mfa_kr": 512, "mla": 1152, "gla": 1152,
            "mlra_128k": 1152}
    for name, n in want.items():
        assert BU.kv_bytes_per_token(W.WORKLOADS[name]) == n, name


def test_suite_covers_every_benchmark_problem():
    """The default run times every benchmark problem except the tiny parity
    case, with MLA (the largest single-GPU problem) as the headline."""
    from shared_kv_caches_b200 import workloads as W
    assert bench.DEFAULT_WORKLOAD == "suite"
    assert set(bench.SUITE) == set(W.WORKLOADS) - {"tiny_mla"}
    assert bench.SUITE[0] == "mla"
    assert bench.problem_names("suite") == ("mla",)
    assert bench.problem_names("gqa+mfa") == ("gqa", "mfa")


def test_clock_summary_over_several_windows():
    from shared_kv_caches_b200.benchutil import ClockSampler
    cs = ClockSampler()
    none = {r: False for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")}
    cap = dict(none, sw_power_cap=True)
    cs.samples = [(1.0, 1965.0, 1965.0, 500.0, none), (2.0, 1900.0, 1965.0, 900.0, cap),
                  (5.0, 1000.0, 1965.0, 100.0, none), (8.0, 1965.0, 1965.0, 600.0, none)]
    s = cs.summary_windows([(0.5, 2.5), (7.5, 8.5)])
    assert s["samples"] == 3 and s["reasons"] == ["sw_power_cap"] and s["sm_mhz"] == 1965.0
    assert cs.summary(4.0, 6.0)["window"] == "nearest"
