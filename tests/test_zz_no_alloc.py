"""kvattn_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (an engine that has reserved all of HBM for its own pool, a
plugin host that passes only inputs and outputs, a path where a cudaMalloc's
possible device synchronisation is not acceptable) get an entry point whose
scratch is a fixed device array inside the library.  These tests call it
through the C ABI twice in a row, on two different problems, and compare each
result with kvattn_decode's within the parity tolerances and with the fp64
oracle; they also run a problem that fits the array only with fewer parts per
context than the library would choose, check that a problem too large for the
array is refused, and that the per-call device error word is reported and
cleared.  This file is collected last on purpose.
"""

import numpy as np
import pytest

from shared_kv_caches_b200 import kvattn as K
from shared_kv_caches_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_REL, TOL_LSE = 2e-2, 5e-3, 1e-3


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from shared_kv_caches_b200 import build
    build.build()
    return torch.device("cuda:0")


def _noalloc(p, err=None):
    import torch
    st = K.kvattn_decode_noalloc(p.variant, p.params, p.q_nope.data_ptr(),
                                 None if p.q_rope is None else p.q_rope.data_ptr(), p.kv.data_ptr(),
                                 None if p.block_table is None else p.block_table.data_ptr(),
                                 p.seq_lens.data_ptr(), p.sm_scale, p.out.data_ptr(), p.lse.data_ptr(),
                                 None if err is None else err.data_ptr(),
                                 torch.cuda.current_stream(p.device).cuda_stream)
    return st


def _close(a_out, a_lse, b_out, b_lse):
    err = np.abs(a_out - b_out).max()
    rel = np.linalg.norm(a_out - b_out) / max(np.linalg.norm(b_out), 1e-30)
    fin = np.isfinite(b_lse)
    assert (np.isfinite(a_lse) == fin).all()
    dl = np.abs(a_lse[fin] - b_lse[fin]).max() if fin.any() else 0.0
    assert err <= TOL_MAX and rel <= TOL_REL and dl <= TOL_LSE, (err, rel, dl)


def test_two_calls_in_a_row_match_kvattn_decode(dev, oracle_mod):
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    shapes = [W.WORKLOADS["gqa"].replace(batch=4, ctx=(1, 3000)),
              W.WORKLOADS["mlra_128k"].replace(batch=2, ctx=(100, 2000))]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for i, shape in enumerate(shapes):
        x = W.make_inputs(shape, seed=20 + i)
        p = DeviceProblem(x, dev)
        p.run()
        torch.cuda.synchronize()
        ref_out, ref_lse = p.results()
        p.out.fill_(float("nan"))
        p.lse.fill_(float("nan"))
        assert _noalloc(p, err) == K.KVATTN_OK
        torch.cuda.synchronize()
        out, lse = p.results()
        _close(out, lse, ref_out, ref_lse)
        assert int(err.item()) == 0
        orc_out, orc_lse = oracle_mod.decode(x)
        _close(out, lse, orc_out, orc_lse)


def test_problem_that_fits_only_with_fewer_parts(dev, oracle_mod):
    """The library's own plan for this MLA batch needs more scratch than the
    array holds; the entry point lowers the part count until it fits and
    must then give kvattn_decode's result for that part count."""
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    shape = W.WORKLOADS["mla"].replace(batch=64, ctx=(8192, 8192))
    x = W.make_inputs(shape, seed=41)
    params = K.params_for(shape, x["max_pages_per_seq"], x["num_pages"], 8192)
    auto = K.kvattn_get_plan(K.KVATTN_MLA, params)
    assert auto.workspace_bytes > K.KVATTN_NOALLOC_SCRATCH_BYTES, auto.workspace_bytes
    fit = None
    for s in range(auto.num_splits - 1, 0, -1):
        q = K.params_for(shape, x["max_pages_per_seq"], x["num_pages"], 8192, num_splits=s)
        if K.kvattn_get_plan(K.KVATTN_MLA, q).workspace_bytes <= K.KVATTN_NOALLOC_SCRATCH_BYTES:
            fit = s
            break
    assert fit is not None
    p = DeviceProblem(x, dev, num_splits=fit)
    p.run()
    torch.cuda.synchronize()
    ref_out, ref_lse = p.results()
    p.params = params                        # the caller's request: library choice of parts
    p.out.fill_(float("nan"))
    p.lse.fill_(float("nan"))
    err = torch.full((1,), -1, dtype=torch.int32, device=dev)
    assert _noalloc(p, err) == K.KVATTN_OK
    torch.cuda.synchronize()
    out, lse = p.results()
    _close(out, lse, ref_out, ref_lse)
    assert int(err.item()) == 0
    b_list = [0, 37, 63]
    orc_out, orc_lse = oracle_mod.decode(x, b_list=b_list)
    _close(out[b_list], lse[b_list], orc_out, orc_lse)


def test_refused_call_leaves_the_array_alone(dev):
    """A call refused for a bad pointer enqueues nothing (the next good call
    still reports only its own errors)."""
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    x = W.make_inputs(W.WORKLOADS["gla"].replace(batch=1, ctx=(100, 100)), seed=42)
    p = DeviceProblem(x, dev)
    st = K.kvattn_decode_noalloc(p.variant, p.params, p.q_nope.data_ptr() + 2, p.q_rope.data_ptr(),
                                 p.kv.data_ptr(), p.block_table.data_ptr(), p.seq_lens.data_ptr(),
                                 p.sm_scale, p.out.data_ptr(), p.lse.data_ptr(), None,
                                 torch.cuda.current_stream(dev).cuda_stream)
    assert st == K.KVATTN_ERR_MISALIGNED
    st = K.kvattn_decode_noalloc(p.variant, p.params, p.q_nope.data_ptr(), p.q_rope.data_ptr(),
                                 p.kv.data_ptr(), p.block_table.data_ptr(), None, p.sm_scale,
                                 p.out.data_ptr(), p.lse.data_ptr(), None, 0)
    assert st == K.KVATTN_ERR_INVALID_ARG


def test_noalloc_reports_and_clears_device_errors(dev):
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    shape = W.WORKLOADS["gla"].replace(batch=2, ctx=(300, 300))
    x = W.make_inputs(shape, seed=30)
    bt = x["block_table"].copy()
    bt[0, 1] = x["num_pages"] + 7           # a frame id outside the pool: skipped, reported
    p = DeviceProblem(dict(x, block_table=bt), dev)
    err = torch.full((1,), -1, dtype=torch.int32, device=dev)
    assert _noalloc(p, err) == K.KVATTN_OK
    torch.cuda.synchronize()
    assert int(err.item()) & K.KVATTN_DEVERR_PAGE_OUT_OF_RANGE
    good = DeviceProblem(x, dev)
    assert _noalloc(good, err) == K.KVATTN_OK
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_problem_larger_than_scratch_is_refused(dev):
    shape = W.WORKLOADS["mla"]
    # 1 part per context already needs B*H*512*4 bytes; B = 256 needs 64 MiB > 32 MiB
    p = K.make_params(256, 128, 1, 512, 64, 8, 2048, 512, 0)
    plan = K.kvattn_get_plan(K.KVATTN_MLA, K.make_params(256, 128, 1, 512, 64, 8, 2048, 512, 1))
    assert plan.workspace_bytes > K.KVATTN_NOALLOC_SCRATCH_BYTES
    fake = 1 << 20      # refused before any pointer is used
    st = K.kvattn_decode_noalloc(K.KVATTN_MLA, p, fake, fake, fake, fake, fake, shape.scale, fake, fake,
                                 None, 0)
    assert st == K.KVATTN_ERR_WORKSPACE_TOO_SMALL
    forced = K.make_params(256, 128, 1, 512, 64, 8, 2048, 512, 3)
    st = K.kvattn_decode_noalloc(K.KVATTN_MLA, forced, fake, fake, fake, fake, fake, shape.scale, fake,
                                 fake, None, 0)
    assert st == K.KVATTN_ERR_WORKSPACE_TOO_SMALL
