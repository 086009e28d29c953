"""Failure detection on the device without a fault.

Every wait in the decode kernels is bounded: when it runs out the kernel sets
KVATTN_DEVERR_WAIT_TIMEOUT, drains what it started and returns.  The
self-test entry point runs that same wait on the device, once on a completed
barrier phase (it must succeed) and once on a barrier nothing arrives on (it
must give up after the few hundred tries asked for), and the context must
stay usable afterwards.
"""

import pytest

from shared_kv_caches_b200 import kvattn as K
from shared_kv_caches_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from shared_kv_caches_b200 import build
    build.build()
    return torch.device("cuda:0")


@pytest.mark.parametrize("tries", [1, 300])
def test_bounded_wait_runs_out_and_reports(dev, tries):
    import torch
    res = torch.zeros(1, dtype=torch.int32, device=dev)
    st = K.kvattn_selftest_bounded_wait(res.data_ptr(), tries, torch.cuda.current_stream(dev).cuda_stream)
    assert st == K.KVATTN_OK
    torch.cuda.synchronize()
    assert int(res.item()) == K.KVATTN_DEVERR_WAIT_TIMEOUT


def test_context_usable_after_a_wait_ran_out(dev, oracle_mod):
    import numpy as np
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    res = torch.zeros(1, dtype=torch.int32, device=dev)
    assert K.kvattn_selftest_bounded_wait(res.data_ptr(), 64, 0) == K.KVATTN_OK
    torch.cuda.synchronize()
    x = W.make_inputs(W.WORKLOADS["mla"].replace(batch=1, ctx=(300, 300)), seed=11)
    p = DeviceProblem(x, dev)
    p.run()
    torch.cuda.synchronize()
    out, lse = p.results()
    ref_out, ref_lse = oracle_mod.decode(x)
    assert np.abs(out - ref_out).max() <= 2e-2
    assert np.abs(lse - ref_lse).max() <= 1e-3
    assert p.device_error() == 0


def test_selftest_rejects_bad_arguments(dev):
    assert K.kvattn_selftest_bounded_wait(0, 10, 0) == K.KVATTN_ERR_INVALID_ARG
    assert K.kvattn_selftest_bounded_wait(1 << 20, 0, 0) == K.KVATTN_ERR_INVALID_ARG
    assert K.kvattn_selftest_bounded_wait(1 << 20, 70000, 0) == K.KVATTN_ERR_INVALID_ARG
    assert K.kvattn_selftest_bounded_wait((1 << 20) + 2, 10, 0) == K.KVATTN_ERR_MISALIGNED
