"""The C ABI without a GPU: the library loads, exports every declared symbol,
plans every workload, and rejects bad arguments before launching anything.

Only argument paths that return before any CUDA call are exercised here (the
fake pointers are never dereferenced)."""

import ctypes
import os
import re

import pytest

from shared_kv_caches_b200 import build as B
from shared_kv_caches_b200 import kvattn as K
from shared_kv_caches_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return K.load()


def declared_functions():
    names = []
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            text = open(os.path.join(ROOT, "include", hdr)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(kvattn_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "kvattn_decode" in names and len(names) >= 7
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        assert n in K.EXPORTS or n.startswith("kvattn_"), n


def test_version_and_status_strings(lib):
    assert K.kvattn_version() >= 100
    assert K.kvattn_status_string(0) == "ok"
    assert "workspace" in K.kvattn_status_string(K.KVATTN_ERR_WORKSPACE_TOO_SMALL)
    assert K.kvattn_status_string(-99) == "unknown status"


def _params(name, **kw):
    s = W.WORKLOADS[name]
    lo, hi = s.ctx
    mpps = (hi + 63) // 64
    p = dict(batch=s.batch, num_q_heads=s.num_q_heads, num_kv=s.num_kv, d_nope=s.d_nope, d_rope=s.d_rope,
             max_pages_per_seq=mpps, num_pages=mpps * s.batch + 1, max_seq_len=hi, num_splits=0,
             out_dtype=1 if s.out_dtype == "fp32" else 0,
             cache_dtype=K.KVATTN_CACHE_FP8_E4M3 if s.cache_dtype == "fp8" else K.KVATTN_CACHE_BF16,
             k_scale=s.k_scale, v_scale=s.v_scale)
    p.update(kw)
    return s, K.make_params(**p)


@pytest.mark.parametrize("name", sorted(W.WORKLOADS))
def test_plan_every_workload(lib, name):
    s, p = _params(name)
    plan = K.kvattn_get_plan(s.variant_id, p)
    assert plan.num_splits >= 1 and plan.pages_per_split >= 1
    assert plan.num_splits * plan.pages_per_split >= (s.ctx[1] + 63) // 64
    assert plan.launches >= 1 and plan.ctas >= 1
    rows = s.batch * plan.num_splits * s.lse_rows
    assert plan.workspace_bytes >= 256 + 4 * rows * (1 + s.d_nope)
    assert K.kvattn_workspace_size(s.variant_id, p) == plan.workspace_bytes


# (kernel, parts, pages per part, CTAs, launches) the planner picks for each
# benchmark shape at its longest context.  Latent kernels run one CTA per SM:
# a B=1 problem fills one wave of 148 CTAs (37 parts x 4 branches), larger
# batches aim at about four waves; GQA aims at four waves of three CTAs per SM
# and merges its parts in place (one launch); MQA aims at 2.5 waves.
EXPECTED_PLANS = {
    "gla": ("latent_tc", 4, 64, 512, 2),
    "gqa": ("gqa", 7, 19, 1792, 1),
    "gqa_fp8": ("gqa_fp8", 7, 19, 1792, 1),
    "mfa": ("mqa_tc", 6, 22, 192, 2),
    "mla": ("latent_pair", 5, 103, 640, 2),
    "mlra_128k": ("latent_tc", 37, 56, 148, 2),
    "mlra_512k": ("latent_tc", 37, 222, 148, 2),
    "mlra_1m": ("latent_tc", 37, 444, 148, 2),
    "mlra_b8_128k": ("latent_tc", 9, 228, 288, 2),
    "tiny_mla": ("generic", 8, 1, 16, 2),
}


@pytest.mark.parametrize("name", sorted(EXPECTED_PLANS))
def test_plan_of_each_benchmark_shape(lib, name):
    s, p = _params(name)
    plan = K.kvattn_get_plan(s.variant_id, p)
    got = (K.KERNEL_NAMES[plan.kernel], plan.num_splits, plan.pages_per_split, plan.ctas, plan.launches)
    assert got == EXPECTED_PLANS[name]
    if name.startswith("mlra"):
        # whole 128-token tiles per part
        assert plan.pages_per_split % 2 == 0


def test_forced_splits_are_clamped(lib):
    s, p = _params("gqa", num_splits=100000)
    plan = K.kvattn_get_plan(s.variant_id, p)
    assert plan.num_splits == 128 and plan.pages_per_split == 1
    s, p = _params("gqa", num_splits=7)
    plan = K.kvattn_get_plan(s.variant_id, p)
    assert plan.num_splits <= 7 and plan.num_splits * plan.pages_per_split >= 128


FAKE = 1 << 20      # 16-byte (and 256-byte) aligned, never dereferenced


def _decode(variant, p, **kw):
    args = dict(q_nope=FAKE, q_rope=FAKE, kv=FAKE, bt=FAKE, sl=FAKE, out=FAKE, lse=FAKE, ws=FAKE,
                ws_bytes=1 << 40, scale=0.1)
    args.update(kw)
    return K.kvattn_decode(variant, p, args["q_nope"], args["q_rope"], args["kv"], args["bt"], args["sl"],
                           args["scale"], args["out"], args["lse"], args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("field,value,status", [
    ("page_size", 32, K.KVATTN_ERR_UNSUPPORTED),
    ("batch", 0, K.KVATTN_ERR_INVALID_ARG),
    ("num_kv", 3, K.KVATTN_ERR_INVALID_ARG),           # MLA needs one latent
    ("d_rope", 60, K.KVATTN_ERR_UNSUPPORTED),          # not a multiple of 8
    ("d_nope", 1024, K.KVATTN_ERR_UNSUPPORTED),
    ("max_seq_len", 1 << 30, K.KVATTN_ERR_INVALID_ARG),  # beyond capacity
    ("out_dtype", 7, K.KVATTN_ERR_INVALID_ARG),
])
def test_bad_params_rejected(lib, field, value, status):
    s, p = _params("mla", **{field: value})
    assert _decode(s.variant_id, p) == status


def test_bad_variant_and_shapes(lib):
    s, p = _params("gqa")
    assert _decode(9, p) == K.KVATTN_ERR_UNSUPPORTED
    s, p = _params("gqa", num_kv=5)                     # 32 heads do not split into 5 groups
    assert _decode(K.KVATTN_GQA, p) == K.KVATTN_ERR_INVALID_ARG
    s, p = _params("gqa", d_rope=64)                    # GQA has no rope key
    assert _decode(K.KVATTN_GQA, p) == K.KVATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("which", ["q_nope", "kv", "sl", "out", "ws"])
def test_null_pointers_rejected(lib, which):
    s, p = _params("gla")
    assert _decode(s.variant_id, p, **{which: None}) == K.KVATTN_ERR_INVALID_ARG


def test_missing_rope_query_rejected(lib):
    s, p = _params("mlra_128k")
    assert _decode(s.variant_id, p, q_rope=None) == K.KVATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("which", ["q_nope", "q_rope", "kv", "out", "ws"])
def test_misaligned_pointers_rejected(lib, which):
    s, p = _params("mla")
    assert _decode(s.variant_id, p, **{which: FAKE + 8}) == K.KVATTN_ERR_MISALIGNED


def test_small_workspace_rejected(lib):
    s, p = _params("mla")
    need = K.kvattn_workspace_size(s.variant_id, p)
    assert _decode(s.variant_id, p, ws_bytes=need - 1) == K.KVATTN_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("field,value,status", [
    ("k_scale", 0.0, K.KVATTN_ERR_INVALID_ARG),
    ("k_scale", -1.0, K.KVATTN_ERR_INVALID_ARG),
    ("v_scale", float("nan"), K.KVATTN_ERR_INVALID_ARG),
    ("v_scale", float("inf"), K.KVATTN_ERR_INVALID_ARG),
    ("cache_dtype", 2, K.KVATTN_ERR_INVALID_ARG),
    ("d_nope", 64, K.KVATTN_ERR_UNSUPPORTED),           # the fp8 kernel holds 128-dim heads
    ("num_kv", 16, K.KVATTN_ERR_UNSUPPORTED),           # 2 query heads per KV head
])
def test_bad_fp8_params_rejected(lib, field, value, status):
    s, p = _params("gqa_fp8", **{field: value})
    assert _decode(s.variant_id, p) == status


@pytest.mark.parametrize("name", ["mfa", "mla", "gla", "mlra_128k", "gta"])
def test_fp8_cache_only_for_gqa(lib, name):
    s, p = _params(name, cache_dtype=K.KVATTN_CACHE_FP8_E4M3, k_scale=1.0, v_scale=1.0)
    assert _decode(s.variant_id, p) == K.KVATTN_ERR_UNSUPPORTED
    with pytest.raises(K.KvattnError):
        K.kvattn_get_plan(s.variant_id, p)


def test_non_finite_scale_rejected(lib):
    s, p = _params("gqa")
    assert _decode(s.variant_id, p, scale=float("nan")) == K.KVATTN_ERR_INVALID_ARG


def test_workspace_init_and_error_query_args(lib):
    assert K.kvattn_workspace_init(None, 4096, None) == K.KVATTN_ERR_INVALID_ARG
    assert K.kvattn_workspace_init(FAKE, 16, None) == K.KVATTN_ERR_INVALID_ARG
    assert K.kvattn_workspace_init(FAKE + 16, 4096, None) == K.KVATTN_ERR_MISALIGNED
    code = ctypes.c_int32(0)
    assert lib.kvattn_get_device_error(None, None, ctypes.byref(code)) == K.KVATTN_ERR_INVALID_ARG
