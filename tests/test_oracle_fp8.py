"""Pins of the oracle's fp8 (e4m3) cache path: the code decoder against the
format's landmark values, the generator's independent encoder and
monotonicity; the attention over the dequantised cache against brute force
and against the scaling identity that places k_scale in the scores and
v_scale on the output."""

import math

import numpy as np
import pytest

from shared_kv_caches_b200 import workloads as W


def test_e4m3_landmark_codes(oracle_mod):
    """Sign bit 7, exponent bits 6..3 with bias 7, mantissa bits 2..0;
    exponent 0 subnormal; S.1111.111 NaN, no infinities."""
    v = oracle_mod.e4m3_value
    cases = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3F: 1.875,
             0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for code, want in cases.items():
        assert v(code) == want, hex(code)
    assert math.copysign(1.0, v(0x80)) == -1.0 and v(0x80) == 0.0
    assert np.isnan(v(0x7F)) and np.isnan(v(0xFF))


def test_e4m3_codes_are_monotone_and_round_trip_through_the_encoder(oracle_mod):
    codes = np.arange(0x7F)
    vals = oracle_mod.e4m3_value(codes)
    assert np.all(np.diff(vals) > 0)
    np.testing.assert_array_equal(oracle_mod.e4m3_value(codes | 0x80), -vals)
    every = np.concatenate([codes, codes | 0x80])
    np.testing.assert_array_equal(W.f32_to_e4m3_bits(oracle_mod.e4m3_value(every)), every)


def _tiny(seed, **kw):
    s = W.WORKLOADS["gqa_fp8"].replace(batch=2, num_q_heads=8, num_kv=2, d_nope=16, ctx=(5, 140), **kw)
    return W.make_inputs(s, seed=seed)


def test_fp8_attention_brute_force(oracle_mod):
    """numpy softmax(scale q K^T) V with K = k_scale * K8 and V = v_scale * V8
    gathered by fancy indexing over the pool."""
    x = _tiny(3)
    s = x["shape"]
    out, lse = oracle_mod.decode(x)
    kv = oracle_mod.e4m3_value(x["kv"])
    q = (np.asarray(x["q_nope"], np.uint32) << 16).view(np.float32).astype(np.float64)
    for b in range(s.batch):
        L = int(x["seq_lens"][b])
        j = np.arange(L)
        pages = x["block_table"][b, j // 64]
        for h in range(s.num_q_heads):
            u = h // (s.num_q_heads // s.num_kv)
            K = s.k_scale * kv[pages, 0, j % 64, u]
            V = s.v_scale * kv[pages, 1, j % 64, u]
            sc = x["sm_scale"] * (K @ q[b, h])
            p = np.exp(sc - sc.max())
            np.testing.assert_allclose(out[b, h], (p / p.sum()) @ V, rtol=1e-12, atol=1e-12)
            assert abs(lse[b, h] - (sc.max() + np.log(p.sum()))) < 1e-12


@pytest.mark.parametrize("ks,vs", [(0.5, 2.0), (3.0, 0.25)])
def test_fp8_scales_enter_scores_and_output(oracle_mod, ks, vs):
    """out(k_scale, v_scale, sm_scale) = v_scale * out(1, 1, sm_scale * k_scale)
    and the lse depends on k_scale only through sm_scale * k_scale."""
    x = _tiny(4, k_scale=ks, v_scale=vs)
    y = dict(x, shape=x["shape"].replace(k_scale=1.0, v_scale=1.0))
    out, lse = oracle_mod.decode(x)
    out1, lse1 = oracle_mod.decode(y, sm_scale=x["sm_scale"] * ks)
    np.testing.assert_allclose(out, vs * out1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, lse1, rtol=0, atol=1e-12)
