"""The seeded input generator: bf16 rounding, pool placement and poison."""

import numpy as np

from shared_kv_caches_b200 import workloads as W


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 1e4, 3.0e38], dtype=np.float32)
    b = W.f32_to_bf16_bits(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert list(b[:4]) == [0x3F80, 0x3F80, 0x3F82, 0xC020]
    assert b[4] == W.BF16_POS_1E4
    back = W.bf16_bits_to_f32(b)
    assert back[3] == -2.5 and back[4] == 9984.0


def test_e4m3_round_to_nearest_even_and_saturate():
    e = W.f32_to_e4m3_bits
    # 1 + 2^-4 is a tie between 1.0 (0x38) and 1.125 (0x39): the even code wins;
    # 1 + 3 * 2^-4 ties 1.125 and 1.25: 0x3A
    assert list(e([1.0625, 1.0625 + 1e-6, 1.1875, -1.0625])) == [0x38, 0x39, 0x3A, 0xB8]
    # subnormals are multiples of 2^-9: 2^-10 ties 0 and 2^-9, 3 * 2^-10 and
    # 5 * 2^-10 tie onto 2 * 2^-9; 7.75 * 2^-9 rounds up to the smallest normal
    assert list(e([2.0 ** -10, 3 * 2.0 ** -10, 5 * 2.0 ** -10, 7.75 * 2.0 ** -9])) == [0x00, 0x02, 0x02, 0x08]
    assert list(e([448.0, 460.0, 1e9, np.inf, -np.inf])) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]
    assert e(np.nan) == 0x7F
    assert e(0.0) == 0x00 and e(-0.0) == 0x80


def test_e4m3_midpoints_between_every_pair_of_codes(oracle_mod):
    """Brute force over the format: halfway between neighbouring finite codes
    goes to the even code, a little above halfway to the upper one."""
    codes = np.arange(0x7E)
    lo, hi = oracle_mod.e4m3_value(codes), oracle_mod.e4m3_value(codes + 1)
    mid = (lo + hi) / 2
    even = np.where(codes % 2 == 0, codes, codes + 1)
    np.testing.assert_array_equal(W.f32_to_e4m3_bits(mid), even)
    np.testing.assert_array_equal(W.f32_to_e4m3_bits(mid + (hi - lo) * 1e-3), codes + 1)
    np.testing.assert_array_equal(W.f32_to_e4m3_bits(-mid), even | 0x80)


def test_fp8_cache_draws_and_poison():
    s = W.WORKLOADS["gqa_fp8"].replace(batch=3, ctx=(5, 140))
    x = W.make_inputs(s, seed=2, seq_lens=[5, 64, 140])
    assert x["kv"].dtype == np.uint8 and x["kv"].shape == s.pool_shape(x["kv"].shape[0])
    inside = []
    for b, L in enumerate([5, 64, 140]):
        for j in range(L):
            page, slot = W.token_location(x, b, j)
            inside.append(x["kv"][page, :, slot])
    inside = np.concatenate([v.ravel() for v in inside])
    assert not np.isin(inside, [0x7F, 0xFF]).any()           # no NaN inside any context
    # slot 5 of the first sequence's page is past its context: poison codes only
    page, _ = W.token_location(x, 0, 0)
    assert np.isin(x["kv"][page, :, 5:], W.POISON_FP8).all()


def test_deterministic_and_seeded():
    s = W.Shape("gqa", 3, 8, 2, 16, 0, (10, 200))
    a = W.make_inputs(s, seed=4)
    b = W.make_inputs(s, seed=4)
    c = W.make_inputs(s, seed=5)
    for k in ("seq_lens", "q_nope", "kv", "block_table"):
        np.testing.assert_array_equal(a[k], b[k])
    assert not np.array_equal(a["kv"], c["kv"])


def test_pool_pages_and_poison_layout():
    s = W.Shape("mla", 4, 2, 1, 8, 4, (1, 300))
    x = W.make_inputs(s, seed=1, seq_lens=[1, 64, 65, 300])
    bt = x["block_table"]
    need = [1, 1, 2, 5]
    used = [int(bt[b, i]) for b in range(4) for i in range(need[b])]
    assert len(set(used)) == len(used)              # every logical page has its own frame
    assert x["num_pages"] == sum(need) + 1          # 1% spare, at least one
    spare = sorted(set(range(x["num_pages"])) - set(used))
    assert len(spare) == 1
    kv = x["kv"]
    assert np.isin(kv[spare[0]], W.POISON_BITS).all()
    # sequence 2: 65 tokens, slot 0 of its second page is data, slots 1.. poison
    p = bt[2, 1]
    assert not np.isin(kv[p, 0], W.POISON_BITS).all()
    assert np.isin(kv[p, 1:], W.POISON_BITS).all()
    # unused block-table entries point at spare frames
    assert set(bt[0, 1:].tolist()) <= set(spare)


def test_gqa_pool_shape_and_contiguous_mode():
    s = W.Shape("gqa", 2, 8, 2, 16, 0, (100, 100), paged=False)
    x = W.make_inputs(s, seed=0)
    assert x["block_table"] is None
    assert x["kv"].shape == (2 * 2, 2, 64, 2, 16)
    loc = W.token_location(x, 1, 70)
    assert loc == (3, 6)
    # contiguous mode: tokens past the context of the second page are poison
    assert np.isin(x["kv"][1, :, 36:], W.POISON_BITS).all()


def test_named_workloads_shapes():
    wl = W.WORKLOADS
    assert wl["mla"].key_dim == 576 and wl["mla"].row_elems == 576
    assert wl["gla"].row_elems == 576 and wl["gla"].key_dim == 320
    assert wl["mlra_1m"].row_elems == 576 and wl["mlra_1m"].key_dim == 192
    assert wl["tiny_mla"].key_dim == 80 and abs(wl["tiny_mla"].scale - 80 ** -0.5) < 1e-15
    assert wl["gqa"].row_elems == 8 * 128
    assert wl["mlra_128k"].lse_shape() == (1, 128, 4)
