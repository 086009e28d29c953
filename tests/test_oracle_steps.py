"""Pins of the oracle of the steps either side of attention (oracle/steps.py):
rotary embedding, cache append, query absorption and the up-projection.

Each test relies on a fact fixed by the pages or by mathematics, reached by a
route other than the function under test: a closed form of a rotation, the
complex-number form of RoPE, norm and relative-position invariance, brute
force over the page pool, the materialised keys and values of the MLA
explainer (sections 2.2-2.3), and the MLRA page's per-branch form.
"""

import math

import numpy as np
import pytest

from oracle import oracle, steps


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ RoPE
def test_rope_two_wide_is_a_plane_rotation():
    """A 2-wide vector has one pair with angle pos * base^0 = pos: (1, 0) goes to (cos pos, sin pos)."""
    for pos in (0, 1, 3, 100):
        y = steps.rope(np.array([1.0, 0.0]), pos, 10000.0)
        np.testing.assert_allclose(y, [math.cos(pos), math.sin(pos)], rtol=0, atol=1e-15)


def test_rope_frequency_schedule_and_pairing():
    """d = 4, base 100: pair 0 turns at rate 1, pair 1 (entries 2, 3) at rate
    100^(-1/2) = 0.1.  At pos = 10 pi pair 0 is back where it was and pair 1 is
    turned by pi (negated).  A half-split pairing ((0, 2), (1, 3)) or another
    exponent gives a different vector."""
    x = np.array([0.3, -1.2, 0.7, 2.5])
    y = steps.rope(x, 10 * math.pi, 100.0)
    np.testing.assert_allclose(y, [0.3, -1.2, -0.7, -2.5], rtol=0, atol=1e-12)


def test_rope_is_complex_multiplication():
    """RoPE treats (x[2i], x[2i+1]) as x[2i] + j x[2i+1] multiplied by exp(j pos theta_i)."""
    rng = _rng(1)
    x = rng.standard_normal((5, 64))
    pos = np.array([0, 1, 17, 4095, 131071])
    theta = 10000.0 ** (-np.arange(32) / 32.0)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * pos[:, None] * theta)
    y = steps.rope(x, pos, 10000.0)
    np.testing.assert_allclose(y[:, 0::2], z.real, rtol=0, atol=1e-11)
    np.testing.assert_allclose(y[:, 1::2], z.imag, rtol=0, atol=1e-11)


def test_rope_keeps_pair_norms_and_scores_depend_on_offset_only():
    rng = _rng(2)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in ((5, 2), (1000, 37), (0, 0)):
        qm, kn = steps.rope(q, m, 10000.0), steps.rope(k, n, 10000.0)
        np.testing.assert_allclose(qm[0::2] ** 2 + qm[1::2] ** 2, q[0::2] ** 2 + q[1::2] ** 2, rtol=1e-12)
        for t in (1, 64, 5000):
            shifted = steps.rope(q, m + t, 10000.0) @ steps.rope(k, n + t, 10000.0)
            assert abs(shifted - qm @ kn) < 1e-10
        # the score is q against k turned by the offset n - m
        assert abs(q @ steps.rope(k, n - m, 10000.0) - qm @ kn) < 1e-10
    np.testing.assert_array_equal(steps.rope(q, 0, 10000.0), q)


# ---------------------------------------------------------------- append
def _pool(rng, B, mpps, width, spare=3):
    pages = rng.permutation(B * mpps + spare)[:B * mpps].reshape(B, mpps).astype(np.int32)
    cache = rng.standard_normal((B * mpps + spare, 64, width))
    return pages, cache


def test_append_latent_places_rows_by_the_block_table():
    """Every written row is found again by scanning the pool page by page (the
    inverse of the block table); every other row is untouched; the rope slice
    is the rotated one."""
    rng = _rng(3)
    B, Q, mpps, dn, dr = 3, 2, 4, 10, 4
    pages, cache = _pool(rng, B, mpps, dn + dr)
    rows = rng.standard_normal((B, Q, dn + dr))
    pos = np.array([[0, 1], [63, 64], [200, 255]])
    new = steps.append_latent(cache, rows, pos, pages, dr, 10000.0)
    owner = {}
    for b in range(B):
        for i, pg in enumerate(pages[b]):
            owner[int(pg)] = (b, i)
    written = set()
    for pg in range(cache.shape[0]):
        for slot in range(64):
            hit = None
            if pg in owner:
                b, i = owner[pg]
                for q in range(Q):
                    if pos[b, q] == i * 64 + slot:
                        hit = (b, q)
            if hit is None:
                np.testing.assert_array_equal(new[pg, slot], cache[pg, slot])
            else:
                b, q = hit
                written.add(hit)
                np.testing.assert_array_equal(new[pg, slot, :dn], rows[b, q, :dn])
                y = rows[b, q, dn:]
                z = (y[0::2] + 1j * y[1::2]) * np.exp(1j * pos[b, q] * 10000.0 ** (-np.arange(dr // 2) * 2.0 / dr))
                np.testing.assert_allclose(new[pg, slot, dn::2], z.real, atol=1e-12)
                np.testing.assert_allclose(new[pg, slot, dn + 1::2], z.imag, atol=1e-12)
    assert len(written) == B * Q


def test_append_heads_rotates_keys_only():
    rng = _rng(4)
    B, Q, nkv, D = 2, 1, 2, 8
    pages = np.array([[2, 0], [1, 3]], dtype=np.int32)
    cache = rng.standard_normal((4, 2, 64, nkv, D))
    kv = rng.standard_normal((B, Q, 2, nkv, D))
    pos = np.array([[70], [5]])
    new = steps.append_heads(cache, kv, pos, pages, 500.0)
    np.testing.assert_array_equal(new[0, 1, 6], kv[0, 0, 1])          # V of sequence 0 at slot 70
    np.testing.assert_allclose(new[0, 0, 6, 1], steps.rope(kv[0, 0, 0, 1], 70, 500.0), atol=1e-14)
    np.testing.assert_array_equal(new[1, 1, 5], kv[1, 0, 1])
    norm = lambda v: v[..., 0::2] ** 2 + v[..., 1::2] ** 2
    np.testing.assert_allclose(norm(new[1, 0, 5]), norm(kv[1, 0, 0]), rtol=1e-12)
    untouched = np.ones((4, 2, 64), bool)
    untouched[0, :, 6] = untouched[1, :, 5] = False
    np.testing.assert_array_equal(new[untouched], cache[untouched])


# ------------------------------------------- absorption and up-projection
def test_head_proj_against_loops():
    rng = _rng(5)
    x, w = rng.standard_normal((3, 2, 5)), rng.standard_normal((2, 5, 4))
    y = steps.head_proj(x, w)
    for r in range(3):
        for h in range(2):
            for n in range(4):
                assert abs(y[r, h, n] - sum(x[r, h, k] * w[h, k, n] for k in range(5))) < 1e-12


def test_absorbed_query_scores_equal_materialised_key_scores():
    """MLRA page, MLA paragraph: absorbing W_UK into the query leaves the
    scores unchanged: (q^C W_UK[h]) . c == q^C . (W_UK[h] c)."""
    rng = _rng(6)
    H, dh, dc, L = 3, 8, 12, 9
    q_c, w_uk = rng.standard_normal((1, H, dh)), rng.standard_normal((H, dh, dc))
    c = rng.standard_normal((L, dc))
    q_abs = steps.head_proj(q_c, w_uk)[0]                  # [H][dc]
    for h in range(H):
        keys = c @ w_uk[h].T                               # [L][dh], materialised
        np.testing.assert_allclose(q_abs[h] @ c.T, keys @ q_c[0, h], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("R", [1, 4])
def test_absorbed_decode_chain_equals_materialised_attention(R):
    """The whole absorbed path -- append the new token with its rotated k^R,
    absorb W_UK into the query, attend the latent cache (one output per
    branch), up-project with W_UV stacked over the branches -- against
    explicit per-head keys and values (MLA explainer 2.2-2.3; MLRA per-branch
    form with the branch outputs summed)."""
    rng = _rng(10 + R)
    H, dh, dc, dr, dv, L, base = 3, 8, 6, 4, 5, 70, 10000.0
    q_c = rng.standard_normal((H, R, dh))
    q_r_raw = rng.standard_normal((H, R, dr))
    latent = rng.standard_normal((L, R, dc))
    k_r_raw = rng.standard_normal((L, dr))
    w_uk = rng.standard_normal((H, R, dh, dc))
    w_uv = rng.standard_normal((H, R, dc, dv))
    scale = 1 / math.sqrt(dh + dr)
    pos_q = L - 1
    ref = steps.materialized_attention(q_c, steps.rope(q_r_raw, pos_q, base), latent,
                                       steps.rope(k_r_raw, np.arange(L), base), w_uk, w_uv, scale)

    # the cache: one sequence, two pages, tokens appended one by one
    rows = np.concatenate([latent.reshape(L, R * dc), k_r_raw], axis=1)
    cache = np.full((2, 64, R * dc + dr), np.nan)
    for j in range(L):
        cache = steps.append_latent(cache, rows[j][None, None], np.array([[j]]), None, dr, base)
    # absorption: one projection per head with the branches' W_UK side by side
    w_abs = np.concatenate([w_uk[:, r] for r in range(R)], axis=2)           # [H][dh][R dc]
    q_nope = np.stack([steps.head_proj(q_c[None, :, r], w_uk[:, r])[0] for r in range(R)], axis=1)
    if R > 1:
        np.testing.assert_allclose(q_nope.reshape(H, R * dc),
                                   np.einsum("hrk,hkn->hrn", q_c, w_abs).reshape(H, R, R, dc)
                                   [:, np.arange(R), np.arange(R)].reshape(H, R * dc), rtol=1e-12)
    q_rope = steps.rope(q_r_raw, pos_q, base)
    variant = "mla" if R == 1 else "mlra"
    qn = q_nope[None] if R > 1 else q_nope[None, :, 0]
    qr = q_rope[None] if R > 1 else q_rope[None, :, 0]
    o_lat, _ = oracle.decode_f64(variant, R, qn, qr, cache, np.array([L], np.int32), scale, branch_out=True)
    o = steps.head_proj(o_lat.reshape(1, H, R * dc), w_uv.reshape(H, R * dc, dv))[0]
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)
