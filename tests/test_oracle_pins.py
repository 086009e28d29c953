"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Each test states the passage or identity it relies on.  None of them compares
the oracle with a re-typed copy of itself: they use closed forms, structural
identities between variants (absorbed MLA vs explicit up-projection, MLRA with
one branch vs MLA, GLA as two MLA problems, GQA as MHA with repeated heads),
special cases that reduce to a textbook routine (a mean, a one-hot softmax),
the split-merge identity, and brute force through numpy's matrix routines on
tiny inputs.
"""

import json
import math
import os

import numpy as np
import pytest

from shared_kv_caches_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _tiny_f64(variant, B=2, H=4, NU=2, dn=6, dr=3, lens=(5, 3), ps=2, seed=0):
    """Small float64 problem in the library layouts with a permuted page pool."""
    rng = _rng(seed)
    latent = variant in ("mla", "gla", "mlra")
    if variant == "mla":
        NU = 1
    if variant == "mqa":
        NU = 1
    if not latent:
        dr = 0
    need = [(L + ps - 1) // ps for L in lens]
    mpps = max(need) + 1
    num_pages = sum(need) + 2
    if latent:
        kv = rng.standard_normal((num_pages, ps, NU * dn + dr))
    elif variant == "gta":
        kv = rng.standard_normal((num_pages, ps, NU, dn))
    else:
        kv = rng.standard_normal((num_pages, 2, ps, NU, dn))
    perm = rng.permutation(num_pages)
    bt = np.zeros((B, mpps), dtype=np.int32)
    k = 0
    for b in range(B):
        bt[b, :need[b]] = perm[k:k + need[b]]
        bt[b, need[b]:] = perm[-1]
        k += need[b]
    if variant == "mlra":
        qn = rng.standard_normal((B, H, NU, dn))
        qr = rng.standard_normal((B, H, NU, dr))
    else:
        qn = rng.standard_normal((B, H, dn))
        qr = rng.standard_normal((B, H, dr)) if dr else None
    return dict(variant=variant, NU=NU, dn=dn, dr=dr, ps=ps, kv=kv, bt=bt,
                lens=np.array(lens, dtype=np.int32), qn=qn, qr=qr, B=B, H=H)


def _run(oracle_mod, P, scale=0.37, bt=None, lens=None):
    return oracle_mod.decode_f64(P["variant"], P["NU"], P["qn"], P["qr"], P["kv"],
                                 P["lens"] if lens is None else lens, scale,
                                 block_table=P["bt"] if bt is None else bt, page_size=P["ps"])


def _gather_rows(P, b):
    """Token rows of sequence b, in order, via numpy fancy indexing."""
    L = int(P["lens"][b])
    j = np.arange(L)
    pages = P["bt"][b, j // P["ps"]]
    return pages, j % P["ps"]


def _softmax_attend(q, K, V, scale):
    """Brute force with numpy's matrix product: softmax(scale q K^T) V and lse."""
    s = scale * (K @ q)
    m = s.max()
    e = np.exp(s - m)
    return (e / e.sum()) @ V, m + np.log(e.sum())


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("variant", ["gqa", "mqa", "mla", "gla", "mlra"])
def test_brute_force_tiny(oracle_mod, variant):
    """Brute force on tiny inputs: numpy softmax(QK^T)V per (b, h[, r]).

    The keys and values are taken with numpy fancy indexing of the whole pool
    (a different route from the oracle's per-element addressing), so a wrong
    page, slot, unit, rope offset or K/V plane fails here.
    """
    P = _tiny_f64(variant, H=4, NU=2, seed=11)
    scale = 0.37
    out, lse = _run(oracle_mod, P, scale)
    B, H, NU, dn, dr = P["B"], P["H"], P["NU"], P["dn"], P["dr"]
    for b in range(B):
        pages, slots = _gather_rows(P, b)
        for h in range(H):
            if variant == "mlra":
                acc = np.zeros(dn)
                for r in range(NU):
                    rows = P["kv"][pages, slots]            # [L][row]
                    K = np.concatenate([rows[:, r * dn:(r + 1) * dn], rows[:, NU * dn:]], axis=1)
                    V = rows[:, r * dn:(r + 1) * dn]
                    q = np.concatenate([P["qn"][b, h, r], P["qr"][b, h, r]])
                    o, l = _softmax_attend(q, K, V, scale)
                    acc += o
                    assert abs(lse[b, h, r] - l) < 1e-12
                np.testing.assert_allclose(out[b, h], acc, rtol=0, atol=1e-12)
                continue
            if variant in ("mla", "gla"):
                g = 0 if variant == "mla" else h // (H // NU)
                rows = P["kv"][pages, slots]
                K = np.concatenate([rows[:, g * dn:(g + 1) * dn], rows[:, NU * dn:]], axis=1)
                V = rows[:, g * dn:(g + 1) * dn]
                q = np.concatenate([P["qn"][b, h], P["qr"][b, h]])
            else:
                g = h // (H // NU)
                K = P["kv"][pages, 0, slots, g]
                V = P["kv"][pages, 1, slots, g]
                q = P["qn"][b, h]
            o, l = _softmax_attend(q, K, V, scale)
            np.testing.assert_allclose(out[b, h], o, rtol=0, atol=1e-12)
            assert abs(lse[b, h] - l) < 1e-12


# ---------------------------------------------------------------- closed forms

def test_golden_closed_form_mla(oracle_mod):
    """Hand-worked MLA example (MLA explainer, section 2.3 formula).

    The fixture states inputs chosen so the scores are small integers; the
    expected output and lse are the closed forms written out in the fixture.
    """
    with open(os.path.join(GOLDEN, "mla_closed_form.json")) as f:
        g = json.load(f)
    rows = np.array(g["rows"], dtype=np.float64)          # [L][d_c + d_r]
    L = rows.shape[0]
    kv = rows.reshape(1, L, rows.shape[1])
    qn = np.array(g["q_nope"], dtype=np.float64).reshape(1, 1, -1)
    qr = np.array(g["q_rope"], dtype=np.float64).reshape(1, 1, -1)
    out, lse = oracle_mod.decode_f64("mla", 1, qn, qr, kv, np.array([L], np.int32), g["sm_scale"],
                                     page_size=L)
    e2 = math.exp(2.0)
    Z = 2.0 + e2
    expect = [(e2 - 1.0) / Z, 6.0 / Z]
    assert g["scores"] == [0.0, 2.0, 0.0]
    np.testing.assert_allclose(out[0, 0], expect, rtol=1e-14)
    np.testing.assert_allclose(out[0, 0], g["expected_out"], rtol=1e-14)
    assert abs(lse[0, 0] - math.log(Z)) < 1e-14
    assert abs(lse[0, 0] - g["expected_lse"]) < 1e-14


def test_two_token_closed_form(oracle_mod):
    """Two tokens with scores 0 and t: p = (1, e^t) / (1 + e^t), lse = ln(1 + e^t)."""
    t = 1.25
    dn = 4
    kv = np.zeros((1, 2, 2, 1, dn))
    kv[0, 0, 1, 0, 0] = t                     # k_1 = t e_0, k_0 = 0
    v0 = np.array([1.0, -2.0, 0.5, 3.0])
    v1 = np.array([-1.0, 4.0, 2.0, 0.0])
    kv[0, 1, 0, 0] = v0
    kv[0, 1, 1, 0] = v1
    qn = np.zeros((1, 1, dn))
    qn[0, 0, 0] = 1.0
    out, lse = oracle_mod.decode_f64("mqa", 1, qn, None, kv, np.array([2], np.int32), 1.0,
                                     page_size=2)
    w1 = math.exp(t) / (1.0 + math.exp(t))
    np.testing.assert_allclose(out[0, 0], (1 - w1) * v0 + w1 * v1, rtol=1e-14, atol=1e-15)
    assert abs(lse[0, 0] - math.log1p(math.exp(t))) < 1e-14


def test_ctx1_returns_value_exactly(oracle_mod):
    """A context of one token returns its value exactly and lse = scale*q.k."""
    inputs = W.make_inputs(W.Shape("mla", 3, 4, 1, 32, 8, (1, 1)), seed=5)
    out, lse = oracle_mod.decode(inputs)
    for b in range(3):
        page, slot = W.token_location(inputs, b, 0)
        row = W.bf16_bits_to_f32(inputs["kv"][page, slot]).astype(np.float64)
        for h in range(4):
            assert np.array_equal(out[b, h], row[:32])
            q = np.concatenate([W.bf16_bits_to_f32(inputs["q_nope"][b, h]),
                                W.bf16_bits_to_f32(inputs["q_rope"][b, h])]).astype(np.float64)
            assert abs(lse[b, h] - inputs["sm_scale"] * float(q @ row)) < 1e-12


def test_softmax_weights_sum_to_one(oracle_mod):
    """One-hot values expose the weights: out = p, sum(p) = 1, p_j = exp(s_j - lse)."""
    L, dn, dr = 7, 8, 2
    rng = _rng(3)
    rows = np.zeros((1, L, dn + dr))
    rows[0, np.arange(L), np.arange(L)] = 1.0          # c_j = e_j
    rows[0, :, dn:] = rng.standard_normal((L, dr))
    qn = rng.standard_normal((1, 2, dn))
    qr = rng.standard_normal((1, 2, dr))
    scale = 0.9
    out, lse = oracle_mod.decode_f64("mla", 1, qn, qr, rows, np.array([L], np.int32), scale,
                                     page_size=L)
    for h in range(2):
        p = out[0, h, :L]
        assert abs(p.sum() - 1.0) < 1e-15
        s = scale * (qn[0, h, :L] + rows[0, :, dn:] @ qr[0, h])
        np.testing.assert_allclose(p, np.exp(s - lse[0, h]), rtol=1e-13)
        assert np.all(out[0, h, L:] == 0.0)


def test_constant_values_return_the_value(oracle_mod):
    """If every value row is w, the output is w whatever the scores."""
    P = _tiny_f64("gqa", lens=(5, 4), seed=4)
    w = np.array([0.25, -1.5, 3.0, 0.0, 2.0, -0.75])
    P["kv"][:, 1] = w
    out, _ = _run(oracle_mod, P, 0.8)
    np.testing.assert_allclose(out, np.broadcast_to(w, out.shape), rtol=1e-15, atol=1e-15)


def test_zero_scale_is_mean_of_values(oracle_mod):
    """sm_scale = 0 makes every weight 1/L: out = mean_j v_j, lse = ln L."""
    P = _tiny_f64("gla", H=4, NU=2, lens=(5, 3), seed=9)
    out, lse = _run(oracle_mod, P, 0.0)
    for b in range(2):
        L = int(P["lens"][b])
        j = np.arange(L)
        rows = P["kv"][P["bt"][b, j // P["ps"]], j % P["ps"]]
        for h in range(4):
            g = h // 2
            np.testing.assert_allclose(out[b, h], np.mean(rows[:, g * 6:(g + 1) * 6], axis=0),
                                       rtol=1e-14, atol=1e-15)
            assert abs(lse[b, h] - math.log(L)) < 1e-14


def test_empty_sequence(oracle_mod):
    """seq_len = 0: out = 0 and lse = -inf (reading taken where the pages are silent)."""
    P = _tiny_f64("mla", lens=(0, 3), seed=2)
    out, lse = _run(oracle_mod, P, 0.5)
    assert np.all(out[0] == 0.0)
    assert np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


# ---------------------------------------------------------------- structure

def test_absorbed_mla_equals_explicit(oracle_mod):
    """Absorbing W_UK into the query (MLRA page: MLA paragraph on absorption;
    it makes MLA a 576-d MQA) equals the explicit per-head up-projection of
    keys and values followed by standard attention (MLA explainer, sections
    2.2-2.3)."""
    rng = _rng(21)
    B, H, dc, dr, dh, L = 2, 3, 12, 4, 5, 9
    c = rng.standard_normal((B, L, dc))
    kr = rng.standard_normal((B, L, dr))
    W_UK = rng.standard_normal((H, dh, dc))
    W_UV = rng.standard_normal((H, dh, dc))
    q_c = rng.standard_normal((B, H, dh))
    q_r = rng.standard_normal((B, H, dr))
    scale = 1.0 / math.sqrt(dh + dr)

    # explicit: k_h = W_UK[h] c, v_h = W_UV[h] c, scores over [q_c ; q_r] . [k_h ; k_r]
    explicit = np.zeros((B, H, dh))
    for b in range(B):
        for h in range(H):
            K = np.concatenate([c[b] @ W_UK[h].T, kr[b]], axis=1)
            V = c[b] @ W_UV[h].T
            explicit[b, h], _ = _softmax_attend(np.concatenate([q_c[b, h], q_r[b, h]]), K, V, scale)

    # absorbed: q_nope = W_UK[h]^T q_c, attend the cached [c ; k_r] rows, then W_UV
    q_nope = np.einsum("hkc,bhk->bhc", W_UK, q_c)
    pool = np.concatenate([c, kr], axis=2)                       # [B][L][dc+dr], contiguous
    o_lat, _ = oracle_mod.decode_f64("mla", 1, q_nope, q_r, pool, np.full(B, L, np.int32), scale,
                                     page_size=L)
    absorbed = np.einsum("hkc,bhc->bhk", W_UV, o_lat)
    np.testing.assert_allclose(absorbed, explicit, rtol=1e-12, atol=1e-12)


def test_mlra_one_branch_is_mla(oracle_mod):
    """MLRA with a single branch is MLA (the block decomposition with one block)."""
    P = _tiny_f64("mla", H=4, seed=31)
    out_mla, lse_mla = _run(oracle_mod, P, 0.6)
    Q = dict(P, variant="mlra", qn=P["qn"][:, :, None, :], qr=P["qr"][:, :, None, :])
    out_r, lse_r = _run(oracle_mod, Q, 0.6)
    np.testing.assert_allclose(out_r, out_mla, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse_r[:, :, 0], lse_mla, rtol=0, atol=1e-14)


def test_mlra_is_sum_of_branch_mla(oracle_mod):
    """MLRA-R = sum over branches of MLA on the branch slice [c_r ; k_rope]
    (MLRA page, "moving the sum outside": attention per branch, then sum)."""
    P = _tiny_f64("mlra", H=4, NU=4, dn=5, dr=3, seed=41)
    out, lse = _run(oracle_mod, P, 0.45)
    acc = np.zeros_like(out)
    for r in range(4):
        sl = np.concatenate([P["kv"][..., r * 5:(r + 1) * 5], P["kv"][..., 20:]], axis=-1)
        Q = dict(P, variant="mla", NU=1, kv=sl, qn=P["qn"][:, :, r], qr=P["qr"][:, :, r])
        o, l = _run(oracle_mod, Q, 0.45)
        acc += o
        np.testing.assert_allclose(lse[:, :, r], l, rtol=0, atol=1e-13)
    np.testing.assert_allclose(out, acc, rtol=0, atol=1e-13)


def test_gla_is_two_mla_problems(oracle_mod):
    """GLA-2 = MLA on (c_0, k_rope) for heads 0..H/2-1 and MLA on (c_1, k_rope)
    for heads H/2..H-1 (GLA page: each latent head serves one query group)."""
    P = _tiny_f64("gla", H=6, NU=2, dn=4, dr=2, seed=51)
    out, lse = _run(oracle_mod, P, 0.7)
    for g in range(2):
        hs = slice(3 * g, 3 * g + 3)
        sl = np.concatenate([P["kv"][..., g * 4:(g + 1) * 4], P["kv"][..., 8:]], axis=-1)
        Q = dict(P, variant="mla", NU=1, H=3, kv=sl, qn=P["qn"][:, hs], qr=P["qr"][:, hs])
        o, l = _run(oracle_mod, Q, 0.7)
        np.testing.assert_allclose(out[:, hs], o, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, hs], l, rtol=0, atol=1e-14)


def test_gta_is_gqa_with_keys_and_values_tied(oracle_mod):
    """GTA/GLA page, "Grouped Tied Attention": the cached vector of a group is
    both key and value.  GTA on a one-plane pool = GQA on the pool whose K and
    V planes are both that plane; with one group (MFA page, key reuse) it is
    MQA on such a pool."""
    P = _tiny_f64("gta", H=6, NU=3, seed=63)
    out, lse = _run(oracle_mod, P, 0.45)
    both = np.stack([P["kv"], P["kv"]], axis=1)          # [pages][2][ps][NU][d]
    out_g, lse_g = _run(oracle_mod, dict(P, variant="gqa", kv=both), 0.45)
    np.testing.assert_array_equal(out, out_g)
    np.testing.assert_array_equal(lse, lse_g)
    M = _tiny_f64("gta", H=5, NU=1, seed=64)
    out_m, _ = _run(oracle_mod, M, 0.45)
    out_q, _ = _run(oracle_mod, dict(M, variant="mqa", kv=np.stack([M["kv"], M["kv"]], axis=1)), 0.45)
    np.testing.assert_array_equal(out_m, out_q)


def test_gta_brute_force_tiny(oracle_mod):
    """Brute force through numpy: softmax(scale q K^T) K with the group's tied
    vectors gathered by fancy indexing."""
    P = _tiny_f64("gta", H=4, NU=2, seed=65)
    out, lse = _run(oracle_mod, P, 0.41)
    for b in range(P["B"]):
        pages, slots = _gather_rows(P, b)
        for h in range(P["H"]):
            KV = P["kv"][pages, slots, h // (P["H"] // P["NU"])]
            o, l = _softmax_attend(P["qn"][b, h], KV, KV, 0.41)
            np.testing.assert_allclose(out[b, h], o, rtol=1e-12, atol=1e-13)
            assert abs(lse[b, h] - l) < 1e-12


def test_gqa_is_mha_with_repeated_kv(oracle_mod):
    """GQA = MHA whose KV heads are repeated over each query group (MLRA page,
    GQA bullet); MQA is the one-KV-head case (MQA bullet)."""
    P = _tiny_f64("gqa", H=6, NU=3, seed=61)
    out, lse = _run(oracle_mod, P, 0.5)
    rep = np.repeat(P["kv"], 2, axis=3)                 # [pages][2][ps][6][d]
    Q = dict(P, NU=6, kv=rep)
    out_mha, lse_mha = _run(oracle_mod, Q, 0.5)
    np.testing.assert_allclose(out, out_mha, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, lse_mha, rtol=0, atol=1e-15)
    M = _tiny_f64("mqa", H=6, seed=62)
    out_m, _ = _run(oracle_mod, M, 0.5)
    out_g, _ = _run(oracle_mod, dict(M, variant="gqa"), 0.5)
    np.testing.assert_array_equal(out_m, out_g)


# ---------------------------------------------------------------- split merge

def test_split_merge_identity(oracle_mod):
    """The result on a whole context equals the LSE-merge of the results on a
    split of it into consecutive page ranges (flash-decoding combine)."""
    P = _tiny_f64("mlra", H=2, NU=2, lens=(9, 7), ps=2, seed=71)
    out, lse = _run(oracle_mod, P, 0.55)
    # first part: pages [0, 2); second part: the rest
    lens = P["lens"]
    l1 = np.minimum(lens, 4)
    l2 = lens - l1
    bt2 = np.concatenate([P["bt"][:, 2:], P["bt"][:, :2]], axis=1)
    r1 = oracle_mod.decode_f64("mlra", 2, P["qn"], P["qr"], P["kv"], l1, 0.55, block_table=P["bt"],
                               page_size=2)
    r2 = oracle_mod.decode_f64("mlra", 2, P["qn"], P["qr"], P["kv"], l2, 0.55, block_table=bt2,
                               page_size=2)
    # per-branch outputs are needed for the merge: rebuild them branch by branch
    for b in range(2):
        for h in range(2):
            merged = np.zeros(6)
            for r in range(2):
                parts_o, parts_l = [], []
                for lens_x, bt_x in ((l1, P["bt"]), (l2, bt2)):
                    sl = np.concatenate([P["kv"][..., r * 6:(r + 1) * 6], P["kv"][..., 12:]], axis=-1)
                    o, l = oracle_mod.decode_f64("mla", 1, P["qn"][:, :, r], P["qr"][:, :, r], sl,
                                                 lens_x, 0.55, block_table=bt_x, page_size=2)
                    parts_o.append(o[b, h][None])
                    parts_l.append([l[b, h]])
                o_m, l_m = oracle_mod.merge(np.stack(parts_o), np.array(parts_l))
                merged += o_m[0]
                assert abs(l_m[0] - lse[b, h, r]) < 1e-12
                assert abs(np.logaddexp(r1[1][b, h, r], r2[1][b, h, r]) - lse[b, h, r]) < 1e-12
            np.testing.assert_allclose(merged, out[b, h], rtol=0, atol=1e-12)


def test_merge_closed_forms(oracle_mod):
    """merge of one part is that part; an empty part (-inf) has no weight; two
    parts give lse = logaddexp(a, b) and o = (e^a o1 + e^b o2) / (e^a + e^b)."""
    rng = _rng(81)
    o1, o2 = rng.standard_normal((2, 3, 5))
    a, b = np.array([0.3, -2.0, 5.0]), np.array([1.1, -2.0, -7.0])
    o, l = oracle_mod.merge(o1[None], a[None])
    np.testing.assert_array_equal(o, o1)
    np.testing.assert_array_equal(l, a)
    o, l = oracle_mod.merge(np.stack([o1, o2]), np.stack([a, np.full(3, -np.inf)]))
    np.testing.assert_allclose(o, o1, rtol=1e-15)
    np.testing.assert_allclose(l, a, rtol=1e-15)
    o, l = oracle_mod.merge(np.stack([o1, o2]), np.stack([a, b]))
    np.testing.assert_allclose(l, np.logaddexp(a, b), rtol=1e-15)
    wa = np.exp(a) / (np.exp(a) + np.exp(b))
    np.testing.assert_allclose(o, wa[:, None] * o1 + (1 - wa)[:, None] * o2, rtol=1e-13)
    o, l = oracle_mod.merge(np.zeros((2, 1, 2)), np.full((2, 1), -np.inf))
    assert np.all(o == 0) and np.isneginf(l[0])


# ---------------------------------------------------------------- masking

def test_poison_outside_context_is_never_read(oracle_mod):
    """Slots past seq_len and spare pages may hold NaN / +-1e4: changing them
    changes nothing (cache rows past the context are not part of it)."""
    shape = W.Shape("gla", 3, 4, 2, 16, 8, (65, 130))
    x = W.make_inputs(shape, seed=7, seq_lens=[65, 130, 100])
    out, lse = oracle_mod.decode(x)
    assert np.isfinite(out).all()
    kv = x["kv"].copy()
    page, slot = W.token_location(x, 0, 64)          # last page of a 65-token sequence
    assert np.any(kv[page, slot + 1:] == W.BF16_NAN) or np.any(np.abs(
        W.bf16_bits_to_f32(kv[page, slot + 1:])) == 9984.0)
    kv[page, slot + 1:] = 0x4000                     # 2.0 instead of poison
    y = dict(x, kv=kv)
    out2, lse2 = oracle_mod.decode(y)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_sample_of_sequences_matches_full(oracle_mod):
    """Computing a subset of sequences (used by the sampled full-size parity
    checks) gives the same numbers as computing all of them."""
    x = W.make_inputs(W.Shape("mqa", 4, 8, 1, 32, 0, (10, 200)), seed=3)
    out, lse = oracle_mod.decode(x)
    o2, l2 = oracle_mod.decode(x, b_list=[3, 1])
    np.testing.assert_array_equal(o2, out[[3, 1]])
    np.testing.assert_array_equal(l2, lse[[3, 1]])
    o3, l3 = oracle_mod.decode(x, b_list=[2], h_list=[5, 0])
    np.testing.assert_array_equal(o3[0], out[2, [5, 0]])
    np.testing.assert_array_equal(l3[0], lse[2, [5, 0]])
    y = W.make_inputs(W.Shape("mlra", 2, 4, 3, 16, 8, (10, 90)), seed=3)
    out, lse = oracle_mod.decode(y)
    o4, l4 = oracle_mod.decode(y, b_list=[1], h_list=[3])
    np.testing.assert_array_equal(o4[0, 0], out[1, 3])
    np.testing.assert_array_equal(l4[0, 0], lse[1, 3])


# ----------------------------------------------------- several query tokens

def _q_shape(name, q_len):
    base = {"mla": W.WORKLOADS["mla"].replace(num_q_heads=4, d_nope=64, d_rope=16),
            "mlra": W.WORKLOADS["mlra_128k"].replace(num_q_heads=4, num_kv=2, d_nope=32, d_rope=16),
            "gqa": W.WORKLOADS["gqa"].replace(num_q_heads=4, num_kv=2, d_nope=32)}[name]
    return base.replace(batch=2, ctx=(20, 150), q_len=q_len)


@pytest.mark.parametrize("name", ["mla", "mlra", "gqa"])
def test_queries_last_position_sees_the_whole_context(oracle_mod, name):
    """The newest query token attends every cached token: it equals the
    single-token decode of that token's query."""
    x = W.make_inputs(_q_shape(name, 3), seed=21)
    out, lse = oracle_mod.decode(x)
    single = dict(x, shape=x["shape"].replace(q_len=1), q_nope=x["q_nope"][:, -1],
                  q_rope=None if x["q_rope"] is None else x["q_rope"][:, -1])
    ref_out, ref_lse = oracle_mod.decode(single)
    np.testing.assert_allclose(out[:, -1], ref_out, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, -1], ref_lse, rtol=0, atol=1e-13)


@pytest.mark.parametrize("name", ["mla", "gqa"])
def test_queries_are_causal(oracle_mod, name):
    """Changing the newest cached token changes only the newest query's
    result; changing the token before it leaves position 0 of 3 alone and
    changes positions 1 and 2."""
    x = W.make_inputs(_q_shape(name, 3), seed=22)
    out0, _ = oracle_mod.decode(x)
    for back, unchanged in ((1, [0, 1]), (2, [0])):
        kv = x["kv"].copy()
        for b in range(x["shape"].batch):
            page, slot = W.token_location(x, b, int(x["seq_lens"][b]) - back)
            if x["shape"].latent:
                kv[page, slot] = W.f32_to_bf16_bits(np.full(kv[page, slot].shape, 3.0, np.float32))
            else:
                kv[page, :, slot] = W.f32_to_bf16_bits(np.full(kv[page, :, slot].shape, 3.0, np.float32))
        out1, _ = oracle_mod.decode(dict(x, kv=kv))
        np.testing.assert_array_equal(out1[:, unchanged], out0[:, unchanged])
        changed = [i for i in range(3) if i not in unchanged]
        assert np.abs(out1[:, changed] - out0[:, changed]).max() > 1e-3


def test_queries_match_a_masked_brute_force(oracle_mod):
    """Tiny MLA with 3 query tokens against numpy softmax(QK^T + causal mask) V
    over the gathered cache, all positions at once."""
    s = W.WORKLOADS["mla"].replace(batch=1, num_q_heads=2, d_nope=8, d_rope=8, ctx=(7, 7), q_len=3,
                                   page_size=64)
    x = W.make_inputs(s, seed=23)
    out, lse = oracle_mod.decode(x)
    L = int(x["seq_lens"][0])
    rows = np.stack([W.bf16_bits_to_f32(x["kv"][W.token_location(x, 0, j)]) for j in range(L)]).astype(np.float64)
    qn = W.bf16_bits_to_f32(x["q_nope"][0]).astype(np.float64)     # [3][H][8]
    qr = W.bf16_bits_to_f32(x["q_rope"][0]).astype(np.float64)
    q = np.concatenate([qn, qr], axis=-1)                          # [3][H][16]
    scores = np.einsum("ihd,jd->ihj", q, rows) * x["sm_scale"]
    mask = np.arange(L)[None, :] <= (L - 3 + np.arange(3))[:, None]    # [3][L]
    scores = np.where(mask[:, None, :], scores, -np.inf)
    m = scores.max(-1, keepdims=True)
    p = np.exp(scores - m)
    z = p.sum(-1, keepdims=True)
    ref = np.einsum("ihj,jd->ihd", p / z, rows[:, :8])
    np.testing.assert_allclose(out[0], ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[0], (m + np.log(z))[..., 0], rtol=1e-12, atol=1e-12)
