"""GPU parity of the steps either side of attention (kvattn_rope,
kvattn_append_kv, kvattn_head_proj, MLRA branch outputs) against the fp64
oracle (oracle/steps.py, oracle.decode).

Tolerances, from the arithmetic:
* RoPE and append: the kernel turns each pair in double precision and rounds
  once to bf16, as the oracle's fp64 result rounded to nearest even is; the
  two agree bit for bit except where the fp64 value sits within a double's
  rounding of a bf16 tie, so at most one bf16 ulp apart, and rarely (< 0.1%
  of the turned entries).  Copied parts (the latent, V, every other cache
  row) are bit-exact.
* head_proj: bf16 x bf16 products are exact in fp32; the tensor cores add k
  of them in fp32, so |err| <= 1e-5 * sum_k |x w| covers the accumulation;
  bf16 output adds the final rounding, 2^-8 |y| (twice the half-ulp bound).
* the absorbed chain (append, RoPE, absorption, decode, up-projection): the
  GPU rounds the absorbed query, the softmax weights, the latent output and
  the result to bf16 (each <= 2^-9 relative), so against the unrounded fp64
  chain max |err| <= 3e-2 * max|ref| and relative L2 <= 1e-2.
"""

import numpy as np
import pytest

from oracle import steps
from shared_kv_caches_b200 import workloads as W

pytestmark = pytest.mark.gpu

BASE = W.ROPE_BASE


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from shared_kv_caches_b200 import build
    build.build()
    return torch.device("cuda:0")


def bf16_round(x):
    """Round float64 values to the nearest bf16 (ties to even), exactly."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


def f64(bits):
    return W.bf16_bits_to_f32(np.asarray(bits)).astype(np.float64)


def to_dev(bits, dev):
    from shared_kv_caches_b200.device import bf16_tensor
    return bf16_tensor(bits, dev)


def ulps(a, b):
    """Distance in bf16 ulps between two arrays of bf16 values (as float64)."""
    ia = W.f32_to_bf16_bits(np.asarray(a, np.float32)).astype(np.int32)
    ib = W.f32_to_bf16_bits(np.asarray(b, np.float32)).astype(np.int32)
    # sign-magnitude to a monotone integer line
    ia = np.where(ia & 0x8000, -(ia & 0x7FFF), ia)
    ib = np.where(ib & 0x8000, -(ib & 0x7FFF), ib)
    return np.abs(ia - ib)


def assert_turned(got, ref, what):
    d = ulps(got, ref)
    assert d.max() <= 1, f"{what}: {d.max()} ulps apart"
    assert (d > 0).mean() < 1e-3, f"{what}: {(d > 0).mean():.2e} of the entries differ"


SHAPES = {
    "mla": W.WORKLOADS["mla"].replace(batch=3, ctx=(70, 400)),
    "gla": W.WORKLOADS["gla"].replace(batch=3, ctx=(70, 400)),
    "mlra": W.WORKLOADS["mlra_128k"].replace(batch=3, ctx=(70, 400)),
}


# ------------------------------------------------------------------ RoPE
@pytest.mark.parametrize("name,q_len", [("mla", 1), ("mla", 3), ("mlra", 2), ("gla", 1)])
def test_rope_of_the_query_matches_oracle(dev, name, q_len):
    import torch
    from shared_kv_caches_b200 import kvattn as K
    s = SHAPES[name].replace(q_len=q_len)
    x = W.make_step_inputs(s, seed=3)
    rng = np.random.default_rng(4)
    pos = rng.integers(0, 1 << 20, size=(s.batch, q_len)).astype(np.int32)
    q = to_dev(x["q_rope"], dev).contiguous()
    per_pos = s.num_q_heads * (s.num_kv if s.variant == "mlra" else 1)
    K.rope_tensor(q, torch.from_numpy(pos).to(dev), 0, s.d_rope, BASE, per_pos)
    torch.cuda.synchronize()
    got = q.float().cpu().numpy().astype(np.float64)
    raw = f64(x["q_rope"]).reshape(s.batch, q_len, per_pos, s.d_rope)
    ref = bf16_round(steps.rope(raw, pos[:, :, None], BASE)).reshape(got.shape)
    assert_turned(got, ref, f"rope {name}")


def test_rope_of_a_slice_leaves_the_rest(dev):
    """rot_offset > 0: only the slice turns (a GQA-style row with a partial rotary part)."""
    import torch
    from shared_kv_caches_b200 import kvattn as K
    rng = np.random.default_rng(5)
    bits = W.f32_to_bf16_bits(rng.standard_normal((40, 8, 192)).astype(np.float32))
    pos = rng.integers(0, 5000, size=40).astype(np.int32)
    t = to_dev(bits, dev).contiguous()
    K.rope_tensor(t, torch.from_numpy(pos).to(dev), 64, 128, 500.0, 8)
    torch.cuda.synchronize()
    got = t.float().cpu().numpy().astype(np.float64)
    src = f64(bits)
    np.testing.assert_array_equal(got[..., :64], src[..., :64])
    assert_turned(got[..., 64:], bf16_round(steps.rope(src[..., 64:], pos[:, None], 500.0)), "slice")


# ---------------------------------------------------------------- append
@pytest.mark.parametrize("name,q_len", [("mla", 1), ("mla", 2), ("gla", 1), ("mlra", 3)])
def test_append_latent_matches_oracle(dev, name, q_len):
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    s = SHAPES[name].replace(q_len=q_len)
    x = W.make_step_inputs(s, seed=6)
    p = DeviceProblem(x, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    p.append_kv(to_dev(x["new_kv"], dev), torch.from_numpy(x["pos"]).to(dev), BASE, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = p.kv.float().cpu().numpy().astype(np.float64)
    ref = bf16_round(steps.append_latent(f64(x["kv"]), f64(x["new_kv"]), x["pos"], x["block_table"],
                                         s.d_rope, BASE))
    lat = s.row_elems - s.d_rope
    # everything but the turned slices is bit-exact (NaN poison included)
    np.testing.assert_array_equal(got[..., :lat], ref[..., :lat])
    touched = np.zeros(got.shape[:2], bool)
    for b in range(s.batch):
        for i in range(q_len):
            pg, sl = steps.slot_of(x["block_table"], b, int(x["pos"][b, i]), None)
            touched[pg, sl] = True
    np.testing.assert_array_equal(got[~touched][:, lat:], ref[~touched][:, lat:])
    assert_turned(got[touched][:, lat:], ref[touched][:, lat:], f"append {name}")


def test_append_heads_matches_oracle(dev):
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    s = W.WORKLOADS["gqa"].replace(batch=3, ctx=(70, 400), q_len=2)
    x = W.make_inputs(s, seed=7)
    rng = np.random.default_rng(8)
    new = W.f32_to_bf16_bits(rng.standard_normal((s.batch, 2, 2, s.num_kv, s.d_nope)).astype(np.float32))
    pos = (x["seq_lens"][:, None] - 2 + np.arange(2)).astype(np.int32)
    p = DeviceProblem(x, dev)
    p.append_kv(to_dev(new, dev), torch.from_numpy(pos).to(dev), BASE)
    torch.cuda.synchronize()
    got = p.kv.float().cpu().numpy().astype(np.float64)
    ref = bf16_round(steps.append_heads(f64(x["kv"]), f64(new), pos, x["block_table"], BASE))
    np.testing.assert_array_equal(got[:, 1], ref[:, 1])                    # V plane, copied
    touched = np.zeros((got.shape[0], 64), bool)
    for b in range(s.batch):
        for i in range(2):
            pg, sl = steps.slot_of(x["block_table"], b, int(pos[b, i]), None)
            touched[pg, sl] = True
    np.testing.assert_array_equal(got[:, 0][~touched], ref[:, 0][~touched])
    assert_turned(got[:, 0][touched], ref[:, 0][touched], "append K")


def test_append_tied_rows_copies_bits_and_refuses_rope(dev):
    """GTA / MFA-KR: the tied vector is the value too, so it is stored as given."""
    import torch
    from shared_kv_caches_b200 import kvattn as K
    from shared_kv_caches_b200.device import DeviceProblem
    s = W.WORKLOADS["gta"].replace(batch=3, ctx=(70, 400), q_len=2)
    x = W.make_inputs(s, seed=14)
    rng = np.random.default_rng(15)
    new = W.f32_to_bf16_bits(rng.standard_normal((s.batch, 2, s.num_kv, s.d_nope)).astype(np.float32))
    pos = (x["seq_lens"][:, None] - 2 + np.arange(2)).astype(np.int32)
    p = DeviceProblem(x, dev)
    before = p.kv.clone()
    new_d, pos_d = to_dev(new, dev), torch.from_numpy(pos).to(dev)
    st = K.kvattn_append_kv(p.variant, p.params, new_d.data_ptr(), pos_d.data_ptr(), p.block_table.data_ptr(),
                            p.kv.data_ptr(), BASE, None, torch.cuda.current_stream(dev).cuda_stream)
    assert st == K.KVATTN_ERR_INVALID_ARG
    p.append_kv(new_d, pos_d, 0.0)
    torch.cuda.synchronize()
    got = p.kv.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = before.cpu().view(torch.int16).numpy().view(np.uint16).copy()
    for b in range(s.batch):
        for i in range(2):
            pg, sl = steps.slot_of(x["block_table"], b, int(pos[b, i]), None)
            ref[pg, sl] = new[b, i]
    np.testing.assert_array_equal(got, ref)


def test_append_without_rope_copies_bits(dev):
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    s = SHAPES["mla"]
    x = W.make_step_inputs(s, seed=9)
    p = DeviceProblem(x, dev)
    p.append_kv(to_dev(x["new_kv"], dev), torch.from_numpy(x["pos"]).to(dev), 0.0)
    torch.cuda.synchronize()
    got = p.kv.cpu().view(torch.int16).numpy().view(np.uint16)
    for b in range(s.batch):
        pg, sl = steps.slot_of(x["block_table"], b, int(x["pos"][b, 0]), None)
        np.testing.assert_array_equal(got[pg, sl], x["new_kv"][b, 0])


def test_append_out_of_range_sets_errors_and_skips(dev):
    import torch
    from shared_kv_caches_b200 import kvattn as K
    from shared_kv_caches_b200.device import DeviceProblem
    s = SHAPES["mla"]
    x = W.make_step_inputs(s, seed=10)
    p = DeviceProblem(x, dev)
    before = p.kv.clone()
    pos = x["pos"].copy()
    pos[0, 0] = p.max_pages_per_seq * 64          # past the sequence's pages
    pos[1, 0] = -1
    bt = p.block_table.clone()
    bt[2, :] = p.num_pages + 5                     # a page outside the pool
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    st = K.kvattn_append_kv(p.variant, p.params, to_dev(x["new_kv"], dev).data_ptr(),
                            torch.from_numpy(pos).to(dev).data_ptr(), bt.data_ptr(), p.kv.data_ptr(), BASE,
                            err.data_ptr(), torch.cuda.current_stream(dev).cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert int(err.item()) == K.KVATTN_DEVERR_POS_OUT_OF_RANGE | K.KVATTN_DEVERR_PAGE_OUT_OF_RANGE
    assert torch.equal(p.kv.view(torch.int16), before.view(torch.int16))


# ------------------------------------------------------- head projection
PROJ = {
    "absorb_mla": (64, 128, 128, 512),
    "up_mla": (64, 128, 512, 128),
    "up_gla": (64, 128, 256, 128),
    "up_mlra": (64, 128, 512, 128),
    "ragged": (130, 3, 192, 320),
    "one_row": (1, 5, 64, 64),
    "wide": (200, 2, 128, 768),
}


@pytest.mark.parametrize("out_fp32", [False, True])
@pytest.mark.parametrize("case", sorted(PROJ))
def test_head_proj_matches_oracle(dev, case, out_fp32):
    import torch
    from shared_kv_caches_b200 import kvattn as K
    rows, heads, k, n = PROJ[case]
    rng = np.random.default_rng(11)
    xb = W.f32_to_bf16_bits(rng.standard_normal((rows, heads, k)).astype(np.float32))
    wb = W.f32_to_bf16_bits((rng.standard_normal((heads, k, n)) / np.sqrt(k)).astype(np.float32))
    y = K.head_proj_tensor(to_dev(xb, dev), to_dev(wb, dev), out_fp32=out_fp32)
    torch.cuda.synchronize()
    got = y.float().cpu().numpy().astype(np.float64)
    xf, wf = f64(xb), f64(wb)
    ref = steps.head_proj(xf, wf)
    bound = 1e-5 * steps.head_proj(np.abs(xf), np.abs(wf))
    if not out_fp32:
        bound = bound + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    assert (err <= bound + 1e-30).all(), f"{case}: worst {np.max(err - bound):.3e} over the bound"


def test_head_proj_refuses_bad_shapes(dev):
    from shared_kv_caches_b200 import kvattn as K
    import torch
    t = torch.zeros(64 * 64, dtype=torch.bfloat16, device=dev)
    assert K.kvattn_head_proj(t.data_ptr(), t.data_ptr(), t.data_ptr(), 0, 1, 1, 48, 64) == K.KVATTN_ERR_INVALID_ARG
    assert K.kvattn_head_proj(t.data_ptr(), t.data_ptr(), t.data_ptr(), 0, 1, 1, 64, 96) == K.KVATTN_ERR_INVALID_ARG
    assert K.kvattn_head_proj(t.data_ptr() + 2, t.data_ptr(), t.data_ptr(), 0, 1, 1, 64, 64) == \
        K.KVATTN_ERR_MISALIGNED


# ------------------------------------------------- MLRA branch outputs
@pytest.mark.parametrize("q_len", [1, 2])
def test_mlra_branch_outputs_match_oracle(dev, oracle_mod, q_len):
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    s = SHAPES["mlra"].replace(q_len=q_len, branch_out=True, out_dtype="fp32")
    x = W.make_inputs(s, seed=12)
    p = DeviceProblem(x, dev)
    p.run()
    torch.cuda.synchronize()
    out, lse = p.results()
    ref_out, ref_lse = oracle_mod.decode(x, branch_out=True)
    assert out.shape == ref_out.shape
    err = np.abs(out - ref_out)
    assert err.max() <= 2e-2 and np.linalg.norm(out - ref_out) / np.linalg.norm(ref_out) <= 5e-3
    np.testing.assert_allclose(lse, ref_lse, atol=1e-3, rtol=0)
    # their sum is the summed decode, up to fp32 rounding
    summed = DeviceProblem(dict(x, shape=s.replace(branch_out=False)), dev)
    summed.run()
    torch.cuda.synchronize()
    np.testing.assert_allclose(out.sum(axis=-2), summed.results()[0], atol=1e-5, rtol=0)


# ------------------------------------------------------- the whole chain
@pytest.mark.parametrize("name,q_len", [("mla", 1), ("mla", 2), ("gla", 1), ("mlra", 1)])
def test_absorbed_chain_end_to_end(dev, oracle_mod, name, q_len):
    """append (k^R turned) -> RoPE of the query -> absorption (W_UK) -> decode
    (MLRA: per-branch outputs) -> up-projection (W_UV, MLRA branch blocks
    stacked), on the GPU through the C ABI, against the same chain in fp64."""
    import torch
    from shared_kv_caches_b200 import kvattn as K
    from shared_kv_caches_b200.device import DeviceProblem
    s = SHAPES[name].replace(q_len=q_len, branch_out=(name == "mlra"))
    x = W.make_step_inputs(s, seed=13)
    d_h, n_abs, d_v = W.step_widths(s)
    H = s.num_q_heads
    rows = s.batch * q_len
    pos_d = torch.from_numpy(x["pos"]).to(dev)

    p = DeviceProblem(x, dev)
    p.append_kv(to_dev(x["new_kv"], dev), pos_d, BASE)
    q_nope = K.head_proj_tensor(to_dev(x["q_c"], dev).reshape(rows, H, d_h), to_dev(x["w_uk"], dev))
    q_rope = to_dev(x["q_rope"], dev).contiguous()
    per_pos = H * (s.num_kv if s.variant == "mlra" else 1)
    K.rope_tensor(q_rope, pos_d, 0, s.d_rope, BASE, per_pos)
    p.run(q_nope=q_nope.reshape(p.q_nope.shape), q_rope=q_rope)
    o = K.head_proj_tensor(p.out.reshape(rows, H, n_abs), to_dev(x["w_uv"], dev))
    torch.cuda.synchronize()
    got = o.float().cpu().numpy().astype(np.float64)

    # the same chain in fp64; the appended rows are stored as bf16, as the cache holds them
    cache = bf16_round(steps.append_latent(f64(x["kv"]), f64(x["new_kv"]), x["pos"], x["block_table"],
                                           s.d_rope, BASE))
    qn = steps.head_proj(f64(x["q_c"]).reshape(rows, H, d_h), f64(x["w_uk"]))
    qr = steps.rope(f64(x["q_rope"]).reshape(rows, per_pos, s.d_rope), x["pos"].reshape(rows)[:, None], BASE)
    units = (s.num_kv,) if s.variant == "mlra" else ()
    qn = qn.reshape((rows, H) + units + (s.d_nope,))
    qr = qr.reshape((rows, H) + units + (s.d_rope,))
    # one row per (sequence, query token), each attending its causal prefix
    lens = np.maximum(np.repeat(x["seq_lens"], q_len) - np.tile(q_len - 1 - np.arange(q_len), s.batch), 0)
    o_lat, _ = oracle_mod.decode_f64(s.variant, s.num_kv, qn, qr, cache, lens.astype(np.int32), x["sm_scale"],
                                     block_table=np.repeat(x["block_table"], q_len, axis=0), branch_out=True)
    ref = steps.head_proj(o_lat.reshape(rows, H, n_abs), f64(x["w_uv"]))
    err = np.abs(got - ref)
    assert err.max() <= 3e-2 * np.abs(ref).max(), f"max err {err.max():.3e} of {np.abs(ref).max():.3e}"
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-2
