"""GPU parity: the CUDA path (called through the C ABI) against the fp64 oracle.

Tolerances (every case): max |err| <= 2e-2 and relative L2 <= 5e-3 on out,
|lse error| <= 1e-3.  fp32 output computed by the generic CUDA-core kernel
(the tiny MLA case) is also held to max |err| <= 1e-4: every product and sum
there is fp32 over at most 512 tokens of 80-wide dots, so the error is a few
fp32 ulps of O(1) values times the accumulation depth.  The tensor-core paths
round the softmax weights to bf16 before P.V (relative error up to 2^-9 per
weight), so fp32 output from them gets only the common tolerances.
"""

import numpy as np
import pytest

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


def check(out, lse, ref_out, ref_lse, fp32=False, what=""):
    assert out.shape == ref_out.shape, (out.shape, ref_out.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref_out)
    rel = np.linalg.norm(out - ref_out) / max(np.linalg.norm(ref_out), 1e-30)
    assert err.max() <= TOL_MAX, f"{what}: max err {err.max():.3e}"
    assert rel <= TOL_REL, f"{what}: rel L2 {rel:.3e}"
    if fp32:
        assert err.max() <= 1e-4, f"{what}: fp32 max err {err.max():.3e}"
    both_inf = np.isneginf(lse) & np.isneginf(ref_lse)
    assert (np.isneginf(lse) == np.isneginf(ref_lse)).all(), f"{what}: -inf lse mismatch"
    with np.errstate(invalid="ignore"):          # -inf - -inf where both rows are empty
        dl = np.abs(np.where(both_inf, 0.0, lse - ref_lse))
    assert dl.max() <= TOL_LSE, f"{what}: lse err {dl.max():.3e}"


def kernel_of(name_or_shape):
    """Name of the decode kernel the library plans for a workload shape."""
    from shared_kv_caches_b200 import kvattn as K
    s = name_or_shape
    lo, hi = s.ctx
    p = K.params_for(s, (hi + 63) // 64, 1024, hi)
    return K.KERNEL_NAMES[K.kvattn_get_plan(s.variant_id, p).kernel]


def run_gpu(inputs, dev, num_splits=0, max_seq_len=None):
    import torch
    from shared_kv_caches_b200.device import DeviceProblem
    p = DeviceProblem(inputs, dev, num_splits=num_splits, max_seq_len=max_seq_len)
    p.run()
    torch.cuda.synchronize()
    out, lse = p.results()
    return p, out, lse


SMALL = {
    "tiny_mla": (W.WORKLOADS["tiny_mla"], None),
    "gqa": (W.WORKLOADS["gqa"].replace(batch=3, ctx=(1, 700)), None),
    "mfa": (W.WORKLOADS["mfa"].replace(batch=3, ctx=(1, 700)), None),
    "mla": (W.WORKLOADS["mla"].replace(batch=2, ctx=(100, 700)), None),
    "mla_scaled_inputs": (W.WORKLOADS["mla"].replace(batch=2, ctx=(100, 700), input_scale=1 / 24), None),
    "gla": (W.WORKLOADS["gla"].replace(batch=2, ctx=(100, 700)), None),
    "mlra": (W.WORKLOADS["mlra_128k"].replace(batch=2, ctx=(100, 700)), None),
    "gqa_contiguous": (W.WORKLOADS["gqa"].replace(batch=2, ctx=(1, 300), paged=False), None),
    "mlra_fp32_out": (W.WORKLOADS["mlra_128k"].replace(batch=1, ctx=(333, 333), out_dtype="fp32"), None),
    # more groups / branches on the same tensor-core kernel, and the single
    # group or branch a tensor-parallel rank holds
    "gla1_shard": (W.WORKLOADS["gla"].replace(batch=2, num_q_heads=64, num_kv=1, ctx=(100, 700)), None),
    "gla4": (W.WORKLOADS["gla"].replace(batch=2, num_kv=4, d_nope=128, ctx=(100, 700)), None),
    "gla8": (W.WORKLOADS["gla"].replace(batch=2, num_kv=8, d_nope=64, ctx=(100, 700)), None),
    "mlra1_shard": (W.WORKLOADS["mlra_128k"].replace(batch=2, num_kv=1, ctx=(100, 700)), None),
    "mlra2": (W.WORKLOADS["mlra_128k"].replace(batch=2, num_kv=2, d_nope=256, ctx=(100, 700)), None),
    "mlra8": (W.WORKLOADS["mlra_128k"].replace(batch=2, num_kv=8, d_nope=64, ctx=(100, 700)), None),
    # tied keys and values: GTA on the GQA kernel, MFA-KR on the MQA kernel,
    # and a tied shape only the generic kernel covers
    "gta": (W.WORKLOADS["gta"].replace(batch=3, ctx=(1, 700)), None),
    "mfa_kr": (W.WORKLOADS["mfa_kr"].replace(batch=3, ctx=(1, 700)), None),
    "gta_generic": (W.WORKLOADS["gta"].replace(batch=2, num_q_heads=8, num_kv=2, d_nope=64, ctx=(1, 300)), None),
    # fp8 (e4m3) cache with per-tensor scales, and with unit scales
    "gqa_fp8": (W.WORKLOADS["gqa_fp8"].replace(batch=3, ctx=(1, 700)), None),
    "gqa_fp8_unit_scales": (W.WORKLOADS["gqa_fp8"].replace(batch=3, ctx=(1, 700), k_scale=1.0, v_scale=1.0), None),
    "gqa_fp8_contiguous": (W.WORKLOADS["gqa_fp8"].replace(batch=2, ctx=(1, 300), paged=False), None),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_parity_small(dev, oracle_mod, name):
    shape, lens = SMALL[name]
    x = W.make_inputs(shape, seed=0, seq_lens=lens)
    ref_out, ref_lse = oracle_mod.decode(x)
    p, out, lse = run_gpu(x, dev)
    tight = shape.out_dtype == "fp32" and p.plan_kernel_name() == "generic"
    check(out, lse, ref_out, ref_lse, fp32=tight, what=name)


SWEEP_LENS = [1, 2, 63, 64, 65, 127, 128, 4097]
SWEEP_SHAPES = {
    "gqa": W.WORKLOADS["gqa"],
    "mfa": W.WORKLOADS["mfa"],
    "mla": W.WORKLOADS["mla"],
    "gla": W.WORKLOADS["gla"],
    "mlra": W.WORKLOADS["mlra_128k"],
    "gta": W.WORKLOADS["gta"],
    "mfa_kr": W.WORKLOADS["mfa_kr"],
    "gqa_fp8": W.WORKLOADS["gqa_fp8"],
}


@pytest.mark.parametrize("splits", [0, 1, 2, 7, 1000])
@pytest.mark.parametrize("name", sorted(SWEEP_SHAPES))
def test_parity_ctx_sweep(dev, oracle_mod, name, splits):
    """Edge lengths (one token, page boundaries +-1, a long ragged tail) in one
    batch, with forced split counts up to more parts than pages."""
    shape = SWEEP_SHAPES[name].replace(batch=len(SWEEP_LENS), ctx=(1, 4097))
    x = W.make_inputs(shape, seed=1, seq_lens=SWEEP_LENS)
    ref_out, ref_lse = oracle_mod.decode(x)
    _, out, lse = run_gpu(x, dev, num_splits=splits)
    check(out, lse, ref_out, ref_lse, what=f"{name} splits={splits}")


@pytest.mark.parametrize("batch", [1, 3])
def test_parity_batch_sizes(dev, oracle_mod, batch):
    shape = W.WORKLOADS["gla"].replace(batch=batch, ctx=(1, 1500))
    x = W.make_inputs(shape, seed=2)
    ref_out, ref_lse = oracle_mod.decode(x)
    _, out, lse = run_gpu(x, dev)
    check(out, lse, ref_out, ref_lse, what=f"gla batch {batch}")


def _sample(x, shape):
    lens = np.asarray(x["seq_lens"])
    if shape.batch == 1:
        return [0], [0, 31, 64, 101, 127]
    picks = sorted({int(np.argmax(lens)), int(np.argmin(lens)), shape.batch - 1})
    return picks, None


@pytest.mark.parametrize("name", ["gqa", "mfa", "mla", "gla", "mlra_128k", "mlra_512k", "mlra_1m",
                                  "mlra_b8_128k", "gta", "mfa_kr", "gqa_fp8"])
def test_parity_full_size_sampled(dev, oracle_mod, name):
    """Full benchmark sizes, library-chosen launch (as timed by bench.py);
    the oracle computes sampled sequences (and heads for batch 1)."""
    shape = W.WORKLOADS[name]
    x = W.make_inputs(shape, seed=0)
    _, out, lse = run_gpu(x, dev)
    b_list, h_list = _sample(x, shape)
    ref_out, ref_lse = oracle_mod.decode(x, b_list=b_list, h_list=h_list)
    g_out = out[b_list] if h_list is None else out[b_list][:, h_list]
    g_lse = lse[b_list] if h_list is None else lse[b_list][:, h_list]
    check(g_out, g_lse, ref_out, ref_lse, what=name)


def test_benchmark_shapes_use_the_specialised_kernels(dev):
    """The benchmark shapes run on their specialised kernels, not the generic one."""
    assert kernel_of(W.WORKLOADS["gqa"]) == "gqa"
    assert kernel_of(W.WORKLOADS["mfa"]) == "mqa_tc"
    assert kernel_of(W.WORKLOADS["mla"]) == "latent_pair"
    for n in ("gla", "mlra_128k", "mlra_1m", "mlra_b8_128k"):
        assert kernel_of(W.WORKLOADS[n]) == "latent_tc", n
    assert kernel_of(W.WORKLOADS["tiny_mla"]) == "generic"
    assert kernel_of(W.WORKLOADS["gta"]) == "gqa"
    assert kernel_of(W.WORKLOADS["mfa_kr"]) == "mqa_tc"
    assert kernel_of(W.WORKLOADS["gqa_fp8"]) == "gqa_fp8"
    assert kernel_of(SMALL["gta_generic"][0]) == "generic"
    for name in ("gla1_shard", "gla4", "gla8", "mlra1_shard", "mlra2", "mlra8"):
        assert kernel_of(SMALL[name][0]) == "latent_tc", name


def test_tiny_config_exact_shape(dev, oracle_mod):
    """The tiny contiguous MLA problem, whole, fp32 output."""
    x = W.make_inputs(W.WORKLOADS["tiny_mla"], seed=0)
    ref_out, ref_lse = oracle_mod.decode(x)
    p, out, lse = run_gpu(x, dev)
    assert p.out.dtype.is_floating_point and p.out.element_size() == 4
    assert p.plan_kernel_name() == "generic"
    check(out, lse, ref_out, ref_lse, fp32=True, what="tiny")


# ------------------------------------------------------------ properties

def _repermute(x, seed):
    """Same logical cache under another physical page permutation."""
    rng = np.random.default_rng(seed)
    n = x["num_pages"]
    newpos = rng.permutation(n).astype(np.int32)     # old page p -> new page newpos[p]
    kv2 = np.empty_like(x["kv"])
    kv2[newpos] = x["kv"]
    return dict(x, kv=kv2, block_table=newpos[x["block_table"]])


@pytest.mark.parametrize("name", ["gqa", "mla", "mlra", "gqa_fp8"])
def test_block_table_permutation_is_bit_identical(dev, name):
    shape = SWEEP_SHAPES[name].replace(batch=3, ctx=(500, 3000))
    x = W.make_inputs(shape, seed=3)
    _, out1, lse1 = run_gpu(x, dev)
    _, out2, lse2 = run_gpu(_repermute(x, 99), dev)
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(lse1, lse2)


@pytest.mark.parametrize("name", ["gqa", "gla"])
def test_poison_outside_context_changes_nothing(dev, name):
    shape = SWEEP_SHAPES[name].replace(batch=3, ctx=(65, 1000))
    x = W.make_inputs(shape, seed=4)
    _, out1, lse1 = run_gpu(x, dev)
    kv = x["kv"].copy()
    pois = np.isin(kv, W.POISON_BITS)
    kv[pois] = np.where(kv[pois] == W.BF16_NAN, W.BF16_POS_1E4, W.BF16_NAN).astype(np.uint16)
    _, out2, lse2 = run_gpu(dict(x, kv=kv), dev)
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(lse1, lse2)


def test_poison_outside_context_changes_nothing_fp8(dev):
    """fp8 cache: NaN and +-448 codes past each context swapped for one another."""
    shape = SWEEP_SHAPES["gqa_fp8"].replace(batch=3, ctx=(65, 1000))
    x = W.make_inputs(shape, seed=4)
    _, out1, lse1 = run_gpu(x, dev)
    kv = x["kv"].copy()
    pois = np.isin(kv, W.POISON_FP8)
    kv[pois] = np.where(kv[pois] == 0x7F, 0x7E, 0x7F).astype(np.uint8)
    _, out2, lse2 = run_gpu(dict(x, kv=kv), dev)
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(lse1, lse2)


def test_context_of_one_returns_scaled_value_fp8(dev, oracle_mod):
    """ctx = 1 over an fp8 cache: the output is v_scale times the decoded value
    row, exactly (an e4m3 value times a power of two fits bf16)."""
    import torch
    shape = SWEEP_SHAPES["gqa_fp8"].replace(batch=2, ctx=(1, 1))
    x = W.make_inputs(shape, seed=7)
    p, _, _ = run_gpu(x, dev)
    got = p.out.view(dtype=torch.int16).cpu().numpy().view(np.uint16)
    g_of = np.arange(shape.num_q_heads) // (shape.num_q_heads // shape.num_kv)
    for b in range(2):
        page, slot = W.token_location(x, b, 0)
        # + 0.0: a -0 code comes out as +0 (the accumulators start at +0)
        want = shape.v_scale * oracle_mod.e4m3_value(x["kv"][page, 1, slot, g_of]) + 0.0
        bits = (want.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal(want.astype(np.float32).view(np.uint32) & 0xFFFF, np.zeros_like(bits))
        np.testing.assert_array_equal(got[b], bits)


def test_split_count_changes_only_rounding(dev):
    shape = SWEEP_SHAPES["mlra"].replace(batch=2, ctx=(3000, 5000))
    x = W.make_inputs(shape, seed=5)
    _, out1, lse1 = run_gpu(x, dev, num_splits=1)
    _, out2, lse2 = run_gpu(x, dev, num_splits=40)
    check(out2, lse2, out1, lse1, what="splits 1 vs 40")


def test_empty_sequences(dev, oracle_mod):
    shape = SWEEP_SHAPES["mla"].replace(batch=3, ctx=(0, 200))
    x = W.make_inputs(shape, seed=6, seq_lens=[0, 130, 0])
    _, out, lse = run_gpu(x, dev)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    ref_out, ref_lse = oracle_mod.decode(x, b_list=[1])
    check(out[[1]], lse[[1]], ref_out, ref_lse, what="non-empty neighbour")


def test_all_sequences_empty(dev):
    shape = SWEEP_SHAPES["gqa"].replace(batch=2, ctx=(0, 0))
    x = W.make_inputs(shape, seed=6, seq_lens=[0, 0], max_pages_per_seq=2)
    _, out, lse = run_gpu(x, dev)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("name", ["gqa", "mla", "gla", "mlra"])
def test_context_of_one_returns_value_bits(dev, name):
    """ctx = 1: the output is the value row itself, bit for bit after bf16 rounding."""
    shape = SWEEP_SHAPES[name].replace(batch=2, ctx=(1, 1))
    x = W.make_inputs(shape, seed=7)
    p, _, _ = run_gpu(x, dev)
    got = p.out.view(dtype=__import__("torch").int16).cpu().numpy().view(np.uint16)
    for b in range(2):
        page, slot = W.token_location(x, b, 0)
        for h in range(shape.num_q_heads):
            if shape.variant == "mlra":
                continue
            if shape.latent:
                g = 0 if shape.variant == "mla" else h // (shape.num_q_heads // shape.num_kv)
                v = x["kv"][page, slot, g * shape.d_nope:(g + 1) * shape.d_nope]
            else:
                g = h // (shape.num_q_heads // shape.num_kv)
                v = x["kv"][page, 1, slot, g]
            np.testing.assert_array_equal(got[b, h], v)


@pytest.mark.parametrize("name", ["gla", "mla"])
def test_page_id_out_of_range_sets_error_and_skips(dev, oracle_mod, name):
    """A bad page id in one sequence: the error bit is set, that tile loads
    nothing (both ring groups of the MLA kernel still arrive), and the other
    sequences are unaffected."""
    shape = SWEEP_SHAPES[name].replace(batch=3, ctx=(200, 200))
    x = W.make_inputs(shape, seed=8)
    bt = x["block_table"].copy()
    bt[1, 2] = x["num_pages"] + 3          # bad frame id for sequence 1
    y = dict(x, block_table=bt)
    p, out, lse = run_gpu(y, dev)
    code = p.device_error()
    assert code & 1, code
    ref_out, ref_lse = oracle_mod.decode(x, b_list=[0, 2])
    check(out[[0, 2]], lse[[0, 2]], ref_out, ref_lse, what="unaffected sequences")
    p.clear_device_error()
    assert p.device_error() == 0


def test_sequence_longer_than_hint_sets_error_and_clamps(dev, oracle_mod):
    shape = SWEEP_SHAPES["mla"].replace(batch=2, ctx=(100, 300))
    x = W.make_inputs(shape, seed=9, seq_lens=[300, 150])
    p, out, lse = run_gpu(x, dev, max_seq_len=200)
    assert p.device_error() & 2
    y = dict(x, seq_lens=np.array([200, 150], np.int32))
    ref_out, ref_lse = oracle_mod.decode(y)
    check(out, lse, ref_out, ref_lse, what="clamped")


def test_timed_entry_point_records_ordered_events(dev):
    """kvattn_decode_timed gives the same result as kvattn_decode and records
    its three events in order on the launching stream."""
    import torch
    shape = SWEEP_SHAPES["mfa"].replace(batch=2, ctx=(300, 900))
    x = W.make_inputs(shape, seed=10)
    p, out_ref, lse_ref = run_gpu(x, dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in ev:
        e.record()
    p.out.zero_()
    p.run(events=ev)
    torch.cuda.synchronize()
    out, lse = p.results()
    np.testing.assert_array_equal(out, out_ref)
    np.testing.assert_array_equal(lse, lse_ref)
    assert ev[0].elapsed_time(ev[1]) > 0.0
    assert ev[1].elapsed_time(ev[2]) >= 0.0


def test_gqa_plan_merges_in_kernel(dev):
    """The GQA kernel merges its own parts (one launch); the others use the combine pass."""
    from shared_kv_caches_b200 import kvattn as K
    for name, launches in (("gqa", 1), ("mfa", 2), ("mla", 2), ("mlra_128k", 2)):
        s = W.WORKLOADS[name]
        lo, hi = s.ctx
        plan = K.kvattn_get_plan(s.variant_id, K.params_for(s, (hi + 63) // 64, 1 << 20, hi))
        assert plan.launches == launches, name
        assert plan.header_bytes >= 256


@pytest.mark.parametrize("name,world", [("mlra_128k", 4), ("mlra_128k", 2), ("gla", 2)])
def test_tensor_parallel_shards_on_one_device(dev, oracle_mod, name, world):
    """What each tensor-parallel rank computes (its MLRA branches or GLA
    groups, through the library), solved in turn on one GPU and assembled as
    the collective would (branch outputs summed in fp32, heads side by side),
    against the oracle on the whole problem."""
    from shared_kv_caches_b200 import tp as TP
    shape = W.WORKLOADS[name].replace(batch=2, ctx=(300, 900))
    x = W.make_inputs(shape, seed=12)
    out, lse = TP.tp_decode_one_device(x, world, dev)
    ref_out, ref_lse = oracle_mod.decode(x)
    check(out, lse, ref_out, ref_lse, what=f"tp {name} x{world}")


Q_SHAPES = {
    "gqa": W.WORKLOADS["gqa"].replace(batch=3, ctx=(1, 700)),
    "mfa": W.WORKLOADS["mfa"].replace(batch=3, ctx=(1, 700)),
    "mla": W.WORKLOADS["mla"].replace(batch=2, ctx=(100, 700)),
    "gla": W.WORKLOADS["gla"].replace(batch=2, ctx=(100, 700)),
    "mlra": W.WORKLOADS["mlra_128k"].replace(batch=2, ctx=(100, 700)),
    "tiny_mla": W.WORKLOADS["tiny_mla"],
    "gta": W.WORKLOADS["gta"].replace(batch=3, ctx=(1, 700)),
    "gqa_fp8": W.WORKLOADS["gqa_fp8"].replace(batch=3, ctx=(1, 700)),
}


@pytest.mark.parametrize("q_len", [2, 4])
@pytest.mark.parametrize("name", sorted(Q_SHAPES))
def test_parity_several_query_tokens(dev, oracle_mod, name, q_len):
    """Several query tokens per sequence (the newest q_len cached tokens, each
    attending the cache up to itself), on every kernel; the first sequence
    is shorter than q_len for the GQA and MFA shapes, so its first positions
    see nothing."""
    shape = Q_SHAPES[name].replace(q_len=q_len)
    lens = [1, 300, 700] if shape.batch == 3 else None
    x = W.make_inputs(shape, seed=14, seq_lens=lens)
    ref_out, ref_lse = oracle_mod.decode(x)
    p, out, lse = run_gpu(x, dev)
    assert out.shape == ref_out.shape
    check(out, lse, ref_out, ref_lse, what=f"{name} q_len={q_len}")
    assert p.device_error() == 0
