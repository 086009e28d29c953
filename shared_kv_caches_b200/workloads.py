"""Seeded synthetic decode-attention workloads.

This module only draws random numbers, rounds them to bf16 and places them in
the paged cache layout.  It holds none of the attention arithmetic, so both
the CPU oracle (``oracle/``) and the CUDA path take their inputs from here.

Layouts (all bf16 stored as uint16 bit patterns, row-major):

* latent variants (MLA, GLA, MLRA): pool ``[num_pages][page_size][row]`` with
  ``row = num_kv * d_nope + d_rope``.  Each token row is
  ``[c_0 | c_1 | ... | c_{num_kv-1} | k_rope]``: the latent of every group or
  branch followed by the one decoupled-RoPE key they share (MLA explainer,
  section 2.2 "dual-branch" and 2.4 "what is cached"; MLRA block
  decomposition).
* GQA / MQA (MFA at decode time): pool ``[num_pages][2][page_size][num_kv][d]``
  with index 0 = K and 1 = V.
* ``block_table[b][i]`` (int32) names the physical page holding tokens
  ``[64 i, 64 i + 64)`` of sequence ``b``.  Contiguous mode (``paged=False``)
  has no block table: sequence ``b`` owns pages ``b * max_pages_per_seq + i``.

Queries: ``q_nope`` is ``[B][H][d_nope]`` (MLRA ``[B][H][R][d_nope]``) and
``q_rope`` is ``[B][H][d_rope]`` (MLRA ``[B][H][R][d_rope]``); ``None`` for
GQA/MQA.

Draw order for one seed: sequence lengths, q_nope, q_rope, cache pool,
block-table permutation, poison.  Slots past a sequence's length in its last
page, and the spare pages, hold poison (NaN and +-1e4) that a correct kernel
never lets into a result.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

VARIANT_IDS = {"gqa": 0, "mqa": 1, "mla": 2, "gla": 3, "mlra": 4, "gta": 5}
LATENT_VARIANTS = ("mla", "gla", "mlra")

BF16_NAN = 0x7FC0
BF16_POS_1E4 = 0x461C
BF16_NEG_1E4 = 0xC61C
POISON_BITS = np.array([BF16_NAN, BF16_POS_1E4, BF16_NEG_1E4], dtype=np.uint16)
# fp8 (e4m3) poison: NaN, +448 and -448 (the largest magnitudes)
POISON_FP8 = np.array([0x7F, 0x7E, 0xFE], dtype=np.uint8)

_CHUNK = 1 << 24


@dataclasses.dataclass(frozen=True)
class Shape:
    """One decode-attention problem.

    ``num_kv`` is the number of KV heads (GQA/MQA), 1 for MLA, the number of
    latent groups G for GLA and the number of branches R for MLRA.
    ``d_nope`` is the head dim (GQA/MQA) or the latent width per
    group/branch; ``d_rope`` is the width of the shared RoPE key (0 for
    GQA/MQA).  ``ctx`` is an inclusive range the sequence lengths are drawn
    from (integers, uniform).
    """

    variant: str
    batch: int
    num_q_heads: int
    num_kv: int
    d_nope: int
    d_rope: int
    ctx: tuple
    paged: bool = True
    page_size: int = 64
    out_dtype: str = "bf16"
    sm_scale: float | None = None
    input_scale: float = 1.0
    q_len: int = 1          # query tokens per sequence (the newest q_len cached tokens)
    branch_out: bool = False  # MLRA: the branch outputs side by side instead of their sum
    cache_dtype: str = "bf16"  # "fp8": the cache holds e4m3 bytes (GQA), key = k_scale * K8, value = v_scale * V8
    k_scale: float = 1.0
    v_scale: float = 1.0

    @property
    def variant_id(self) -> int:
        return VARIANT_IDS[self.variant]

    @property
    def latent(self) -> bool:
        return self.variant in LATENT_VARIANTS

    @property
    def key_dim(self) -> int:
        return self.d_nope + self.d_rope

    @property
    def value_dim(self) -> int:
        return self.d_nope

    @property
    def row_elems(self) -> int:
        """Elements of one token row of one page (per K or V plane for GQA)."""
        if self.latent:
            return self.num_kv * self.d_nope + self.d_rope
        return self.num_kv * self.d_nope

    @property
    def tied(self) -> bool:
        """GTA / MFA-KR: one cached vector per unit is both key and value."""
        return self.variant == "gta"

    @property
    def page_elems(self) -> int:
        if self.latent or self.tied:
            return self.page_size * self.row_elems
        return 2 * self.page_size * self.row_elems

    @property
    def lse_rows(self) -> int:
        """LSE entries per sequence: one per head, or per (head, branch) for MLRA."""
        if self.variant == "mlra":
            return self.num_q_heads * self.num_kv
        return self.num_q_heads

    @property
    def scale(self) -> float:
        if self.sm_scale is not None:
            return float(self.sm_scale)
        return 1.0 / math.sqrt(self.key_dim)

    def _rows(self) -> tuple:
        """Leading axes: sequence, and query token when there are several."""
        return (self.batch,) if self.q_len == 1 else (self.batch, self.q_len)

    def q_nope_shape(self) -> tuple:
        if self.variant == "mlra":
            return self._rows() + (self.num_q_heads, self.num_kv, self.d_nope)
        return self._rows() + (self.num_q_heads, self.d_nope)

    def q_rope_shape(self) -> tuple | None:
        if self.d_rope == 0:
            return None
        if self.variant == "mlra":
            return self._rows() + (self.num_q_heads, self.num_kv, self.d_rope)
        return self._rows() + (self.num_q_heads, self.d_rope)

    def out_shape(self) -> tuple:
        if self.branch_out:
            return self._rows() + (self.num_q_heads, self.num_kv, self.d_nope)
        return self._rows() + (self.num_q_heads, self.d_nope)

    def lse_shape(self) -> tuple:
        if self.variant == "mlra":
            return self._rows() + (self.num_q_heads, self.num_kv)
        return self._rows() + (self.num_q_heads,)

    def pool_shape(self, num_pages: int) -> tuple:
        if self.latent:
            return (num_pages, self.page_size, self.row_elems)
        if self.tied:
            return (num_pages, self.page_size, self.num_kv, self.d_nope)
        return (num_pages, 2, self.page_size, self.num_kv, self.d_nope)

    def replace(self, **kw) -> "Shape":
        return dataclasses.replace(self, **kw)


# The workloads of the decode-attention benchmark suite.  Names state what
# they are; sizes follow the shapes the pages discuss (DeepSeek-V3-like MLA
# 512+64, GLA-2 with two 256-wide latent heads, MLRA-4 with four 128-wide
# branches, GQA 32q/8kv and an MFA-style single wide KV head; GTA and MFA-KR
# are the same GQA and MFA shapes with keys and values tied into one cached
# vector).
WORKLOADS = {
    "tiny_mla": Shape("mla", 2, 8, 1, 64, 16, (512, 512), paged=False, out_dtype="fp32"),
    "gqa": Shape("gqa", 32, 32, 8, 128, 0, (1024, 8192)),
    "mfa": Shape("mqa", 32, 32, 1, 256, 0, (1024, 8192)),
    "mla": Shape("mla", 64, 128, 1, 512, 64, (4096, 32768)),
    "gla": Shape("gla", 64, 128, 2, 256, 64, (16384, 16384)),
    "mlra_128k": Shape("mlra", 1, 128, 4, 128, 64, (131072, 131072)),
    "mlra_512k": Shape("mlra", 1, 128, 4, 128, 64, (524288, 524288)),
    "mlra_1m": Shape("mlra", 1, 128, 4, 128, 64, (1048576, 1048576)),
    "mlra_b8_128k": Shape("mlra", 8, 128, 4, 128, 64, (131072, 131072)),
    "gta": Shape("gta", 32, 32, 8, 128, 0, (1024, 8192)),
    "mfa_kr": Shape("gta", 32, 32, 1, 256, 0, (1024, 8192)),
    "gqa_fp8": Shape("gqa", 32, 32, 8, 128, 0, (1024, 8192), cache_dtype="fp8", k_scale=0.5, v_scale=2.0),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); finite inputs.

    In 32-bit arithmetic: a finite float's bits plus at most 0x8000 stay below
    2**32, so nothing wraps."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    v = (u >> 16) & 1
    v += u
    v += 0x7FFF
    return (v >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, scale: float) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    for start in range(0, n, _CHUNK):
        stop = min(n, start + _CHUNK)
        draw = rng.standard_normal(stop - start, dtype=np.float32)
        if scale != 1.0:
            draw *= np.float32(scale)
        out[start:stop] = f32_to_bf16_bits(draw)
    return out.reshape(shape)


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """float values -> fp8 e4m3 codes (sign, 4 exponent bits with bias 7, 3
    mantissa bits), rounded to nearest even and saturated at +-448; NaN maps
    to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.where(np.signbit(x), 0x80, 0).astype(np.int64)
    nan = np.isnan(x)
    a = np.where(nan, 0.0, np.minimum(np.abs(x), 448.0))
    m, e = np.frexp(a)                                   # a = m 2^e, 0.5 <= m < 1
    exp = e.astype(np.int64) - 1                         # a = (2m) 2^exp
    normal = (exp >= -6) & (a > 0)
    # normal: code = (exp + 7) * 8 + rint((2m - 1) * 8); a mantissa carry moves to the next exponent
    code_n = (exp + 7) * 8 + np.rint((2.0 * m - 1.0) * 8.0).astype(np.int64)
    # subnormal (and the smallest normal reached by rounding up): multiples of 2^-9
    code_s = np.rint(np.ldexp(a, 9)).astype(np.int64)
    code = np.where(normal, code_n, code_s)
    code = np.minimum(code, 0x7E)
    out = (code | sign).astype(np.uint8)
    return np.where(nan, np.uint8(0x7F), out)


def _normal_e4m3(rng: np.random.Generator, shape, scale: float) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint8)
    for start in range(0, n, _CHUNK):
        stop = min(n, start + _CHUNK)
        draw = rng.standard_normal(stop - start, dtype=np.float32)
        if scale != 1.0:
            draw *= np.float32(scale)
        out[start:stop] = f32_to_e4m3_bits(draw)
    return out.reshape(shape)


def pages_for(seq_len: int, page_size: int = 64) -> int:
    return (int(seq_len) + page_size - 1) // page_size


def make_inputs(shape: Shape, seed: int = 0, seq_lens=None, poison: bool = True,
                max_pages_per_seq: int | None = None) -> dict:
    """Draw one seeded decode batch for ``shape``.

    ``seq_lens`` overrides the drawn lengths (the draw still happens so the
    rest of the stream is unchanged).  Returns a dict of numpy arrays plus
    the pool geometry.
    """
    rng = np.random.default_rng(seed)
    ps = shape.page_size
    lo, hi = shape.ctx
    drawn = rng.integers(lo, hi + 1, size=shape.batch, dtype=np.int64)
    if seq_lens is None:
        lens = drawn.astype(np.int32)
    else:
        lens = np.asarray(seq_lens, dtype=np.int32).reshape(shape.batch)
    if (lens < 0).any():
        raise ValueError("negative sequence length")

    q_nope = _normal_bf16(rng, shape.q_nope_shape(), shape.input_scale)
    q_rope = None
    if shape.q_rope_shape() is not None:
        q_rope = _normal_bf16(rng, shape.q_rope_shape(), shape.input_scale)

    need = [pages_for(x, ps) for x in lens]
    mpps = max([pages_for(hi, ps), 1] + need)
    if max_pages_per_seq is not None:
        if max_pages_per_seq < max(need + [1]):
            raise ValueError("max_pages_per_seq below the longest sequence")
        mpps = int(max_pages_per_seq)

    if shape.paged:
        used = int(sum(need))
        spare = max(1, math.ceil(0.01 * used))
        num_pages = used + spare
    else:
        num_pages = shape.batch * mpps

    if shape.cache_dtype == "fp8":
        kv = _normal_e4m3(rng, shape.pool_shape(num_pages), shape.input_scale)
    else:
        kv = _normal_bf16(rng, shape.pool_shape(num_pages), shape.input_scale)

    if shape.paged:
        perm = rng.permutation(num_pages).astype(np.int32)
        spares = perm[used:]
        block_table = np.empty((shape.batch, mpps), dtype=np.int32)
        k = 0
        for b in range(shape.batch):
            n = need[b]
            block_table[b, :n] = perm[k:k + n]
            k += n
            fill = mpps - n
            if fill:
                block_table[b, n:] = spares[np.arange(fill) % len(spares)]
    else:
        spares = np.zeros(0, dtype=np.int32)
        block_table = None

    if poison:
        table = POISON_FP8 if shape.cache_dtype == "fp8" else POISON_BITS

        def pois(count):
            return table[rng.integers(0, len(table), size=count)]
        for p in spares:
            kv[p] = pois(kv[p].size).reshape(kv[p].shape)
        for b in range(shape.batch):
            n = need[b]
            tail = int(lens[b]) - (n - 1) * ps if n else ps
            if n == 0 or tail == ps:
                continue
            page = block_table[b, n - 1] if shape.paged else b * mpps + n - 1
            if shape.latent or shape.tied:
                seg = kv[page, tail:]
            else:
                seg = kv[page, :, tail:, :, :]
            seg[...] = pois(seg.size).reshape(seg.shape)
        if not shape.paged:
            for b in range(shape.batch):
                for i in range(need[b], mpps):
                    page = b * mpps + i
                    kv[page] = pois(kv[page].size).reshape(kv[page].shape)

    return {
        "shape": shape,
        "seed": seed,
        "seq_lens": lens,
        "q_nope": q_nope,
        "q_rope": q_rope,
        "kv": kv,
        "block_table": block_table,
        "num_pages": num_pages,
        "max_pages_per_seq": mpps,
        "sm_scale": shape.scale,
    }


def token_location(inputs: dict, b: int, j: int) -> tuple:
    """(page, slot) of token ``j`` of sequence ``b``: pure index bookkeeping."""
    ps = inputs["shape"].page_size
    bt = inputs["block_table"]
    if bt is None:
        return b * inputs["max_pages_per_seq"] + j // ps, j % ps
    return int(bt[b, j // ps]), j % ps


# The steps either side of attention: what a decode step gets before the
# cache and the absorbed query exist.  Head width d_h and value width d_v are
# 128 (the per-head widths of the pages' MLA-family models); the position
# base is 10000.
HEAD_DIM = 128
ROPE_BASE = 10000.0


def step_widths(shape: Shape) -> tuple:
    """(k of the absorption = d_h, latent columns each head reads = n of the
    absorption and k of the up-projection, d_v)."""
    per_head = shape.num_kv * shape.d_nope if shape.variant == "mlra" else shape.d_nope
    return HEAD_DIM, per_head, HEAD_DIM


def make_step_inputs(shape: Shape, seed: int = 0, seq_lens=None) -> dict:
    """Seeded inputs of the steps around decode for a latent ``shape``:

    q_c     bf16 [B][Q][H][d_h]            semantic query before absorption
    w_uk    bf16 [H][d_h][n_abs]            per-head key up-projection (MLRA: the R
                                            branch blocks side by side, n_abs = R d_c)
    w_uv    bf16 [H][n_abs][d_v]            per-head value up-projection (MLRA: the R
                                            branch blocks stacked)
    new_kv  bf16 [B][Q][row]                the newest tokens' rows, k^R not yet rotated
    pos     int32 [B][Q]                    their positions: seq_lens[b] - Q + i
    plus everything ``make_inputs`` returns (the cache, the raw q_rope, ...).
    Weights are N(0, 1/fan_in) so the projections stay O(1)."""
    if not shape.latent:
        raise ValueError("the absorbed steps concern the latent variants")
    x = make_inputs(shape, seed, seq_lens=seq_lens)
    rng = np.random.default_rng(seed + 7919)
    d_h, n_abs, d_v = step_widths(shape)
    rows = shape._rows()
    x["q_c"] = _normal_bf16(rng, rows + (shape.num_q_heads, d_h), shape.input_scale)
    x["w_uk"] = _normal_bf16(rng, (shape.num_q_heads, d_h, n_abs), 1.0 / math.sqrt(d_h))
    x["w_uv"] = _normal_bf16(rng, (shape.num_q_heads, n_abs, d_v), 1.0 / math.sqrt(n_abs))
    q = shape.q_len
    x["new_kv"] = _normal_bf16(rng, (shape.batch, q, shape.row_elems), shape.input_scale)
    lens = np.asarray(x["seq_lens"], dtype=np.int64)
    x["pos"] = np.maximum(lens[:, None] - q + np.arange(q)[None, :], 0).astype(np.int32)
    x["rope_base"] = ROPE_BASE
    return x
