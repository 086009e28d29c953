"""Python front of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the cpu_baseline / reference leg of ``bench.py`` may import this module.  The
CUDA library never calls it and shares no code with it; the two meet only in
the seeded inputs of ``shared_kv_caches_b200.workloads``.

``build()`` compiles ``oracle.c`` with gcc into ``liboracle.so`` next to it.
``decode()`` runs the oracle on a workload dict, ``decode_f64()`` on float64
arrays (used by the pins that need inputs bf16 cannot hold), ``merge()`` is the
split combine.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

VARIANT_IDS = {"gqa": 0, "mqa": 1, "mla": 2, "gla": 3, "mlra": 4, "gta": 5}


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "variant", "batch", "num_q_heads", "num_kv", "d_nope", "d_rope",
        "page_size", "max_pages_per_seq", "num_pages", "paged")]


def build(force: bool = False) -> str:
    """Compile the oracle (plain C, -O2, no fast-math) if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, i32p, dp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double)
        lib.orc_decode.argtypes = [ctypes.POINTER(_Shape), ctypes.c_int32, vp, vp, vp, i32p, i32p,
                                   ctypes.c_double, i32p, ctypes.c_int32, i32p, ctypes.c_int32, dp, dp,
                                   ctypes.c_int32, ctypes.c_int32]
        lib.orc_decode.restype = ctypes.c_int
        lib.orc_merge.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, dp, dp, dp, dp]
        lib.orc_merge.restype = None
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _run(variant, batch, num_q_heads, num_kv, d_nope, d_rope, page_size, max_pages_per_seq,
         num_pages, paged, elem_type, q_nope, q_rope, kv, block_table, seq_lens, sm_scale,
         b_list, nthreads, h_list=None, branch_out=False):
    lib = _load()
    branch_out = bool(branch_out) and variant == "mlra"
    shp = _Shape(VARIANT_IDS[variant], batch, num_q_heads, num_kv, d_nope, d_rope, page_size,
                 max_pages_per_seq, num_pages, 1 if paged else 0)
    dt = np.uint16 if elem_type == 0 else np.float64
    q_nope = np.ascontiguousarray(q_nope, dtype=dt)
    q_rope_arr = None if q_rope is None else np.ascontiguousarray(q_rope, dtype=dt)
    kv = np.ascontiguousarray(kv, dtype=dt)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    bt = None if block_table is None else np.ascontiguousarray(block_table, dtype=np.int32)
    if b_list is None:
        b_list = np.arange(batch, dtype=np.int32)
    b_list = np.ascontiguousarray(b_list, dtype=np.int32)
    nb = len(b_list)
    if h_list is not None:
        h_list = np.ascontiguousarray(h_list, dtype=np.int32)
    nh = num_q_heads if h_list is None else len(h_list)
    out = np.zeros((nb, nh, num_kv, d_nope) if branch_out else (nb, nh, d_nope), dtype=np.float64)
    lse_rows = nh * num_kv if variant == "mlra" else nh
    lse = np.zeros((nb, lse_rows), dtype=np.float64)
    rc = lib.orc_decode(ctypes.byref(shp), elem_type, q_nope.ctypes.data,
                        None if q_rope_arr is None else q_rope_arr.ctypes.data, kv.ctypes.data,
                        None if bt is None else _ptr(bt, ctypes.c_int32), _ptr(seq_lens, ctypes.c_int32),
                        float(sm_scale), _ptr(b_list, ctypes.c_int32), nb,
                        None if h_list is None else _ptr(h_list, ctypes.c_int32), nh,
                        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double),
                        int(nthreads or default_threads()), 1 if branch_out else 0)
    if rc != 0:
        raise RuntimeError(f"oracle failed with status {rc}")
    if variant == "mlra":
        lse = lse.reshape(nb, nh, num_kv)
    return out, lse


def e4m3_value(codes) -> np.ndarray:
    """fp8 e4m3 codes -> float64, from the format: sign in bit 7, exponent in
    bits 6..3 with bias 7, mantissa in bits 2..0; exponent 0 holds subnormals
    (m / 8 * 2^-6); exponent 15 with mantissa 7 is NaN (there are no
    infinities)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.power(2.0, e - 7))
    return sign * np.where((e == 15) & (m == 7), np.nan, val)


def _bf16_value(bits) -> np.ndarray:
    """bf16 bit patterns -> float64 (a bf16 is the top half of an fp32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _decode_fp8(inputs: dict, b_list, nthreads, sm_scale, h_list):
    """GQA over an fp8 cache: the attention of the dequantised cache, key =
    k_scale * K8 (plane 0), value = v_scale * V8 (plane 1), in fp64."""
    s = inputs["shape"]
    kv = e4m3_value(inputs["kv"])
    kv[:, 0] *= s.k_scale
    kv[:, 1] *= s.v_scale
    scale = inputs["sm_scale"] if sm_scale is None else sm_scale
    return _run(s.variant, s.batch, s.num_q_heads, s.num_kv, s.d_nope, s.d_rope, s.page_size,
                inputs["max_pages_per_seq"], inputs["num_pages"], s.paged, 1,
                _bf16_value(inputs["q_nope"]), None, kv, inputs["block_table"],
                inputs["seq_lens"], scale, b_list, nthreads, h_list)


def decode(inputs: dict, b_list=None, nthreads: int | None = None, sm_scale=None, h_list=None,
           branch_out: bool = False):
    """fp64 decode attention of a workload dict (from ``workloads.make_inputs``).

    Returns ``(out, lse)``: out ``[n_b][n_h][d_nope]`` float64 (MLRA: the sum
    over branches; with ``branch_out`` the R branch outputs ``[n_b][n_h][R][d_nope]``),
    lse ``[n_b][n_h]`` (MLRA ``[n_b][n_h][R]``), natural log.
    ``b_list`` / ``h_list`` select sequences / heads (default: all).  With
    several query tokens per sequence (``shape.q_len`` = Q > 1) the results
    carry a query axis after the sequence axis: see ``decode_queries``.
    """
    s = inputs["shape"]
    if getattr(s, "q_len", 1) > 1:
        return decode_queries(inputs, b_list, nthreads, sm_scale, h_list, branch_out)
    if getattr(s, "cache_dtype", "bf16") == "fp8":
        return _decode_fp8(inputs, b_list, nthreads, sm_scale, h_list)
    scale = inputs["sm_scale"] if sm_scale is None else sm_scale
    return _run(s.variant, s.batch, s.num_q_heads, s.num_kv, s.d_nope, s.d_rope, s.page_size,
                inputs["max_pages_per_seq"], inputs["num_pages"], s.paged, 0,
                inputs["q_nope"], inputs["q_rope"], inputs["kv"], inputs["block_table"],
                inputs["seq_lens"], scale, b_list, nthreads, h_list, branch_out)


def decode_queries(inputs: dict, b_list=None, nthreads: int | None = None, sm_scale=None, h_list=None,
                   branch_out: bool = False):
    """Decode with Q > 1 query tokens per sequence (speculative or multi-token
    decode; the GLA page sets query length 1 against longer queries).

    The Q newest tokens of sequence b are already in its cache (seq_lens[b]
    counts them); query position i attends the cache up to and including its
    own token, the first seq_lens[b] - (Q - 1 - i) tokens (causal masking
    among the new tokens).  Each (sequence, position) is therefore a
    single-token decode over that prefix of the same pages, which is how this
    computes it.  Returns out ``[n_b][Q][n_h][d_nope]`` and lse
    ``[n_b][Q][n_h]`` (MLRA ``[n_b][Q][n_h][R]``).
    """
    s = inputs["shape"]
    Q = s.q_len
    B = s.batch
    bs = np.arange(B) if b_list is None else np.asarray(b_list)
    lens = np.asarray(inputs["seq_lens"], dtype=np.int64)
    # one row per (sequence, position): its own query, the sequence's pages,
    # the causal prefix length
    q_nope = np.asarray(inputs["q_nope"])
    q_rope = None if inputs["q_rope"] is None else np.asarray(inputs["q_rope"])
    rows_q = q_nope.reshape((B * Q,) + q_nope.shape[2:])
    rows_qr = None if q_rope is None else q_rope.reshape((B * Q,) + q_rope.shape[2:])
    rows_len = np.maximum(np.repeat(lens, Q) - np.tile(Q - 1 - np.arange(Q), B), 0).astype(np.int32)
    bt = inputs["block_table"]
    if bt is None:
        # contiguous: sequence b owns pages b*mpps .. ; row v keeps its sequence's pages
        mpps = inputs["max_pages_per_seq"]
        rows_bt = np.repeat(np.arange(B, dtype=np.int32)[:, None] * mpps + np.arange(mpps, dtype=np.int32), Q, axis=0)
    else:
        rows_bt = np.repeat(np.asarray(bt), Q, axis=0)
    rows = dict(inputs, shape=s.replace(batch=B * Q, q_len=1, paged=True), q_nope=rows_q, q_rope=rows_qr,
                seq_lens=rows_len, block_table=np.ascontiguousarray(rows_bt, dtype=np.int32))
    sel = (bs[:, None] * Q + np.arange(Q)).reshape(-1)
    out, lse = decode(rows, b_list=sel, nthreads=nthreads, sm_scale=sm_scale, h_list=h_list,
                      branch_out=branch_out)
    return out.reshape((len(bs), Q) + out.shape[1:]), lse.reshape((len(bs), Q) + lse.shape[1:])


def decode_f64(variant, num_kv, q_nope, q_rope, kv, seq_lens, sm_scale, block_table=None,
               page_size=64, b_list=None, nthreads=None, branch_out=False):
    """Same computation on float64 arrays in the same layouts.

    ``q_nope`` is ``[B][H][d_nope]`` (MLRA ``[B][H][R][d_nope]``), ``kv`` is the
    pool; without ``block_table`` the pool is contiguous per sequence.
    """
    q_nope = np.asarray(q_nope, dtype=np.float64)
    batch, H = q_nope.shape[0], q_nope.shape[1]
    d_nope = q_nope.shape[-1]
    d_rope = 0 if q_rope is None else np.asarray(q_rope).shape[-1]
    kv = np.asarray(kv, dtype=np.float64)
    num_pages = kv.shape[0]
    if block_table is None:
        mpps = num_pages // batch
    else:
        mpps = np.asarray(block_table).shape[1]
    return _run(variant, batch, H, num_kv, d_nope, d_rope, page_size, mpps, num_pages,
                block_table is not None, 1, q_nope, q_rope, kv, block_table, seq_lens, sm_scale,
                b_list, nthreads, None, branch_out)


def merge(o_s: np.ndarray, lse_s: np.ndarray):
    """Combine per-part results: ``o_s [P][rows][dv]``, ``lse_s [P][rows]``."""
    lib = _load()
    o_s = np.ascontiguousarray(o_s, dtype=np.float64)
    lse_s = np.ascontiguousarray(lse_s, dtype=np.float64)
    P, rows, dv = o_s.shape
    o = np.zeros((rows, dv), dtype=np.float64)
    lse = np.zeros(rows, dtype=np.float64)
    lib.orc_merge(P, rows, dv, _ptr(o_s, ctypes.c_double), _ptr(lse_s, ctypes.c_double),
                  _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    return o, lse
