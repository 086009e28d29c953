"""Thin ctypes binding of libkvattn.so (include/kvattn.h).

The functions carry the C names and only marshal arguments: device pointers
are Python ints (``tensor.data_ptr()``), streams are ``cudaStream_t`` handles
as ints (``torch.cuda.current_stream().cuda_stream``).  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.  If the
library is missing, loading raises.

``decode_tensors`` is a convenience that reads pointers and sizes from torch
tensors and calls ``kvattn_decode``.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvattn.so")

KVATTN_GQA, KVATTN_MQA, KVATTN_MLA, KVATTN_GLA, KVATTN_MLRA, KVATTN_GTA = range(6)
VARIANTS = {"gqa": KVATTN_GQA, "mqa": KVATTN_MQA, "mla": KVATTN_MLA, "gla": KVATTN_GLA,
            "mlra": KVATTN_MLRA, "gta": KVATTN_GTA}
KVATTN_OUT_BF16, KVATTN_OUT_FP32 = 0, 1
KVATTN_OK = 0
KVATTN_ERR_INVALID_ARG = -1
KVATTN_ERR_UNSUPPORTED = -2
KVATTN_ERR_WORKSPACE_TOO_SMALL = -3
KVATTN_ERR_MISALIGNED = -4
KVATTN_ERR_CUDA = -5
KVATTN_DEVERR_PAGE_OUT_OF_RANGE = 1
KVATTN_DEVERR_SEQ_TOO_LONG = 2
KVATTN_DEVERR_WAIT_TIMEOUT = 4
KVATTN_DEVERR_POS_OUT_OF_RANGE = 8
KERNEL_NAMES = {0: "generic", 1: "gqa", 2: "latent_tc", 3: "mqa_tc", 4: "latent_pair", 5: "gqa_fp8"}
KVATTN_CACHE_BF16, KVATTN_CACHE_FP8_E4M3 = 0, 1
KVATTN_SELFTEST_MISSED_PHASE = 256

EXPORTS = ("kvattn_get_plan", "kvattn_workspace_size", "kvattn_workspace_init", "kvattn_decode",
           "kvattn_decode_timed", "kvattn_decode_noalloc", "kvattn_get_device_error",
           "kvattn_status_string", "kvattn_version", "kvattn_selftest_bounded_wait", "kvattn_rope",
           "kvattn_append_kv", "kvattn_head_proj")
KVATTN_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class kvattn_params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "num_kv", "d_nope", "d_rope", "page_size", "max_pages_per_seq",
        "num_pages", "max_seq_len", "num_splits", "out_dtype", "q_len", "branch_out", "cache_dtype")] + [
        ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


class kvattn_plan(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("num_splits", ctypes.c_int32),
                ("pages_per_split", ctypes.c_int32), ("ctas", ctypes.c_int32),
                ("launches", ctypes.c_int32), ("header_bytes", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_uint64)]


class KvattnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {kvattn_status_string(status)} ({status})")
        self.status = status


_lib = None


def load():
    """Load libkvattn.so (must have been built; see ``build.py``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with shared_kv_caches_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(kvattn_params)
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.kvattn_get_plan.argtypes = [i32, P, ctypes.POINTER(kvattn_plan)]
    lib.kvattn_workspace_size.argtypes = [i32, P, ctypes.POINTER(ctypes.c_size_t)]
    lib.kvattn_workspace_init.argtypes = [vp, ctypes.c_size_t, vp]
    lib.kvattn_decode.argtypes = [i32, P, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                                  ctypes.c_size_t, vp]
    lib.kvattn_decode_timed.argtypes = [i32, P, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                                        ctypes.c_size_t, vp, ctypes.POINTER(ctypes.c_void_p)]
    lib.kvattn_decode_noalloc.argtypes = [i32, P, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp]
    lib.kvattn_get_device_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
    lib.kvattn_status_string.argtypes = [ctypes.c_int]
    lib.kvattn_status_string.restype = ctypes.c_char_p
    lib.kvattn_version.argtypes = []
    lib.kvattn_selftest_bounded_wait.argtypes = [vp, i32, vp]
    lib.kvattn_rope.argtypes = [vp, i32, i32, i32, i32, i32, vp, ctypes.c_float, vp]
    lib.kvattn_append_kv.argtypes = [i32, P, vp, vp, vp, vp, ctypes.c_float, vp, vp]
    lib.kvattn_head_proj.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
    for name in ("kvattn_get_plan", "kvattn_workspace_size", "kvattn_workspace_init", "kvattn_decode",
                 "kvattn_decode_timed", "kvattn_decode_noalloc", "kvattn_get_device_error",
                 "kvattn_version", "kvattn_selftest_bounded_wait", "kvattn_rope", "kvattn_append_kv",
                 "kvattn_head_proj"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def make_params(batch, num_q_heads, num_kv, d_nope, d_rope, max_pages_per_seq, num_pages,
                max_seq_len, num_splits=0, out_dtype=KVATTN_OUT_BF16, page_size=64, q_len=1,
                branch_out=0, cache_dtype=0, k_scale=1.0, v_scale=1.0) -> kvattn_params:
    return kvattn_params(int(batch), int(num_q_heads), int(num_kv), int(d_nope), int(d_rope),
                         int(page_size), int(max_pages_per_seq), int(num_pages), int(max_seq_len),
                         int(num_splits), int(out_dtype), int(q_len), int(branch_out), int(cache_dtype),
                         float(k_scale), float(v_scale))


def kvattn_version() -> int:
    return load().kvattn_version()


def kvattn_status_string(status: int) -> str:
    return load().kvattn_status_string(int(status)).decode()


def kvattn_get_plan(variant: int, params: kvattn_params) -> kvattn_plan:
    plan = kvattn_plan()
    st = load().kvattn_get_plan(int(variant), ctypes.byref(params), ctypes.byref(plan))
    if st:
        raise KvattnError(st, "kvattn_get_plan")
    return plan


def kvattn_workspace_size(variant: int, params: kvattn_params) -> int:
    n = ctypes.c_size_t(0)
    st = load().kvattn_workspace_size(int(variant), ctypes.byref(params), ctypes.byref(n))
    if st:
        raise KvattnError(st, "kvattn_workspace_size")
    return n.value


def kvattn_workspace_init(workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return load().kvattn_workspace_init(workspace, workspace_bytes, stream)


def kvattn_decode(variant, params, q_nope, q_rope, kv_cache, block_table, seq_lens, sm_scale, out,
                  lse, workspace, workspace_bytes, stream=0) -> int:
    """Call the C entry point; returns its status (0 = enqueued)."""
    return load().kvattn_decode(int(variant), ctypes.byref(params), q_nope, q_rope, kv_cache,
                                block_table, seq_lens, float(sm_scale), out, lse, workspace,
                                int(workspace_bytes), stream)


def kvattn_decode_timed(variant, params, q_nope, q_rope, kv_cache, block_table, seq_lens, sm_scale,
                        out, lse, workspace, workspace_bytes, stream, events) -> int:
    """``kvattn_decode`` recording three cudaEvent_t handles (ints or None)."""
    ev = (ctypes.c_void_p * 3)(*[e for e in events])
    return load().kvattn_decode_timed(int(variant), ctypes.byref(params), q_nope, q_rope, kv_cache,
                                      block_table, seq_lens, float(sm_scale), out, lse, workspace,
                                      int(workspace_bytes), stream, ev)


def kvattn_decode_noalloc(variant, params, q_nope, q_rope, kv_cache, block_table, seq_lens, sm_scale,
                          out, lse, device_error, stream=0) -> int:
    """Decode without a caller workspace (for callers that cannot allocate
    device memory); scratch is the library's own fixed device array."""
    return load().kvattn_decode_noalloc(int(variant), ctypes.byref(params), q_nope, q_rope, kv_cache,
                                        block_table, seq_lens, float(sm_scale), out, lse, device_error,
                                        stream)


def kvattn_selftest_bounded_wait(result: int, tries: int, stream: int = 0) -> int:
    """Enqueue the bounded-wait self-test; returns its status."""
    return load().kvattn_selftest_bounded_wait(result, int(tries), stream)


def kvattn_get_device_error(workspace: int, stream: int = 0) -> int:
    code = ctypes.c_int32(0)
    st = load().kvattn_get_device_error(workspace, stream, ctypes.byref(code))
    if st:
        raise KvattnError(st, "kvattn_get_device_error")
    return code.value


# ----------------------------------------------------------------- torch glue

def _ptr(t):
    return None if t is None else t.data_ptr()


def params_for(shape, max_pages_per_seq, num_pages, max_seq_len, num_splits=0) -> kvattn_params:
    """Params of a ``workloads.Shape`` problem."""
    return make_params(shape.batch, shape.num_q_heads, shape.num_kv, shape.d_nope, shape.d_rope,
                       max_pages_per_seq, num_pages, max_seq_len, num_splits,
                       KVATTN_OUT_FP32 if shape.out_dtype == "fp32" else KVATTN_OUT_BF16,
                       shape.page_size, shape.q_len, 1 if getattr(shape, "branch_out", False) else 0,
                       KVATTN_CACHE_FP8_E4M3 if getattr(shape, "cache_dtype", "bf16") == "fp8" else KVATTN_CACHE_BF16,
                       getattr(shape, "k_scale", 1.0), getattr(shape, "v_scale", 1.0))


def decode_tensors(variant, params, q_nope, q_rope, kv, block_table, seq_lens, sm_scale, out, lse,
                   workspace, stream=None, events=None) -> None:
    """``kvattn_decode`` on torch tensors; raises on a non-zero status.

    ``events``: three ``torch.cuda.Event`` (or None) recorded around the split
    pass and the combine pass on the launching stream.
    """
    if stream is None:
        import torch
        stream = torch.cuda.current_stream(q_nope.device).cuda_stream
    args = (variant, params, _ptr(q_nope), _ptr(q_rope), _ptr(kv), _ptr(block_table), _ptr(seq_lens),
            sm_scale, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
            stream)
    if events is None:
        st = kvattn_decode(*args)
    else:
        st = kvattn_decode_timed(*args, [None if e is None else e.cuda_event for e in events])
    if st:
        raise KvattnError(st, "kvattn_decode")


# ------------------------------------------------- the steps either side

def kvattn_rope(x, rows, row_elems, rot_offset, rot_dim, rows_per_pos, pos, rope_base, stream=0) -> int:
    return load().kvattn_rope(x, int(rows), int(row_elems), int(rot_offset), int(rot_dim), int(rows_per_pos),
                              pos, float(rope_base), stream)


def kvattn_append_kv(variant, params, new_kv, pos, block_table, kv_cache, rope_base, device_error=None,
                     stream=0) -> int:
    return load().kvattn_append_kv(int(variant), ctypes.byref(params), new_kv, pos, block_table, kv_cache,
                                   float(rope_base), device_error, stream)


def kvattn_head_proj(x, w, y, out_dtype, rows, heads, k, n, device_error=None, stream=0) -> int:
    return load().kvattn_head_proj(x, w, y, int(out_dtype), int(rows), int(heads), int(k), int(n),
                                   device_error, stream)


def rope_tensor(x, pos, rot_offset, rot_dim, rope_base, rows_per_pos):
    """In-place RoPE on a contiguous bf16 tensor whose last axis is the row
    (argument marshalling only; the rotation runs in kvattn_rope)."""
    import torch
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and pos.dtype == torch.int32
    row_elems = x.shape[-1]
    rows = x.numel() // row_elems
    st = kvattn_rope(_ptr(x), rows, row_elems, rot_offset, rot_dim, rows_per_pos, _ptr(pos), rope_base,
                     torch.cuda.current_stream(x.device).cuda_stream)
    if st:
        raise KvattnError(st, "kvattn_rope")


def head_proj_tensor(x, w, out_fp32=False):
    """y[r, h] = x[r, h] @ w[h] for bf16 x [rows][H][k] and w [H][k][n] on the
    device (kvattn_head_proj); returns y [rows][H][n]."""
    import torch
    assert x.dtype == torch.bfloat16 and w.dtype == torch.bfloat16 and x.is_contiguous() and w.is_contiguous()
    rows, heads, k = x.shape
    n = w.shape[2]
    assert w.shape[:2] == (heads, k)
    y = torch.empty((rows, heads, n), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=x.device)
    st = kvattn_head_proj(_ptr(x), _ptr(w), _ptr(y), KVATTN_OUT_FP32 if out_fp32 else KVATTN_OUT_BF16, rows,
                          heads, k, n, None, torch.cuda.current_stream(x.device).cuda_stream)
    if st:
        raise KvattnError(st, "kvattn_head_proj")
    return y
