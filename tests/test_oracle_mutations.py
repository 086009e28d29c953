"""The pins are sharp: each plausible mistake planted in a copy of the oracle
(on the CPU, in a temporary directory) makes at least one pin fail.

The planted mistakes are a dropped RoPE term, a wrong sign, the K plane read
as V, a wrong GLA group, a transposed MLRA query index, a reversed latent
index, a missing scale, a missing max in the lse, logical instead of physical
pages, and a wrong merge weight.  Every mutation keeps all reads in bounds.
"""

import importlib.util
import inspect
import os
import shutil

import pytest

import tests.test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "drop_rope": ("q[dn + d] = elem(J->q_rope, J->elem_type, q_row * dr + d);", "q[dn + d] = 0.0;"),
    "sign": ("Z += exp(sc[j] - m);", "Z += exp(m - sc[j]);"),
    "v_from_k_plane": ("return (((size_t)page * planes(s) + planes(s) - 1)", "return (((size_t)page * planes(s) + 0)"),
    "gla_group": ("u = h / (H / s->num_kv);", "u = h % s->num_kv;"),
    "mlra_q_index": ("size_t q_row = ((size_t)b * H + h) * R + r;",
                     "size_t q_row = ((size_t)b * R + r) * H + h;"),
    "latent_reversed": ("return base + (size_t)u * dn + d;", "return base + (size_t)u * dn + (dn - 1 - d);"),
    "no_scale": ("sc[j] = J->sm_scale * dot;", "sc[j] = dot;"),
    "lse_no_max": ("*lse = m + log(Z);", "*lse = log(Z);"),
    "logical_pages": ("return J->block_table[(size_t)b * s->max_pages_per_seq + i];",
                      "return (int64_t)b * s->max_pages_per_seq + i;"),
    "merge_weight": ("double w = exp(lse_s[(size_t)p * rows + r] - total);",
                     "double w = exp(lse_s[(size_t)p * rows + r] - m);"),
}


def _pin_calls():
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argname, values = params[0].args
            for v in values:
                calls.append((f"{name}[{v}]", fn, {argname: v}))
        else:
            calls.append((name, fn, {}))
    return calls


def _mutant(tmp_path, key):
    src = os.path.join(ROOT, "oracle", "oracle.c")
    text = open(src).read()
    old, new = MUTATIONS[key]
    assert text.count(old) == 1, f"mutation anchor for {key} not found exactly once"
    d = tmp_path / key
    d.mkdir()
    c_path = d / "oracle.c"
    c_path.write_text(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_mut_{key}",
                                                  os.path.join(ROOT, "oracle", "oracle.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(c_path)
    mod._LIB = str(d / "liboracle.so")
    mod.build(force=True)
    return mod


@pytest.mark.parametrize("key", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, key):
    mod = _mutant(tmp_path, key)
    caught = []
    for name, fn, kw in _pin_calls():
        try:
            fn(mod, **kw)
        except (AssertionError, RuntimeError):
            caught.append(name)
    assert caught, f"no pin caught the planted mistake {key}"


def test_unmutated_copy_passes_every_pin(tmp_path):
    d = tmp_path / "clean"
    d.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "oracle.c"), d / "oracle.c")
    spec = importlib.util.spec_from_file_location("oracle_clean", os.path.join(ROOT, "oracle", "oracle.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(d / "oracle.c")
    mod._LIB = str(d / "liboracle.so")
    mod.build(force=True)
    for name, fn, kw in _pin_calls():
        fn(mod, **kw)
