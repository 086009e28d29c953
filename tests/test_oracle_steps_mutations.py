"""The step pins are sharp: each plausible mistake planted in a copy of
oracle/steps.py (loaded from a temporary file, on the CPU) makes at least one
test of tests/test_oracle_steps.py fail."""

import importlib.util
import inspect

import pytest

import tests.test_oracle_steps as pins
from oracle import steps as real_steps

MUTATIONS = {
    "half_split_pairs": [("even, odd = x[..., 0::2], x[..., 1::2]",
                          "even, odd = x[..., :x.shape[-1] // 2], x[..., x.shape[-1] // 2:]"),
                         ("out[..., 0::2] = even * c - odd * s", "out[..., :x.shape[-1] // 2] = even * c - odd * s"),
                         ("out[..., 1::2] = even * s + odd * c", "out[..., x.shape[-1] // 2:] = even * s + odd * c")],
    "turned_the_other_way": [("out[..., 0::2] = even * c - odd * s", "out[..., 0::2] = even * c + odd * s"),
                             ("out[..., 1::2] = even * s + odd * c", "out[..., 1::2] = -even * s + odd * c")],
    "frequency_exponent": [("-2.0 * i / dim", "-1.0 * i / dim")],
    "key_position_plus_one": [("rope(r[width - d_rope:], p, base)", "rope(r[width - d_rope:], p + 1, base)")],
    "rope_on_the_latent": [("r[width - d_rope:] = rope(r[width - d_rope:], p, base)",
                            "r[:d_rope] = rope(r[:d_rope], p, base)")],
    "logical_page": [("page = int(block_table[b][i]) if block_table is not None else",
                      "page = b * (max_pages_per_seq or len(block_table[b])) + i if True else")],
    "values_rotated_too": [("cache[page, 1, slot] = kv[b, i, 1]",
                            "cache[page, 1, slot] = rope(kv[b, i, 1], p, base) if base is not None else kv[b, i, 1]")],
    "projection_transposed": [('"rhk,hkn->rhn"', '"rhk,hnk->rhn"')],
    "branch_outputs_not_summed": [("out[h] += (p / p.sum()) @ vals", "out[h] = (p / p.sum()) @ vals")],
}


def _mutant(tmp_path, key):
    text = open(real_steps.__file__).read()
    for old, new in MUTATIONS[key]:
        assert text.count(old) == 1, f"mutation anchor for {key} not found exactly once: {old}"
        text = text.replace(old, new)
    path = tmp_path / f"steps_{key}.py"
    path.write_text(text)
    spec = importlib.util.spec_from_file_location(f"steps_{key}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pin_calls():
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if params:
            argname, values = params[0].args
            calls += [(f"{name}[{v}]", fn, {argname: v}) for v in values]
        else:
            calls.append((name, fn, {}))
    return calls


@pytest.mark.parametrize("key", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, monkeypatch, key):
    monkeypatch.setattr(pins, "steps", _mutant(tmp_path, key))
    failed = []
    for name, fn, kwargs in _pin_calls():
        try:
            fn(**kwargs)
        except Exception:
            failed.append(name)
    assert failed, f"no pin caught the planted mistake {key}"


def test_unmutated_copy_passes(tmp_path, monkeypatch):
    MUTATIONS["_none"] = []
    try:
        monkeypatch.setattr(pins, "steps", _mutant(tmp_path, "_none"))
        for name, fn, kwargs in _pin_calls():
            fn(**kwargs)
    finally:
        del MUTATIONS["_none"]
