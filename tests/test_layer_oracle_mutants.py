"""Planted mistakes in the layer oracle, each of which the pins in
test_layer_oracle.py must catch.  A mutant is the oracle's source with one
edit, loaded as a separate module on the CPU; the pins run against it."""
import inspect
import os
import types

import pytest

import tests.test_layer_oracle as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "layer.py")

MUTANTS = {
    "W_UK transposed": ('np.einsum("bthd,hdj->bthj", q_nope, W["W_UK"])',
                        'np.einsum("bthd,hdj->bthj", q_nope, W["W_UK"][:, :, ::-1])'),
    "W_UV rows reversed": ('np.einsum("bthj,hij->bthi", rb(out), W["W_UV"])',
                           'np.einsum("bthj,hij->bthi", rb(out), W["W_UV"][:, ::-1, :])'),
    "RoPE sign": ("out[..., 1::2] = a * s + b * c", "out[..., 1::2] = -a * s + b * c"),
    "RoPE half-split pairs": ("a, b = x[..., 0::2], x[..., 1::2]", "a, b = x[..., :d // 2], x[..., d // 2:]"),
    "RoPE frequency": ("theta = base ** (-2.0 * i / d)", "theta = base ** (-1.0 * i / d)"),
    "W_DKV slice off by one": ('"W_DKV": w_hq[o:o + KV_DIM]', '"W_DKV": w_hq[o + 1:o + KV_DIM + 1]'),
    "rope rows taken as nope": ("q_nope = rb(qh[..., :NOPE])", "q_nope = rb(qh[..., ROPE:])"),
    "bf16 truncation": ("np.round(m * 256.0) / 256.0", "np.trunc(m * 256.0) / 256.0"),
    "cache not written": ("out[b, pos[b, t]] = rows[b, t]", "pass"),
    "gate dropped": ('gate = rb(c_q @ W["W_G"].T)', 'gate = rb(c_q @ W["W_G"].T * 0.0)'),
}


def _mutant(old: str, new: str) -> types.ModuleType:
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.layer_mutant")
    mod.__package__ = "oracle"
    mod.__file__ = SRC
    exec(compile(src.replace(old, new), SRC + " (mutant)", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", list(MUTANTS))
def test_layer_pins_catch_planted_mistake(name, monkeypatch):
    monkeypatch.setattr(pins, "L", _mutant(*MUTANTS[name]))
    small = pins.make_small()
    for fn_name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not fn_name.startswith("test_"):
            continue
        try:
            fn(small) if "small" in inspect.signature(fn).parameters else fn()
        except AssertionError:
            return
    pytest.fail(f"no pin caught the mutant: {name}")
