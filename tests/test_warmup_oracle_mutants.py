"""Planted mistakes in the warm-up oracle, each of which the pins in
test_warmup_oracle.py must catch (the mutant is loaded as a separate module)."""
import inspect
import os
import types

import pytest

import tests.test_warmup_oracle as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "warmup.py")

MUTANTS = {
    "gradient sign": ("g = r - p ", "g = p - r "),
    "ReLU mask dropped": ("act = (a > 0) * Wt[b, t][:, None] * g[None, :]", "act = Wt[b, t][:, None] * g[None, :]"),
    "head weight dropped": ("act = (a > 0) * Wt[b, t][:, None] * g[None, :]", "act = (a > 0) * g[None, :]"),
    "key gradient overwritten, not added": ("np.add.at(g_ki[b], sel, act.T @ QI[b, t])",
                                            "g_ki[b, sel] = act.T @ QI[b, t]"),
    "KL reversed": ("return float(np.sum(p[nz] * (np.log(p[nz]) - log_r[nz])))",
                    "return float(np.sum(np.exp(log_r) * (log_r - np.log(np.maximum(p, 1e-300)))))"),
    "heads pooled before the softmax": ("return (e / e.sum(axis=1, keepdims=True)).mean(axis=0)",
                                        "return e.sum(axis=0) / e.sum()"),
    "no softmax scale": ("z = (q @ kv[sel].T) * scale", "z = (q @ kv[sel].T)"),
    "weight gradient without ReLU": ("g_w[b, t] = relu @ g", "g_w[b, t] = a @ g"),
}


def _mutant(old, new):
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.warmup_mutant")
    mod.__package__ = "oracle"
    mod.__file__ = SRC
    exec(compile(src.replace(old, new), SRC + " (mutant)", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", list(MUTANTS))
def test_warmup_pins_catch_planted_mistake(name, monkeypatch):
    monkeypatch.setattr(pins, "W", _mutant(*MUTANTS[name]))
    for fn_name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not fn_name.startswith("test_"):
            continue
        params = inspect.signature(fn).parameters
        cases = [{"sparse": False}, {"sparse": True}] if "sparse" in params else [{}]
        for kw in cases:
            try:
                fn(**kw)
            except AssertionError:
                return
    pytest.fail(f"no pin caught the mutant: {name}")
