"""The seeded input recipe still draws the bytes recorded in tests/golden/input_digests.json
(written by tests/golden/make_input_digests.py with the same torch build)."""
import json
import os

import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def test_input_recipe_bytes_are_unchanged():
    import importlib.util

    spec = importlib.util.spec_from_file_location("make_input_digests",
                                                  os.path.join(HERE, "golden", "make_input_digests.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(os.path.join(HERE, "golden", "input_digests.json")) as f:
        stored = json.load(f)
    if stored["torch"].split("+")[0] != torch.__version__.split("+")[0]:
        pytest.skip(f"digests written with torch {stored['torch']}, running {torch.__version__}")
    assert mod.cases() == stored["digests"]
