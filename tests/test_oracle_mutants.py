"""Planted mistakes: every plausible slip in the oracle must trip at least one pin.

Each mutant is the oracle source with one textual change (a dropped ReLU, a
dropped weight, a transposed index, an off-by-one causal mask, a reversed
tie-break, a missing scale, the value taken from the wrong dims, a flipped gate
sign, a missing softmax normaliser, one slot short, unsorted output).  It is
compiled into a temporary directory on the CPU and run through the pins in
test_oracle_pins.py; the test asserts that some pin fails.  The committed
oracle is never modified.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = {
    "no_relu": [("total += wt[j] * std::max(0.0, dot);", "total += wt[j] * dot;")],
    "no_weight": [("total += wt[j] * std::max(0.0, dot);", "total += std::max(0.0, dot);")],
    "transposed_q": [("q[size_t(j) * Di + d]", "q[size_t(d) * Hi + j]")],
    "causal_off_by_one": [("if (s > t) {", "if (s >= t) {")],
    "tie_to_higher_position": [
        ("cand[s] = {-sc[s], int32_t(s)};", "cand[s] = {-sc[s], int32_t(n - 1 - s)};"),
        ("chosen.push_back(cand[j].second);", "chosen.push_back(int32_t(n - 1 - cand[j].second));"),
    ],
    "no_scale": [("z.push_back(dot * scale);", "z.push_back(dot);")],
    "value_from_tail_dims": [("acc[d] += p * bf16_value(cs[d]);", "acc[d] += p * bf16_value(cs[d + (Dq - Dv)]);")],
    "gate_sign": [("std::exp(-bf16_value(gate[row * H + h]))", "std::exp(bf16_value(gate[row * H + h]))")],
    "no_normaliser": [("o[d] = acc[d] / denom * g;", "o[d] = acc[d] * g;")],
    "one_slot_short": [("for (int j = 0; j < K; ++j) chosen.push_back", "for (int j = 0; j < K - 1; ++j) chosen.push_back")],
    "unsorted_output": [("std::sort(chosen.begin(), chosen.end());", "")],
}

PIN_CALLS = [
    pins.test_indexer_worked_example,
    pins.test_indexer_zero_keys_or_weights,
    pins.test_indexer_odd_even_parts_match_matmul,
    pins.test_indexer_position_pattern,
    pins.test_indexer_is_causal,
    lambda m: pins.test_topk_matches_python_sort(m, 300, 64, 299),
    pins.test_topk_special_cases,
    pins.test_topk_invariants_random,
    pins.test_attention_worked_example,
    pins.test_attention_dense_when_short,
    pins.test_attention_gate_special_values,
    pins.test_attention_closed_forms,
    pins.test_attention_two_rows_is_logistic_mix,
]


def _compile_mutant(name, edits, tmpdir):
    with open(os.path.join(os.path.dirname(oracle.__file__), "sga_oracle.cpp")) as f:
        src = f.read()
    for old, new in edits:
        assert src.count(old) == 1, f"{name}: edit target not found exactly once: {old!r}"
        src = src.replace(old, new)
    path = os.path.join(tmpdir, f"{name}.cpp")
    with open(path, "w") as f:
        f.write(src)
    so = os.path.join(tmpdir, f"lib{name}.so")
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-shared", "-fPIC", "-pthread", path, "-o", so])
    return so


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, oracle_mod):
    so = _compile_mutant(name, MUTANTS[name], str(tmp_path))
    real = oracle_mod._load()
    lib = ctypes.CDLL(so)
    for fn in ("oracle_index_scores", "oracle_topk", "oracle_attend", "oracle_forward", "oracle_hardware_threads"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    caught = []
    oracle_mod._lib = lib
    try:
        for call in PIN_CALLS:
            try:
                call(oracle_mod)
            except (AssertionError, ValueError) as e:  # noqa: PERF203
                caught.append(getattr(call, "__name__", "lambda") + ": " + str(e).splitlines()[0][:80] if str(e) else "")
    finally:
        oracle_mod._lib = real
    assert caught, f"mutant {name} passed every pin"
