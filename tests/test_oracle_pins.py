"""Pins for the fp64 oracle: each check ties it to something other than itself.

The pins are closed forms, invariants, hand-worked fixtures (tests/golden/) and
library routines that compute the same quantity by a different route (numpy
matmul, Python's sort, torch's fp64 scaled_dot_product_attention).  Together
they are meant to fail on a dropped ReLU or weight, a wrong sign, a swapped
head/dim index, a reversed tie-break, a wrong scale, a value slice taken from
the wrong dims or a gate applied with the wrong sign.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def rand_ints(gen, lo, hi, shape):
    return torch.randint(lo, hi + 1, shape, generator=gen, dtype=torch.int32).to(torch.bfloat16)


def rand_normal(gen, shape):
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def f64(t):
    return t.to(torch.float64).numpy()


# ----------------------------------------------------------------------------- indexer


def test_indexer_worked_example(oracle_mod):
    with open(os.path.join(GOLDEN, "indexer_worked_example.json")) as f:
        g = json.load(f)
    q_idx = bf(g["q_idx"])[None, None]
    w = bf(g["w"])[None, None]
    k_idx = bf(g["k_idx"])[None]
    pos = np.array([[g["q_pos"]]], dtype=np.int32)
    sc = oracle_mod.index_scores(q_idx, w, k_idx, pos)[0, 0]
    want = np.array([float(v) for v in g["scores"]])
    np.testing.assert_array_equal(sc, want)
    for k, idx in g["topk"].items():
        got = oracle_mod.topk(sc[None], pos[0], k=int(k))[0]
        np.testing.assert_array_equal(got, np.array(idx, dtype=np.int32))


def test_indexer_zero_keys_or_weights(oracle_mod):
    gen = torch.Generator().manual_seed(1)
    B, T, L, Hi, Di = 2, 1, 40, 8, 16
    q_idx = rand_ints(gen, -3, 3, (B, T, Hi, Di))
    w = rand_ints(gen, 0, 3, (B, T, Hi))
    k_idx = rand_ints(gen, -3, 3, (B, L, Di))
    pos = np.full((B, T), L - 1, np.int32)
    assert np.all(oracle_mod.index_scores(q_idx, w, torch.zeros_like(k_idx), pos) == 0)
    assert np.all(oracle_mod.index_scores(q_idx, torch.zeros_like(w), k_idx, pos) == 0)


def test_indexer_odd_even_parts_match_matmul(oracle_mod):
    """ReLU(x) - ReLU(-x) = x and ReLU(x) + ReLU(-x) = |x|, so
    score(q) - score(-q) = k @ (Q^T w)   and   score(q) + score(-q) = |k Q^T| @ w,
    both computed here by numpy matmul instead of the oracle's loops."""
    gen = torch.Generator().manual_seed(2)
    B, T, L, Hi, Di = 2, 3, 70, 64, 128
    q_idx = rand_ints(gen, -3, 3, (B, T, Hi, Di))
    w = rand_ints(gen, 0, 3, (B, T, Hi))
    k_idx = rand_ints(gen, -3, 3, (B, L, Di))
    pos = np.full((B, T), L - 1, np.int32)
    s_pos = oracle_mod.index_scores(q_idx, w, k_idx, pos)
    s_neg = oracle_mod.index_scores(-q_idx, w, k_idx, pos)
    Q, W, K = f64(q_idx), f64(w), f64(k_idx)
    for b in range(B):
        for t in range(T):
            dots = K[b] @ Q[b, t].T  # [L, Hi]
            np.testing.assert_array_equal(s_pos[b, t] - s_neg[b, t], dots @ W[b, t])
            np.testing.assert_array_equal(s_pos[b, t] + s_neg[b, t], np.abs(dots) @ W[b, t])


def test_indexer_position_pattern(oracle_mod):
    """Only head 0 has weight; q = e0 and key s carries s mod 4 in dim 0 -> score = s mod 4.
    Negating the key entries must give 0 (the ReLU)."""
    B, T, L, Hi, Di = 1, 1, 37, 4, 8
    q = np.zeros((B, T, Hi, Di), np.float32)
    q[0, 0, 0, 0] = 1
    q[0, 0, 1, 1] = 1  # a second head that sees dim 1 only, with weight 0
    w = np.array([[[1, 0, 0, 0]]], np.float32)
    k = np.zeros((B, L, Di), np.float32)
    k[0, :, 0] = np.arange(L) % 4
    k[0, :, 1] = 100.0
    pos = np.array([[L - 1]], np.int32)
    sc = oracle_mod.index_scores(bf(q), bf(w), bf(k), pos)[0, 0]
    np.testing.assert_array_equal(sc, np.arange(L) % 4)
    sc = oracle_mod.index_scores(bf(q), bf(w), bf(-k), pos)[0, 0]
    np.testing.assert_array_equal(sc, np.zeros(L))


def test_indexer_is_causal(oracle_mod):
    gen = torch.Generator().manual_seed(3)
    B, T, L, Hi, Di = 1, 4, 50, 8, 16
    q_idx = rand_ints(gen, -3, 3, (B, T, Hi, Di))
    w = rand_ints(gen, 0, 3, (B, T, Hi))
    k_idx = rand_ints(gen, -3, 3, (B, L, Di))
    pos = np.array([[10, 20, 30, 49]], np.int32)
    a = oracle_mod.index_scores(q_idx, w, k_idx, pos)
    k2 = k_idx.clone()
    k2[0, 31:] = rand_ints(gen, -3, 3, (L - 31, Di))
    b = oracle_mod.index_scores(q_idx, w, k2, pos)
    for t, p in enumerate(pos[0]):
        assert np.all(np.isneginf(a[0, t, p + 1:]))
        assert np.all(np.isfinite(a[0, t, : p + 1]))
        if p <= 30:
            np.testing.assert_array_equal(a[0, t], b[0, t])


# ----------------------------------------------------------------------------- top-k


def brute_topk(scores, t, k):
    cand = sorted(range(t + 1), key=lambda s: (-scores[s], s))[:k]
    out = sorted(cand)
    return out + [-1] * (k - len(out))


@pytest.mark.parametrize("L,k,t", [(100, 10, 99), (100, 10, 5), (300, 64, 299), (5000, 2048, 4999), (2048, 2048, 2047)])
def test_topk_matches_python_sort(oracle_mod, L, k, t):
    rng = np.random.default_rng(L + k + t)
    scores = rng.integers(0, 40, size=L).astype(np.float64)  # many ties
    got = oracle_mod.topk(scores[None], np.array([t]), k=k)[0]
    assert got.tolist() == brute_topk(scores.tolist(), t, k)


def test_topk_special_cases(oracle_mod):
    L, k = 6000, 2048
    t = np.array([L - 1])
    ties = oracle_mod.topk(np.zeros((1, L)), t, k=k)[0]
    np.testing.assert_array_equal(ties, np.arange(k))
    rising = oracle_mod.topk(np.arange(L, dtype=np.float64)[None], t, k=k)[0]
    np.testing.assert_array_equal(rising, np.arange(L - k, L))
    falling = oracle_mod.topk(-np.arange(L, dtype=np.float64)[None], t, k=k)[0]
    np.testing.assert_array_equal(falling, np.arange(k))
    short = oracle_mod.topk(np.ones((1, L)), np.array([100]), k=k)[0]
    np.testing.assert_array_equal(short[:101], np.arange(101))
    assert np.all(short[101:] == -1)


def test_topk_invariants_random(oracle_mod):
    rng = np.random.default_rng(7)
    L, k = 20000, 2048
    scores = rng.integers(-50, 50, size=(3, L)).astype(np.float64)
    pos = np.array([L - 1, 9000, 1500])
    idx = oracle_mod.topk(scores, pos, k=k)
    for r in range(3):
        n = min(pos[r] + 1, k)
        sel = idx[r][idx[r] >= 0]
        assert len(sel) == n and np.all(np.diff(sel) > 0) and sel.max() <= pos[r]
        if pos[r] + 1 > k:
            mask = np.zeros(pos[r] + 1, bool)
            mask[sel] = True
            s = scores[r, : pos[r] + 1]
            assert s[mask].min() >= s[~mask].max()
            thr = s[mask].min()
            # at the threshold score the chosen positions precede the rejected ones
            chosen_eq = np.nonzero(mask & (s == thr))[0]
            rejected_eq = np.nonzero(~mask & (s == thr))[0]
            if len(rejected_eq):
                assert chosen_eq.max() < rejected_eq.min()


# ----------------------------------------------------------------------------- attention


def test_attention_worked_example(oracle_mod):
    with open(os.path.join(GOLDEN, "attention_worked_example.json")) as f:
        g = json.load(f)
    q = bf(g["q"])[None, None, None]
    kv = bf(g["kv"])[None]
    for case in g["cases"]:
        idx = np.array(case["idx"], np.int32)[None, None]
        gate = None if case["gate"] is None else bf([case["gate"]])[None, None]
        out = oracle_mod.attend(q, kv, idx, gate, scale=1.0, v_dim=1)
        assert abs(out[0, 0, 0, 0] - case["out"]) < 1e-15


def sdpa_dense(q, kv, t, scale, v_dim=512):
    """torch fp64 SDPA over rows [0, t] (latent form: k = row, v = row[:v_dim])."""
    qq = q.to(torch.float64)[None]  # [1, H, Dq]
    k = kv[: t + 1].to(torch.float64)[None, None].expand(1, qq.shape[1], t + 1, kv.shape[-1])
    v = kv[: t + 1, :v_dim].to(torch.float64)[None, None].expand(1, qq.shape[1], t + 1, v_dim)
    o = torch.nn.functional.scaled_dot_product_attention(qq[:, :, None, :], k, v, scale=scale)
    return o[0, :, 0, :].numpy()


def test_attention_dense_when_short(oracle_mod):
    """ctx <= K: selecting every past position is dense causal attention."""
    gen = torch.Generator().manual_seed(4)
    B, T, L, H, Dq, K = 2, 2, 300, 64, 576, 2048
    q = rand_normal(gen, (B, T, H, Dq))
    kv = rand_normal(gen, (B, L, Dq))
    pos = np.array([[150, 299], [0, 77]], np.int32)
    idx = np.full((B, T, K), -1, np.int32)
    for b in range(B):
        for t in range(T):
            idx[b, t, : pos[b, t] + 1] = np.arange(pos[b, t] + 1)
    out = oracle_mod.attend(q, kv, idx, None)
    for b in range(B):
        for t in range(T):
            want = sdpa_dense(q[b, t], kv[b], int(pos[b, t]), oracle_mod.SCALE)
            np.testing.assert_allclose(out[b, t], want, rtol=1e-12, atol=1e-12)


def test_attention_permutation_invariance(oracle_mod):
    gen = torch.Generator().manual_seed(5)
    B, T, L, H, Dq, K = 1, 1, 500, 64, 576, 256
    q = rand_normal(gen, (B, T, H, Dq))
    kv = rand_normal(gen, (B, L, Dq))
    gate = rand_normal(gen, (B, T, H))
    rng = np.random.default_rng(0)
    idx = np.sort(rng.choice(L, K - 10, replace=False)).astype(np.int32)
    idx = np.concatenate([idx, -np.ones(10, np.int32)])[None, None]
    base = oracle_mod.attend(q, kv, idx, gate)
    perm = rng.permutation(L)  # new row r holds old row perm[r]
    inv = np.argsort(perm)
    kv_p = kv[:, torch.as_tensor(perm)]
    idx_p = np.where(idx >= 0, inv[np.maximum(idx, 0)], -1).astype(np.int32)
    idx_p = idx_p[..., rng.permutation(K)]
    moved = oracle_mod.attend(q, kv_p, idx_p, gate)
    np.testing.assert_allclose(moved, base, rtol=1e-12, atol=1e-12)


def test_attention_gate_special_values(oracle_mod):
    gen = torch.Generator().manual_seed(6)
    B, T, L, H, Dq, K = 1, 1, 64, 64, 576, 64
    q = rand_normal(gen, (B, T, H, Dq))
    kv = rand_normal(gen, (B, L, Dq))
    idx = np.arange(K, dtype=np.int32)[None, None]
    plain = oracle_mod.attend(q, kv, idx, None)
    inf = oracle_mod.attend(q, kv, idx, torch.full((B, T, H), float("inf")).to(torch.bfloat16))
    ninf = oracle_mod.attend(q, kv, idx, torch.full((B, T, H), float("-inf")).to(torch.bfloat16))
    zero = oracle_mod.attend(q, kv, idx, torch.zeros((B, T, H), dtype=torch.bfloat16))
    np.testing.assert_array_equal(inf, plain)
    assert np.all(ninf == 0)
    np.testing.assert_array_equal(zero, 0.5 * plain)
    # a gate that differs per head scales each head by its own logistic value
    gh = torch.linspace(-4, 4, H).to(torch.bfloat16)
    per = oracle_mod.attend(q, kv, idx, gh[None, None])
    sig = 1.0 / (1.0 + np.exp(-gh.to(torch.float64).numpy()))
    np.testing.assert_allclose(per[0, 0], plain[0, 0] * sig[:, None], rtol=1e-13, atol=0)


def test_attention_closed_forms(oracle_mod):
    gen = torch.Generator().manual_seed(8)
    B, T, L, H, Dq, K = 1, 1, 90, 64, 576, 128
    kv = rand_normal(gen, (B, L, Dq))
    rng = np.random.default_rng(1)
    sel = np.sort(rng.choice(L, 80, replace=False)).astype(np.int32)
    idx = np.concatenate([sel, -np.ones(K - 80, np.int32)])[None, None]
    # q = 0 -> uniform weights -> the mean of the selected value rows
    out = oracle_mod.attend(torch.zeros((B, T, H, Dq), dtype=torch.bfloat16), kv, idx, None)
    mean = f64(kv[0, torch.as_tensor(sel), :512]).mean(axis=0)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(mean, (H, 512)), rtol=1e-12, atol=1e-13)
    # one candidate -> that row's value part times sigma(g)
    q = rand_normal(gen, (B, T, H, Dq))
    gate = rand_normal(gen, (B, T, H))
    one = np.full((1, 1, K), -1, np.int32)
    one[0, 0, 17] = 42
    out = oracle_mod.attend(q, kv, one, gate)
    sig = 1.0 / (1.0 + np.exp(-f64(gate[0, 0])))
    np.testing.assert_allclose(out[0, 0], sig[:, None] * f64(kv[0, 42, :512])[None], rtol=1e-13, atol=0)
    # every row equal -> that row
    same = kv[:, :1].expand(B, L, Dq).contiguous()
    out = oracle_mod.attend(q, same, idx, None)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(f64(kv[0, 0, :512]), (H, 512)), rtol=1e-13, atol=1e-14)


def test_attention_two_rows_is_logistic_mix(oracle_mod):
    """Two rows: o = sigma(z1 - z0) v1 + sigma(z0 - z1) v0 with z = (q.c) * 192^-0.5."""
    gen = torch.Generator().manual_seed(9)
    B, T, L, H, Dq = 1, 1, 4, 64, 576
    q = rand_normal(gen, (B, T, H, Dq))
    kv = rand_normal(gen, (B, L, Dq))
    idx = np.array([[[3, -1, 1, -1]]], np.int32)
    out = oracle_mod.attend(q, kv, idx, None)
    Q, C = f64(q[0, 0]), f64(kv[0])
    z1 = Q @ C[1] * 192 ** -0.5
    z3 = Q @ C[3] * 192 ** -0.5
    a = 1 / (1 + np.exp(-(z1 - z3)))
    want = a[:, None] * C[1, :512] + (1 - a)[:, None] * C[3, :512]
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-11, atol=1e-12)


def test_attention_empty_selection_is_zero(oracle_mod):
    gen = torch.Generator().manual_seed(10)
    q = rand_normal(gen, (1, 1, 64, 576))
    kv = rand_normal(gen, (1, 8, 576))
    out = oracle_mod.attend(q, kv, np.full((1, 1, 64), -1, np.int32), None)
    assert np.all(out == 0)


# ----------------------------------------------------------------------------- whole path


def test_forward_short_context_is_dense_causal(oracle_mod):
    """ctx <= 2048: the indexer cannot change anything, SGA is dense causal attention."""
    gen = torch.Generator().manual_seed(11)
    B, T, L = 2, 3, 700
    q_idx = rand_ints(gen, -3, 3, (B, T, 64, 128))
    w = rand_ints(gen, 0, 3, (B, T, 64))
    k_idx = rand_ints(gen, -3, 3, (B, L, 128))
    q = rand_normal(gen, (B, T, 64, 576))
    kv = rand_normal(gen, (B, L, 576))
    gate = rand_normal(gen, (B, T, 64))
    pos = np.array([[0, 350, 699], [10, 11, 600]], np.int32)
    idx, out = oracle_mod.forward(q_idx, w, k_idx, q, kv, gate, pos)
    for b in range(B):
        for t in range(T):
            p = int(pos[b, t])
            np.testing.assert_array_equal(idx[b, t, : p + 1], np.arange(p + 1))
            assert np.all(idx[b, t, p + 1:] == -1)
            sig = 1.0 / (1.0 + np.exp(-f64(gate[b, t])))
            want = sdpa_dense(q[b, t], kv[b], p, oracle_mod.SCALE) * sig[:, None]
            np.testing.assert_allclose(out[b, t], want, rtol=1e-12, atol=1e-12)


def test_forward_equals_steps(oracle_mod):
    gen = torch.Generator().manual_seed(12)
    B, T, L = 1, 2, 3000
    q_idx = rand_ints(gen, -3, 3, (B, T, 64, 128))
    w = rand_ints(gen, 0, 3, (B, T, 64))
    k_idx = rand_ints(gen, -3, 3, (B, L, 128))
    q = rand_normal(gen, (B, T, 64, 576))
    kv = rand_normal(gen, (B, L, 576))
    gate = rand_normal(gen, (B, T, 64))
    pos = np.array([[2500, 2999]], np.int32)
    idx, out = oracle_mod.forward(q_idx, w, k_idx, q, kv, gate, pos)
    sc = oracle_mod.index_scores(q_idx, w, k_idx, pos)
    idx2 = oracle_mod.topk(sc, pos)
    np.testing.assert_array_equal(idx, idx2)
    assert np.all(idx >= 0)
    np.testing.assert_array_equal(out, oracle_mod.attend(q, kv, idx2, gate))
    # the selection reads 2048 of 2501 / 3000 positions, and they are the best-scored ones
    for t in range(T):
        s = sc[0, t, : pos[0, t] + 1]
        chosen = np.zeros(len(s), bool)
        chosen[idx[0, t]] = True
        assert s[chosen].min() >= s[~chosen].max()


# ----------------------------------------------------------------------------- the E4M3 indexer-key variant
# The fp8 oracle reads each E4M3 code as its exact value (1 sign, 4 exponent bits
# with bias 7, 3 mantissa bits; exponent 0 subnormal; S.1111.111 NaN) and runs the
# bf16 oracle on the same values.  The decoder is pinned to the format definition
# (hand-worked codes) and to torch's float8_e4m3fn conversion.

E4M3_HAND = [
    (0x00, 0.0), (0x80, -0.0), (0x38, 1.0), (0xB8, -1.0), (0x3C, 1.5), (0x30, 0.5), (0x40, 2.0),
    (0x44, 3.0), (0xC4, -3.0), (0x7E, 448.0), (0xFE, -448.0), (0x08, 2.0 ** -6), (0x01, 2.0 ** -9),
    (0x07, 7 * 2.0 ** -9), (0x77, 240.0),
]


def test_e4m3_hand_worked_codes(oracle_mod):
    for code, want in E4M3_HAND:
        got = oracle_mod.e4m3_to_float64([code])[0]
        assert got == want and np.signbit(got) == np.signbit(want), (hex(code), got, want)
    assert np.isnan(oracle_mod.e4m3_to_float64([0x7F, 0xFF])).all()


def test_e4m3_matches_torch_for_every_code(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle_mod.e4m3_to_float64(codes)
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_e4m3_to_bf16_is_exact(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    v = oracle_mod.e4m3_to_float64(codes)
    back = (oracle_mod.e4m3_to_bf16_bits(codes).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    fin = np.isfinite(v)
    np.testing.assert_array_equal(back[fin], v[fin])


def test_index_scores_e4m3_equals_bf16_on_integer_inputs(oracle_mod):
    # integers in [-3, 3] are exact in both formats, so both caches give the same scores
    rng = np.random.default_rng(5)
    q = rng.integers(-3, 4, size=(1, 2, 64, 128)).astype(np.float32)
    k = rng.integers(-3, 4, size=(1, 300, 128)).astype(np.float32)
    w = torch.from_numpy(rng.integers(0, 4, size=(1, 2, 64)).astype(np.float32)).to(torch.bfloat16)
    pos = np.array([[299, 150]], dtype=np.int32)
    qt, kt = torch.from_numpy(q), torch.from_numpy(k)
    want = oracle_mod.index_scores(qt.to(torch.bfloat16), w, kt.to(torch.bfloat16), pos)
    got = oracle_mod.index_scores_e4m3(qt.to(torch.float8_e4m3fn), w, kt.to(torch.float8_e4m3fn), pos)
    np.testing.assert_array_equal(got, want)
