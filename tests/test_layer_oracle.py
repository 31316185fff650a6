"""Pins of the layer oracle (oracle/layer.py): the projections either side of
the path, checked against closed forms, an independent library conversion and
an explicit (non-absorbed) multi-head attention, never against itself."""
import math

import numpy as np
import pytest
import torch

from oracle import layer as L
from sparse_gated_attention_b200 import synth

D_SMALL, R_SMALL = 256, 96  # free widths of the projections; the head shapes are the model's


def make_small():
    """Two sequences of 300 cached rows, two new tokens each (a chunk), small projection widths."""
    wl = synth.custom(batch=2, n_q=2, ctx=300, first_pos=150)
    x = synth.make_layer_inputs(wl, d_model=D_SMALL, q_rank=R_SMALL, seed=3)
    x["q_pos"] = torch.tensor([[150, 151], [298, 299]], dtype=torch.int32)
    return x


@pytest.fixture(scope="module")
def small():
    return make_small()


# ----------------------------------------------------------------------------- bf16 rounding
def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-6, 6, 20000)
    # exact ties: a bf16 value plus half of its last place, both parities
    base = torch.randn(4000).to(torch.bfloat16).float().numpy()
    ulp = np.abs(base) * 2.0 ** -7
    half = np.float32(2.0) ** (np.floor(np.log2(np.abs(base))) - 8)
    ties = (base + half).astype(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, -0.0, 1.0, 3.0])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = L.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)
    assert ulp.min() > 0


def test_bf16_bits_round_trip():
    v = torch.randn(1000).to(torch.bfloat16)
    bits = L.bf16_bits(v.double().numpy())
    np.testing.assert_array_equal(bits, v.view(torch.int16).numpy().view(np.uint16))


# ----------------------------------------------------------------------------- RoPE
def test_rope_is_a_complex_rotation_per_pair():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 64))
    pos = np.array([0, 1, 17, 4096, 131071])
    z = x[:, 0::2] + 1j * x[:, 1::2]
    freq = 1e6 ** (-np.arange(32) / 32.0)
    zr = z * np.exp(1j * pos[:, None] * freq)
    got = L.rope(x, pos)
    np.testing.assert_allclose(got[:, 0::2], zr.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[:, 1::2], zr.imag, rtol=0, atol=1e-12)


def test_rope_frequencies_closed_forms():
    # pair 0 turns by exactly p radians whatever the base; pair 31 by p * 1e6^(-31/32) = p * 10^-5.8125
    e = np.zeros((1, 64))
    e[0, 0] = 1.0
    r = L.rope(e, np.array([3]))
    assert r[0, 0] == pytest.approx(math.cos(3.0), abs=1e-15) and r[0, 1] == pytest.approx(math.sin(3.0), abs=1e-15)
    e = np.zeros((1, 64))
    e[0, 62] = 1.0
    p = 1_000_000
    r = L.rope(e, np.array([p]))
    ang = p * 10 ** -5.8125
    assert r[0, 62] == pytest.approx(math.cos(ang), abs=1e-9) and r[0, 63] == pytest.approx(math.sin(ang), abs=1e-9)


def test_rope_invariants():
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal((2, 64))
    assert np.linalg.norm(L.rope(a[None], np.array([777]))) == pytest.approx(np.linalg.norm(a), rel=1e-13)
    np.testing.assert_array_equal(L.rope(a[None], np.array([0]))[0], a)
    for m, n, s in [(5, 2, 100), (131071, 0, 3), (1000, 4000, 250000)]:
        d0 = L.rope(a[None], np.array([m]))[0] @ L.rope(b[None], np.array([n]))[0]
        d1 = L.rope(a[None], np.array([m + s]))[0] @ L.rope(b[None], np.array([n + s]))[0]
        assert d0 == pytest.approx(d1, rel=1e-9, abs=1e-9)


# ----------------------------------------------------------------------------- projections
def test_one_hot_hidden_state_reads_one_weight_column(small):
    """h = e_k makes every projection of h a single weight column: a transposed
    operand or a wrong slice offset shows up at once.  The expected columns are
    read from the packed matrix at its documented row offsets
    (W_DQ | W_DKV | W_IK | W_IW), not through the oracle's own slicing."""
    W = small["weights"]
    w_hq = L.to_f64(W["w_hq"])
    R = R_SMALL
    k = 37
    h = torch.zeros((1, 1, D_SMALL), dtype=torch.bfloat16)
    h[0, 0, k] = 1.0
    pos = np.array([[123]])
    p = L.project(h, pos, W, rounding=False)
    np.testing.assert_array_equal(p["c_q"][0, 0], w_hq[0:R, k])
    np.testing.assert_array_equal(p["kv_row"][0, 0, :512], w_hq[R:R + 512, k])
    np.testing.assert_allclose(p["kv_row"][0, 0, 512:], L.rope(w_hq[R + 512:R + 576, k][None], np.array([123]))[0],
                               atol=1e-15)
    np.testing.assert_array_equal(p["k_idx_row"][0, 0], w_hq[R + 576:R + 704, k])
    np.testing.assert_array_equal(p["w"][0, 0], w_hq[R + 704:R + 768, k])


def test_query_side_one_hot_latent():
    """c_q = e_r (through a W_DQ whose only non-zero is one entry) reads column r of W_UQ, W_G and W_IQ."""
    W = synth.make_layer_weights(D_SMALL, R_SMALL, seed=5)
    r, k = 11, 3
    w_hq = torch.zeros_like(W["w_hq"])
    w_hq[r, k] = 1.0
    W = dict(W, w_hq=w_hq)
    h = torch.zeros((1, 1, D_SMALL), dtype=torch.bfloat16)
    h[0, 0, k] = 1.0
    p = L.project(h, np.array([[0]]), W, rounding=False)
    w_cq = L.to_f64(W["w_cq"])
    for head in (0, 63):
        np.testing.assert_array_equal(p["q_nope"][0, 0, head], w_cq[192 * head:192 * head + 128, r])
        # position 0: RoPE is the identity
        np.testing.assert_array_equal(p["q"][0, 0, head, 512:], w_cq[192 * head + 128:192 * head + 192, r])
    np.testing.assert_array_equal(p["gate"][0, 0], w_cq[12288:12352, r])
    np.testing.assert_array_equal(p["q_idx"][0, 0].reshape(-1), w_cq[12352:, r])
    # W_UK absorbed: q_lat[h] = W_UK[h]^T q_nope[h]
    w_uk = L.to_f64(W["w_uk"])
    np.testing.assert_allclose(p["q"][0, 0, 5, :512], w_uk[5].T @ p["q_nope"][0, 0, 5], rtol=1e-13, atol=1e-15)


def test_layer_writes_only_the_new_rows(small):
    out = L.layer_forward(small["h"], small["q_pos"], small["kv"], small["k_idx"], small["weights"])
    kv0, ki0 = L.to_f64(small["kv"]), L.to_f64(small["k_idx"])
    pos = small["q_pos"].numpy()
    mask = np.ones(kv0.shape[:2], dtype=bool)
    for b in range(2):
        for t in range(2):
            mask[b, pos[b, t]] = False
            np.testing.assert_array_equal(out["kv"][b, pos[b, t]], out["kv_row"][b, t])
            np.testing.assert_array_equal(out["k_idx"][b, pos[b, t]], out["k_idx_row"][b, t])
    np.testing.assert_array_equal(out["kv"][mask], kv0[mask])
    np.testing.assert_array_equal(out["k_idx"][mask], ki0[mask])
    # every stored activation is a bf16 value
    for key in ("kv_row", "k_idx_row", "w", "q", "gate", "q_idx", "c_q"):
        np.testing.assert_array_equal(L.round_bf16(out[key]), out[key])


def test_absorbed_layer_equals_explicit_multi_head_attention(small):
    """The latent (absorbed) layer against the explicit one: per head, keys
    [W_UK c_kv ; k_rope] (192 dims), values W_UV c_kv (128 dims), queries
    [q_nope ; q_rope], torch SDPA (fp64, default scale 192^-0.5) over every
    position up to the query's (ctx <= 2048, so the selection keeps them all),
    the sigmoid gate on each head, then W_O.  Both sides start from the same
    bf16 activations; the oracle also rounds q_lat, the attention output and o
    to bf16, hence the tolerance."""
    W = small["weights"]
    Wd = L.split_weights(W)
    res = L.layer_forward(small["h"], small["q_pos"], small["kv"], small["k_idx"], W)
    c_kv, k_rope = torch.from_numpy(res["kv"][..., :512]), torch.from_numpy(res["kv"][..., 512:])
    w_uk, w_uv, w_o = (torch.from_numpy(Wd[k]) for k in ("W_UK", "W_UV", "W_O"))
    keys = torch.einsum("hdj,blj->bhld", w_uk, c_kv)                  # [B,64,L,128]
    keys = torch.cat([keys, k_rope[:, None].expand(-1, 64, -1, -1)], -1)  # [B,64,L,192]
    vals = torch.einsum("hij,blj->bhli", w_uv, c_kv)                  # [B,64,L,128]
    q_nope = torch.from_numpy(res["q_nope"])                          # [B,T,64,128]
    q_rope = torch.from_numpy(res["q"][..., 512:])                    # [B,T,64,64]
    queries = torch.cat([q_nope, q_rope], -1).permute(0, 2, 1, 3)     # [B,64,T,192]
    pos = small["q_pos"].long()
    Lc = c_kv.shape[1]
    allowed = torch.arange(Lc)[None, None, :] <= pos[:, :, None]      # [B,T,L]
    o = torch.nn.functional.scaled_dot_product_attention(queries, keys, vals, attn_mask=allowed[:, None])
    g = torch.sigmoid(torch.from_numpy(res["gate"])).permute(0, 2, 1)[..., None]  # [B,64,T,1]
    o = (o * g).permute(0, 2, 1, 3).reshape(2, 2, 64 * 128)
    y = (o @ w_o.T).numpy()
    rel = np.linalg.norm(res["y"] - y) / np.linalg.norm(y)
    assert rel < 1.5e-2, rel
    # selection: every causal position, ascending, then -1
    for b in range(2):
        for t in range(2):
            p = int(pos[b, t])
            np.testing.assert_array_equal(res["idx"][b, t, :p + 1], np.arange(p + 1))
            assert (res["idx"][b, t, p + 1:] == -1).all()


def test_output_projection_is_per_head_then_o_proj():
    """out with one non-zero head h and dim j: o = W_UV[h][:, j] in head h's slot, y = W_O @ o."""
    W = synth.make_layer_weights(D_SMALL, R_SMALL, seed=6)
    Wd = L.split_weights(W)
    out = np.zeros((1, 1, 64, 512))
    out[0, 0, 9, 300] = 1.0
    y = L.output_projection(out, W, rounding=False)
    o = np.zeros(64 * 128)
    o[9 * 128:10 * 128] = Wd["W_UV"][9][:, 300]
    np.testing.assert_allclose(y[0, 0], Wd["W_O"] @ o, rtol=1e-12, atol=1e-14)
