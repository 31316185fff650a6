"""Pins of the indexer warm-up oracle (oracle/warmup.py): the KL objective
against closed forms, the attention target against torch's softmax, and the
gradients against central finite differences in fp64."""
import numpy as np
import pytest
import torch

import oracle
from oracle import warmup as W
from sparse_gated_attention_b200 import synth


def test_kl_closed_forms():
    rng = np.random.default_rng(0)
    p = rng.random(50)
    p /= p.sum()
    # constant scores: the indexer's distribution is uniform, KL = log n - H(p)
    assert W.kl_to_softmax(p, np.full(50, 3.7)) == pytest.approx(np.log(50) + np.sum(p * np.log(p)), rel=1e-12)
    # scores = log p + c: the two distributions agree
    assert W.kl_to_softmax(p, np.log(p) + 11.0) == pytest.approx(0.0, abs=1e-12)
    for _ in range(20):
        assert W.kl_to_softmax(p, rng.standard_normal(50) * 5) > 0
    # a zero-probability row contributes nothing
    p0 = np.array([0.5, 0.5, 0.0])
    assert W.kl_to_softmax(p0, np.array([1.0, 1.0, -50.0])) == pytest.approx(np.log(2 / (2 + np.exp(-51))) * -1,
                                                                          rel=1e-9)


def test_attention_target_against_torch_softmax():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((64, 576))
    kv = rng.standard_normal((30, 576))
    idx = np.array([3, 7, 8, 20, 29, -1, -1])
    want = torch.softmax(torch.from_numpy(q @ kv[[3, 7, 8, 20, 29]].T) * 192 ** -0.5, dim=1).mean(0).numpy()
    np.testing.assert_allclose(W.attention_target(q, kv, idx), want, rtol=1e-12)
    # q = 0: uniform; one row: all of the mass
    np.testing.assert_allclose(W.attention_target(np.zeros((64, 576)), kv, idx), np.full(5, 0.2), rtol=1e-14)
    np.testing.assert_array_equal(W.attention_target(q, kv, np.array([4, -1])), [1.0])


def _continuous_case(seed, L=40, T=2):
    rng = np.random.default_rng(seed)
    QI = rng.standard_normal((1, T, 64, 128))
    Wt = rng.standard_normal((1, T, 64))
    KI = rng.standard_normal((1, L, 128))
    Q = rng.standard_normal((1, T, 64, 576)) * 0.3
    KV = rng.standard_normal((1, L, 576))
    return QI, Wt, KI, Q, KV


@pytest.mark.parametrize("sparse", [False, True])
def test_gradients_against_finite_differences(sparse):
    QI, Wt, KI, Q, KV = _continuous_case(2)
    L = KI.shape[1]
    if sparse:  # two queries sharing some selected rows (their key gradients add up)
        idx = np.array([[[1, 4, 9, 17, 30, 39, -1, -1], [0, 4, 9, 12, 25, 30, 38, -1]]])
    else:
        idx = np.array([[np.arange(L), np.r_[np.arange(30), -np.ones(10, int)]]])
    res = W.loss_on_selection(QI, Wt, KI, Q, KV, idx)
    rng = np.random.default_rng(3)
    h = 1e-6

    def fd(arr, ix):
        old = arr[ix]
        arr[ix] = old + h
        up = W.loss_on_selection(QI, Wt, KI, Q, KV, idx)["loss"]
        arr[ix] = old - h
        dn = W.loss_on_selection(QI, Wt, KI, Q, KV, idx)["loss"]
        arr[ix] = old
        return (up - dn) / (2 * h)

    checks = 0
    for name, arr, grad in (("q_idx", QI, res["grad_q_idx"]), ("w", Wt, res["grad_w"]),
                            ("k_idx", KI, res["grad_k_idx"])):
        for _ in range(12):
            ix = tuple(rng.integers(0, n) for n in arr.shape)
            if name == "k_idx" and ix[1] not in set(idx[ix[0]].ravel().tolist()):
                assert grad[ix] == 0.0  # a row no query selected gets no gradient
                continue
            num = fd(arr, ix)
            assert grad[ix] == pytest.approx(num, rel=1e-5, abs=1e-8), (name, ix)
            checks += 1
    assert checks >= 24


def test_stationary_point_and_selection():
    """Zero attention queries make the target uniform; zero indexer queries make
    every score 0, so the indexer's distribution is uniform too: the loss and all
    gradients vanish.  The selection is the path oracle's."""
    wl = synth.custom(batch=1, n_q=2, ctx=3000, first_pos=2998)
    x = synth.make_inputs(wl, seed=4)
    zero_q = torch.zeros_like(x["q"])
    zero_qi = torch.zeros_like(x["q_idx"])
    res = W.warmup_loss(zero_qi, x["w"], x["k_idx"], zero_q, x["kv"], x["q_pos"])
    assert res["loss"] == pytest.approx(0.0, abs=1e-12)
    for key in ("grad_q_idx", "grad_w", "grad_k_idx"):
        assert np.abs(res[key]).max() <= 1e-12, key
    res = W.warmup_loss(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["q_pos"])
    want_idx, _ = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"])
    np.testing.assert_array_equal(res["idx"], want_idx)
    assert (res["per_query"] > 0).all()
