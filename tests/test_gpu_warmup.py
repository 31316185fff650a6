"""GPU parity of sga_indexer_warmup against the warm-up oracle.

Tolerances: the loss within 1e-4 relative, each gradient within rel-L2 1e-3
(fp32 sums of bf16 products against fp64; the key gradient is accumulated with
float atomics, so its rounding depends on the order in which the queries'
terms arrive); the selection is the oracle's, which the path reproduces bit for
bit on these integer-valued indexer inputs."""
import numpy as np
import pytest
import torch

import oracle
from oracle import warmup as W
import sparse_gated_attention_b200 as sga
from sparse_gated_attention_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_gated_attention_b200 import build
    build.build()
    sga.load_library()
    oracle.build()


def rel_l2(got, want):
    return np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)


@pytest.mark.parametrize("B,T,L,pos", [(2, 2, 3000, [[2998, 2999], [1200, 2047]]), (1, 1, 500, [[499]]),
                                       (3, 1, 9000, [[8999], [4500], [100]])])
def test_indexer_warmup_matches_oracle(B, T, L, pos):
    wl = synth.custom(batch=B, n_q=T, ctx=L, first_pos=int(np.min(pos)))
    x = synth.make_inputs(wl, device="cuda", seed=5)
    q_pos = torch.as_tensor(np.asarray(pos, dtype=np.int32), device="cuda")
    want = W.warmup_loss(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], q_pos.cpu())
    idx = torch.as_tensor(want["idx"], device="cuda")  # the oracle's selection (bit-exact with the path's)
    ws = torch.zeros(sga.indexer_warmup_workspace_size(sga.make_dims(B, T, L)), dtype=torch.uint8, device="cuda")
    got = sga.indexer_warmup(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], idx, ws=ws)
    torch.cuda.synchronize()
    assert sga.device_status(ws) == 0
    np.testing.assert_allclose(got["loss"].cpu().numpy(), want["per_query"], rtol=1e-4)
    for k in ("grad_q_idx", "grad_w", "grad_k_idx"):
        r = rel_l2(got[k].cpu().numpy().astype(np.float64), want[k])
        assert r <= 1e-3, (k, r)


@pytest.mark.parametrize("K", [64, 960])
def test_indexer_warmup_other_top_k(K):
    """Selections of one chunk (64 slots) and of 15 chunks: the per-chunk softmax
    statistics are merged over that many chunks; three queries of one sequence
    select overlapping rows, so their key gradients meet in the same rows."""
    B, T, L = 1, 3, 2500
    pos = [[2499, 1800, 900]]
    wl = synth.custom(batch=B, n_q=T, ctx=L, first_pos=int(np.min(pos)))
    x = synth.make_inputs(wl, device="cuda", seed=9)
    q_pos = torch.as_tensor(np.asarray(pos, dtype=np.int32), device="cuda")
    want = W.warmup_loss(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], q_pos.cpu(), k=K)
    idx = torch.as_tensor(want["idx"], device="cuda")
    ws = torch.zeros(sga.indexer_warmup_workspace_size(sga.make_dims(B, T, L, K)), dtype=torch.uint8, device="cuda")
    got = sga.indexer_warmup(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], idx, ws=ws)
    torch.cuda.synchronize()
    assert sga.device_status(ws) == 0
    np.testing.assert_allclose(got["loss"].cpu().numpy(), want["per_query"], rtol=1e-4)
    for k in ("grad_q_idx", "grad_w", "grad_k_idx"):
        r = rel_l2(got[k].cpu().numpy().astype(np.float64), want[k])
        assert r <= 1e-3, (k, r)


def test_indexer_warmup_back_to_back_calls():
    """Two calls on one stream with one workspace and no synchronisation between
    them, the second call's selection coming straight from sga_forward on the same
    stream.  The launches overlap through programmatic dependent launch: the
    second call's kernels must still see the forward's indices, and must not
    overwrite the workspace's logits and statistics before the first call's
    gradient kernel has read them.  Both results are checked against the oracle."""
    B, T, L = 2, 1, 3000
    wl = synth.custom(batch=B, n_q=T, ctx=L, first_pos=L - 1)
    x1 = synth.make_inputs(wl, device="cuda", seed=11)
    x2 = synth.make_inputs(wl, device="cuda", seed=12)
    want1 = W.warmup_loss(x1["q_idx"], x1["w"], x1["k_idx"], x1["q"], x1["kv"], x1["q_pos"].cpu())
    want2 = W.warmup_loss(x2["q_idx"], x2["w"], x2["k_idx"], x2["q"], x2["kv"], x2["q_pos"].cpu())
    idx1 = torch.as_tensor(want1["idx"], device="cuda")
    ws = torch.zeros(sga.indexer_warmup_workspace_size(sga.make_dims(B, T, L)), dtype=torch.uint8, device="cuda")
    fws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_FORWARD, "cuda")
    torch.cuda.synchronize()
    got1 = sga.indexer_warmup(x1["q_idx"], x1["w"], x1["k_idx"], x1["q"], x1["kv"], idx1, ws=ws)
    idx2, _ = sga.forward(x2["q_idx"], x2["w"], x2["k_idx"], x2["q"], x2["kv"], x2["gate"], x2["q_pos"], ws=fws)
    got2 = sga.indexer_warmup(x2["q_idx"], x2["w"], x2["k_idx"], x2["q"], x2["kv"], idx2, ws=ws)
    torch.cuda.synchronize()
    assert sga.device_status(ws) == 0 and sga.device_status(fws) == 0
    np.testing.assert_array_equal(idx2.cpu().numpy(), want2["idx"])
    for got, want in ((got1, want1), (got2, want2)):
        np.testing.assert_allclose(got["loss"].cpu().numpy(), want["per_query"], rtol=1e-4)
        for k in ("grad_q_idx", "grad_w", "grad_k_idx"):
            r = rel_l2(got[k].cpu().numpy().astype(np.float64), want[k])
            assert r <= 1e-3, (k, r)
