"""The fused selection (sga_forward_fused / sga_forward_fused_fp8) against the
fp64 oracle and against sga_forward, through the C ABI.

For decode rows the indexer writes no scores: it appends the keys at or above
a running per-query threshold to a candidate list, and the selection reads the
list.  The results must be those of the plain path: the same indices bit for
bit (and so the same attention outputs), whatever order the keys arrive in.
The cases cover thresholds that rise early (falling scores) or late (rising
scores), a K-th key whose bin holds more keys than the selection lists (every
score equal), heavy ties, other K, a query with fewer than K positions, a bad
position, workspace reuse, and the full-size decode workloads on every row.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gated_attention_b200 as sga
from sparse_gated_attention_b200 import synth

from tests.test_gpu_parity import assert_close, check_status, gen_small

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_gated_attention_b200 import build

    build.build()
    sga.load_library()
    oracle.build()
    yield
    torch.cuda.synchronize()


def _fused(x, fp8, ws, top_k=2048):
    fn = sga.forward_fused_fp8 if fp8 else sga.forward_fused
    return fn(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], top_k=top_k, ws=ws)


def _oracle(x, fp8, k=2048):
    fn = oracle.forward_e4m3 if fp8 else oracle.forward
    return fn(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"].cpu(), k=k)


def _as_fp8(x):
    y = dict(x)
    y["q_idx"], y["k_idx"] = synth.to_e4m3(x["q_idx"]), synth.to_e4m3(x["k_idx"])
    return y


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("B,T,L,pos", [(2, 1, 1500, [[1499], [700]]),  # every query has t + 1 <= K
                                       (2, 2, 6000, [[2047, 2048], [5999, 3000]]),
                                       (4, 1, 8192, [[8191]] * 4),
                                       (1, 1, 20000, [[19999]]),
                                       (2, 12, 6000, [list(range(5988, 6000)), list(range(100, 112))])])  # prefill
def test_fused_matches_oracle(fp8, B, T, L, pos):
    x = gen_small(B, T, L, pos)
    if fp8:
        x = _as_fp8(x)
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_FORWARD_FUSED)
    idx, out = _fused(x, fp8, ws)
    check_status(ws)
    want_idx, want_out = _oracle(x, fp8)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, f"fused forward, fp8 {fp8}")


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("k_range,L", [(0, 9000), (1, 20000)])
def test_fused_wide_threshold_bin(k_range, L, fp8):
    """Every score equal (no threshold ever drops a key, and the K-th key's
    bin holds all 9,000 candidates: the selection narrows it with passes over
    the list down to all 32 bits), or heavy ties; the lowest positions among
    the ties are taken.  Keys in {-1, 0, 1} are exact in E4M3."""
    B = 2
    x = gen_small(B, 1, L, [[L - 1], [L // 2]], k_range=k_range, seed=7)
    if fp8:
        x = _as_fp8(x)
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD_FUSED)
    idx, out = _fused(x, fp8, ws)
    check_status(ws)
    want_idx, want_out = _oracle(x, fp8)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, f"fused forward, k_range {k_range}")


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("order,L", [("rising", 20000), ("falling", 20000), ("rising", 70000),
                                     ("falling", 70000)])
def test_fused_monotone_scores(order, L, fp8):
    """Scores that fall with the position put the top K first, so the
    threshold rises early and drops most later keys; rising scores keep it low
    until the end.  Runs of equal scores split the K-th key's run.  The second
    call checks that the first left the counters and histograms cleared.  In
    E4M3 the key values 0..249 round onto the format's grid, which merges runs
    into longer ties; both sides use the same codes."""
    B = 2
    run = L // 250 + 1
    x = gen_small(B, 1, L, [[L - 1], [L // 2]], seed=11)
    c = torch.arange(L, device="cuda") // run
    if order == "falling":
        c = c.max() - c
    x["k_idx"] = c.to(torch.bfloat16).view(1, L, 1).expand(B, L, 128).contiguous()
    x["q_idx"] = torch.ones_like(x["q_idx"])
    if fp8:
        x = _as_fp8(x)
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD_FUSED)
    for _ in range(2):
        idx, out = _fused(x, fp8, ws)
        check_status(ws)
    want_idx, want_out = _oracle(x, fp8)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, f"fused forward, {order} scores")


@pytest.mark.parametrize("K", [64, 512])
def test_fused_other_top_k(K):
    B, L = 3, 5000
    x = gen_small(B, 1, L, [[L - 1], [2500], [K // 2]], seed=13)
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L, K), sga.OP_FORWARD_FUSED)
    idx, out = _fused(x, False, ws, top_k=K)
    check_status(ws)
    want_idx, want_out = _oracle(x, False, k=K)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, f"fused forward, top_k {K}")


def test_fused_reuses_its_workspace():
    """A bad position is reported and its row selects nothing; every exit of
    the selection clears the row's histogram and candidate counter, so the
    same zero-filled workspace serves the next calls."""
    B, L = 3, 6000
    x = gen_small(B, 1, L, [[5999], [1000], [L + 5]])
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD_FUSED)
    idx, out = _fused(x, False, ws)
    assert sga.device_status(ws) == 6
    sub = {k: v[:2] for k, v in x.items()}
    want_idx, want_out = _oracle(sub, False)
    np.testing.assert_array_equal(idx[:2].cpu().numpy(), want_idx)
    assert_close(out[:2].cpu().numpy(), want_out, "fused forward, first call")
    assert bool((idx[2] == -1).all())
    sga.clear_device_status(ws)
    for pos in ([[1500], [5999], [4500]], [[5999], [2047], [3000]]):
        x["q_pos"] = torch.as_tensor(np.asarray(pos, dtype=np.int32), device="cuda")
        idx, out = _fused(x, False, ws)
        check_status(ws)
        want_idx, want_out = _oracle(x, False)
        np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
        assert_close(out.cpu().numpy(), want_out, f"fused forward, positions {pos}")


@pytest.mark.parametrize("name,fp8", [("decode_b4_ctx8k", False), ("decode_b64_ctx32k", False),
                                      ("decode_b32_ctx128k", False), ("decode_b8_ctx256k_ties", False),
                                      ("decode_b32_ctx128k", True)])
def test_fused_workload_equals_plain_path(name, fp8):
    """At full size, in the benchmark's launch configuration: every row's
    indices equal those of sga_forward bit for bit, and so do the outputs;
    sampled rows are also checked against the oracle."""
    wl = synth.WORKLOADS[name]
    x = (synth.make_inputs_fp8 if fp8 else synth.make_inputs)(wl, device="cuda", seed=0)
    dims = sga.make_dims(wl.batch, wl.n_q, wl.ctx, wl.top_k)
    plain = sga.forward_fp8 if fp8 else sga.forward
    ws0 = sga.alloc_workspace(dims, sga.OP_FORWARD)
    idx0, out0 = plain(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws0)
    check_status(ws0)
    del ws0
    ws = sga.alloc_workspace(dims, sga.OP_FORWARD_FUSED)
    for _ in range(2):  # the second call runs on the workspace the first one left
        idx, out = _fused(x, fp8, ws, top_k=wl.top_k)
        torch.cuda.synchronize()
        check_status(ws)
        assert torch.equal(idx, idx0)
        assert torch.equal(out, out0)
    for b in sorted({0, wl.batch - 1}):
        sel = lambda t: t[b:b + 1].contiguous().cpu()  # noqa: E731
        fn = oracle.forward_e4m3 if fp8 else oracle.forward
        want_idx, want_out = fn(sel(x["q_idx"]), sel(x["w"]), sel(x["k_idx"]), sel(x["q"]), sel(x["kv"]),
                                sel(x["gate"]), sel(x["q_pos"]), k=wl.top_k)
        np.testing.assert_array_equal(idx[b].cpu().numpy(), want_idx[0])
        assert_close(out[b].cpu().numpy(), want_out[0], f"{name} seq {b}")


def test_fused_above_the_candidate_length_limit():
    """Rows longer than 262,144 positions take sga_forward's kernels (the
    candidate lists hold at most that many keys); the results are the same."""
    B, L = 1, 262144 + 64
    x = gen_small(B, 1, L, [[L - 1]], k_range=1, seed=17)
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD_FUSED)
    assert ws.numel() == sga.workspace_size(sga.make_dims(B, 1, L), sga.OP_FORWARD)
    idx, out = _fused(x, False, ws)
    check_status(ws)
    ws0 = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD)
    idx0, out0 = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws0)
    assert torch.equal(idx, idx0) and torch.equal(out, out0)
    want_idx, want_out = _oracle(x, False)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, "fused forward above the length limit")
