"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Indices and indexer scores must match bit for bit (the indexer inputs are
integers, so every score is an exact fp32 integer).  Attention outputs must be
within rel-L2 <= 1e-3 and max-abs <= 1e-2 of the oracle.  Small cases cover
several tiles, ragged tails, multi-query rows, empty slots and the degenerate
cases; the full-size workloads run in the same launch configuration as the
benchmark and are checked on sampled queries.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gated_attention_b200 as sga
from sparse_gated_attention_b200 import synth

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS = 1e-2


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


def assert_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = got - want
    rel = np.linalg.norm(err) / max(np.linalg.norm(want), 1e-30)
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS, f"{what}: rel-L2 {rel:.3e}, max-abs {mx:.3e}"


def check_status(ws):
    assert sga.device_status(ws) == 0


def gen_small(B, T, L, pos, k_range=3, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dev = "cuda"
    q_idx = torch.randint(-3, 4, (B, T, 64, 128), generator=g, device=dev, dtype=torch.int32).to(torch.bfloat16)
    w = torch.randint(0, 4, (B, T, 64), generator=g, device=dev, dtype=torch.int32).to(torch.bfloat16)
    k_idx = torch.randint(-k_range, k_range + 1, (B, L, 128), generator=g, device=dev, dtype=torch.int32).to(torch.bfloat16)
    q = torch.randn((B, T, 64, 576), generator=g, device=dev).to(torch.bfloat16)
    kv = torch.randn((B, L, 576), generator=g, device=dev).to(torch.bfloat16)
    gate = torch.randn((B, T, 64), generator=g, device=dev).to(torch.bfloat16)
    q_pos = torch.as_tensor(np.asarray(pos, dtype=np.int32).reshape(B, T), device=dev)
    return dict(q_idx=q_idx, w=w, k_idx=k_idx, q=q, kv=kv, gate=gate, q_pos=q_pos)


# ----------------------------------------------------------------------------- step 1: indexer

INDEX_CASES = [
    (1, 1, 128, [[127]]),
    (2, 1, 1000, [[999], [500]]),  # ragged last tile, a query in the middle
    (3, 2, 700, [[0, 699], [130, 131], [255, 256]]),  # several queries per sequence
    (4, 1, 8192, [[8191]] * 4),
    (2, 3, 5000, [[4000, 4001, 4999], [17, 2047, 2048]]),
]


@pytest.mark.parametrize("B,T,L,pos", INDEX_CASES)
def test_index_scores_bit_exact(B, T, L, pos):
    x = gen_small(B, T, L, pos)
    scores = torch.full((B, T, L), float("nan"), device="cuda")
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_INDEX_SCORES)
    sga.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"], scores=scores, ws=ws)
    check_status(ws)
    want = oracle.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"].cpu())
    got = scores.cpu().numpy().astype(np.float64)
    pos = np.asarray(pos)
    for b in range(B):
        for t in range(T):
            p = pos[b, t]
            np.testing.assert_array_equal(got[b, t, : p + 1], want[b, t, : p + 1])


# Eight or more queries per sequence take the prefill indexer (blocks of 8
# queries share each key tile).  Cases: one exact block over whole tiles; a
# ragged block (13 = 8 + 5) over a ragged last tile; a block of one row;
# positions out of order inside a block, including 0 and small ones.
def _prefill_positions(B, T, L, seed):
    rng = np.random.default_rng(seed)
    pos = rng.integers(0, L, size=(B, T))
    pos[0, 0] = L - 1
    pos[-1, -1] = 0
    if T > 2:
        pos[0, 1] = 5
    return pos.tolist()


PREFILL_INDEX_CASES = [
    (1, 8, 1024, [list(range(1016, 1024))]),
    (2, 13, 3001, _prefill_positions(2, 13, 3001, 1)),
    (3, 9, 700, _prefill_positions(3, 9, 700, 2)),
    (1, 40, 5000, _prefill_positions(1, 40, 5000, 3)),
    (1, 64, 8192, [list(range(8128, 8192))]),
]


@pytest.mark.parametrize("B,T,L,pos", PREFILL_INDEX_CASES)
def test_index_scores_prefill_bit_exact(B, T, L, pos):
    x = gen_small(B, T, L, pos)
    scores = torch.full((B, T, L), float("nan"), device="cuda")
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_INDEX_SCORES)
    sga.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"], scores=scores, ws=ws)
    check_status(ws)
    want = oracle.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"].cpu())
    got = scores.cpu().numpy().astype(np.float64)
    pos = np.asarray(pos)
    for b in range(B):
        for t in range(T):
            p = pos[b, t]
            np.testing.assert_array_equal(got[b, t, : p + 1], want[b, t, : p + 1])
            assert np.all(np.isnan(got[b, t, p + 1:])), "entries past the position are left unwritten"


def test_index_scores_prefill_bad_position():
    """A row of a block with a position outside [0, L) is skipped and reported;
    the other rows of its block are exact."""
    B, T, L = 1, 10, 1000
    pos = [[999, 500, 1005, 3, 998, 997, 996, 995, 994, 993]]
    x = gen_small(B, T, L, pos)
    scores = torch.full((B, T, L), float("nan"), device="cuda")
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_INDEX_SCORES)
    sga.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"], scores=scores, ws=ws)
    assert sga.device_status(ws) == 6
    got = scores.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(got[0, 2]))
    good = [t for t in range(T) if t != 2]
    qp = x["q_pos"][:, good].contiguous()
    want = oracle.index_scores(x["q_idx"][:, good].contiguous(), x["w"][:, good].contiguous(), x["k_idx"], qp.cpu())
    for i, t in enumerate(good):
        p = pos[0][t]
        np.testing.assert_array_equal(got[0, t, : p + 1], want[0, i, : p + 1])


def test_index_scores_ties_workload_exact():
    x = gen_small(2, 1, 20000, [[19999], [12345]], k_range=1)
    scores = sga.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"])
    want = oracle.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"].cpu())
    got = scores.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(got[0, 0], want[0, 0])
    np.testing.assert_array_equal(got[1, 0, :12346], want[1, 0, :12346])


# ----------------------------------------------------------------------------- step 2: top-k


def run_topk(scores_np, pos_np, k):
    rows, L = scores_np.shape
    sc = torch.as_tensor(scores_np.astype(np.float32)).reshape(rows, 1, L).cuda()
    qp = torch.as_tensor(pos_np.astype(np.int32)).reshape(rows, 1).cuda()
    ws = sga.alloc_workspace(sga.make_dims(rows, 1, L, k), sga.OP_TOPK_SELECT)
    idx = sga.topk_select(sc, qp, top_k=k, ws=ws)
    check_status(ws)
    want = oracle.topk(scores_np.astype(np.float32).astype(np.float64), pos_np, k=k)
    return idx.cpu().numpy().reshape(rows, k), want


@pytest.mark.parametrize("kind", ["int_spread", "heavy_ties", "all_equal", "rising", "falling", "narrow_float",
                                  "signed", "zeros_signed"])
def test_topk_bit_exact(kind):
    rng = np.random.default_rng(abs(hash(kind)) % 2**32)
    L, K = 100000, 2048
    s = np.arange(L, dtype=np.float64)
    if kind == "int_spread":
        sc = rng.integers(0, 6000, size=(3, L)).astype(np.float64)
    elif kind == "heavy_ties":
        sc = rng.integers(0, 12, size=(3, L)).astype(np.float64)
    elif kind == "all_equal":
        sc = np.full((3, L), 7.0)
    elif kind == "rising":
        sc = np.stack([s, s, s])
    elif kind == "falling":
        sc = np.stack([-s, -s, -s])
    elif kind == "narrow_float":  # all keys share their top bits: deep radix levels
        sc = (1000.0 + rng.integers(0, 50000, size=(3, L)) * 2.0 ** -10).astype(np.float32).astype(np.float64)
    elif kind == "signed":
        sc = rng.normal(size=(3, L)).astype(np.float32).astype(np.float64)
    else:  # +0.0 and -0.0 rank equal, ties go to the lower position
        sc = np.where(rng.random((3, L)) < 0.5, 0.0, -0.0) * np.ones((3, L))
        sc[:, ::7] = -1.0
    pos = np.array([L - 1, 54321, 2047])
    got, want = run_topk(sc, pos, K)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("L,K,t", [(64, 64, 63), (1000, 64, 999), (1000, 128, 50), (5000, 512, 4999),
                                   (3000, 2048, 2046), (262144, 2048, 262143)])
def test_topk_sizes(L, K, t):
    rng = np.random.default_rng(L + K)
    sc = rng.integers(0, 300, size=(2, L)).astype(np.float64)
    got, want = run_topk(sc, np.array([t, t // 2]), K)
    np.testing.assert_array_equal(got, want)


# Rows of up to 8 x 32768 positions are selected with each CTA's segment held
# in shared memory; longer rows stream.  A row stride that is not a multiple
# of 4 takes plain loads instead of bulk copies.  Many rows with a long stride
# give clusters of 3 and 5 CTAs.  The streaming kernel keeps a CTA's selection
# and tie words in shared memory while its segment spans at most 65,536
# positions, i.e. rows up to 8 x 65,536; longer rows (600,001 and up) keep them
# in the workspace.
@pytest.mark.parametrize("rows,L,kind", [(2, 100001, "int"), (2, 100001, "ties"), (100, 70000, "int"),
                                         (40, 131075, "ties"), (2, 300000, "int"), (2, 300000, "ties"),
                                         (3, 300003, "int"), (1, 262145, "float"),
                                         (2, 600004, "int"), (2, 600001, "ties"), (2, 600001, "int"),
                                         (2, 600004, "ties"), (1, 700000, "float")])
def test_topk_kernel_paths(rows, L, kind):
    rng = np.random.default_rng(rows * 7 + L)
    if kind == "int":
        sc = rng.integers(0, 4000, size=(rows, L)).astype(np.float64)
    elif kind == "ties":
        sc = rng.integers(0, 9, size=(rows, L)).astype(np.float64)
    else:
        sc = rng.normal(size=(rows, L)).astype(np.float32).astype(np.float64)
    pos = rng.integers(2048, L, size=rows)
    pos[0] = L - 1
    if L > 8 * 65536 and rows > 1:
        pos[1] = L - 2  # every row of the long cases takes the workspace words
    got, want = run_topk(sc, pos, 2048)
    np.testing.assert_array_equal(got, want)


# ----------------------------------------------------------------------------- steps 3-4: attention + gate


def random_idx(rng, B, T, L, K, holes=0.1, shuffle=True):
    idx = np.full((B, T, K), -1, np.int32)
    for b in range(B):
        for t in range(T):
            n = min(L, K)
            sel = rng.choice(L, n, replace=False).astype(np.int32)
            sel[rng.random(n) < holes] = -1
            if not shuffle:
                sel = np.sort(sel)
            idx[b, t, :n] = sel
    return idx


@pytest.mark.parametrize("B,T,L,K,gated", [(1, 1, 3000, 2048, True), (4, 1, 5000, 2048, True),
                                           (2, 3, 2500, 2048, False), (32, 1, 4096, 2048, True),
                                           (3, 1, 700, 64, True), (1, 2, 900, 192, True),
                                           (1, 1, 2000, 320, True), (2, 1, 3000, 448, False),
                                           (200, 1, 3000, 2048, True)])
def test_attend_matches_oracle(B, T, L, K, gated):
    rng = np.random.default_rng(B * 1000 + L)
    x = gen_small(B, T, L, np.full((B, T), L - 1))
    idx = torch.as_tensor(random_idx(rng, B, T, L, K)).cuda()
    gate = x["gate"] if gated else None
    ws = sga.alloc_workspace(sga.make_dims(B, T, L, K), sga.OP_SPARSE_MLA_ATTEND)
    out = sga.sparse_mla_attend(x["q"], x["kv"], idx, gate, ws=ws)
    check_status(ws)
    want = oracle.attend(x["q"], x["kv"], idx.cpu(), None if gate is None else gate)
    assert_close(out.cpu().numpy(), want, f"attend B{B} T{T} L{L} K{K}")


def test_attend_degenerate_slots():
    """Rows with every slot empty give zeros; a single filled slot gives that row's value part."""
    B, L, K = 3, 500, 2048
    x = gen_small(B, 1, L, np.full((B, 1), L - 1))
    idx = np.full((B, 1, K), -1, np.int32)
    idx[1, 0, 1500] = 42
    idx[2, 0, :L] = np.arange(L)
    out = sga.sparse_mla_attend(x["q"], x["kv"], torch.as_tensor(idx).cuda(), x["gate"]).cpu().numpy()
    assert np.all(out[0] == 0)
    want = oracle.attend(x["q"], x["kv"], idx, x["gate"])
    assert_close(out, want, "degenerate")


def test_attend_permutation_invariance_and_gate():
    B, L, K = 2, 4000, 2048
    rng = np.random.default_rng(3)
    x = gen_small(B, 1, L, np.full((B, 1), L - 1))
    idx = random_idx(rng, B, 1, L, K, shuffle=False)
    base = sga.sparse_mla_attend(x["q"], x["kv"], torch.as_tensor(idx).cuda(), x["gate"]).cpu().numpy()
    perm = rng.permutation(L)
    inv = np.argsort(perm)
    kv_p = x["kv"][:, torch.as_tensor(perm).cuda()].contiguous()
    idx_p = np.where(idx >= 0, inv[np.maximum(idx, 0)], -1).astype(np.int32)
    idx_p = idx_p[..., rng.permutation(K)]
    moved = sga.sparse_mla_attend(x["q"], kv_p, torch.as_tensor(np.ascontiguousarray(idx_p)).cuda(), x["gate"])
    assert_close(moved.cpu().numpy(), base, "permuted")
    # gate = +inf -> ungated; gate = -inf -> zeros; gate = 0 -> half
    inf = torch.full_like(x["gate"], float("inf"))
    a = sga.sparse_mla_attend(x["q"], x["kv"], torch.as_tensor(idx).cuda(), inf).cpu().numpy()
    b = sga.sparse_mla_attend(x["q"], x["kv"], torch.as_tensor(idx).cuda(), None).cpu().numpy()
    np.testing.assert_array_equal(a, b)
    z = sga.sparse_mla_attend(x["q"], x["kv"], torch.as_tensor(idx).cuda(), -inf).cpu().numpy()
    assert np.all(z == 0)
    h = sga.sparse_mla_attend(x["q"], x["kv"], torch.as_tensor(idx).cuda(), torch.zeros_like(x["gate"])).cpu().numpy()
    np.testing.assert_allclose(h, 0.5 * b, rtol=1e-6, atol=1e-7)


# ----------------------------------------------------------------------------- whole path


@pytest.mark.parametrize("B,T,L,pos", [(2, 1, 1500, [[1499], [700]]),  # ctx <= 2048: dense
                                       (2, 2, 6000, [[2047, 2048], [5999, 3000]]),
                                       (4, 1, 8192, [[8191]] * 4),
                                       (2, 12, 6000, _prefill_positions(2, 12, 6000, 4)),  # prefill indexer
                                       (1, 16, 9000, [list(range(8984, 9000))])])
def test_forward_matches_oracle(B, T, L, pos):
    x = gen_small(B, T, L, pos)
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_FORWARD)
    idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    check_status(ws)
    want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"].cpu())
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, "forward")


@pytest.mark.parametrize("k_range,L", [(0, 9000), (1, 20000)])
def test_forward_wide_threshold_bin(k_range, L):
    """Index keys all zero (every score equal: the K-th score's bin holds all
    9,000 keys, more than the 8,192-key candidate list, so the selection
    narrows it with passes over its positions) or in {-1, 0, 1} (heavy ties);
    both take the lowest positions among the ties."""
    B = 2
    x = gen_small(B, 1, L, [[L - 1], [L // 2]], k_range=k_range, seed=7)
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD)
    idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    check_status(ws)
    want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"].cpu())
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, f"forward, k_range {k_range}")


@pytest.mark.parametrize("order,L", [("rising", 20000), ("falling", 20000), ("rising", 70000)])
def test_forward_monotone_scores(order, L):
    """Scores that rise (or fall) with the position, in runs of equal values:
    the top K are the last (or first) positions, the K-th key's run is split,
    and its lowest positions are taken; the second call checks that the first
    left the workspace's histograms cleared."""
    B = 2
    run = L // 250 + 1
    x = gen_small(B, 1, L, [[L - 1], [L // 2]], seed=11)
    c = torch.arange(L, device="cuda") // run
    if order == "falling":
        c = c.max() - c
    x["k_idx"] = c.to(torch.bfloat16).view(1, L, 1).expand(B, L, 128).contiguous()
    x["q_idx"] = torch.ones_like(x["q_idx"])
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD)
    for _ in range(2):
        idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
        check_status(ws)
    want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"].cpu())
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, f"forward, {order} scores")


@pytest.mark.parametrize("K", [64, 512])
def test_forward_other_top_k(K):
    """The whole path with fewer selected positions per query: the top-k's
    candidate refinement, the attention's chunk count and its split merge all
    follow K; one query sits early enough that it has fewer than K positions."""
    B, L = 3, 5000
    pos = [[L - 1], [2500], [K // 2]]
    x = gen_small(B, 1, L, pos, seed=13)
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L, K), sga.OP_FORWARD)
    idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], top_k=K, ws=ws)
    check_status(ws)
    want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"],
                                        x["q_pos"].cpu(), k=K)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, f"forward, top_k {K}")


def test_forward_reuses_its_workspace():
    """The selection clears the indexer's histograms after reading them, on
    every exit (full selection, t + 1 <= K, bad position), so one zero-filled
    workspace serves consecutive calls."""
    B, L = 3, 6000
    x = gen_small(B, 1, L, [[5999], [1000], [L + 5]])
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD)
    idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    assert sga.device_status(ws) == 6  # the bad position is reported
    sub = {k: v[:2] for k, v in x.items()}
    want_idx, want_out = oracle.forward(sub["q_idx"], sub["w"], sub["k_idx"], sub["q"], sub["kv"], sub["gate"],
                                        sub["q_pos"].cpu())
    np.testing.assert_array_equal(idx[:2].cpu().numpy(), want_idx)
    assert_close(out[:2].cpu().numpy(), want_out, "forward, first call")
    sga.clear_device_status(ws)
    for pos in ([[1500], [5999], [4500]], [[5999], [2047], [3000]]):
        x["q_pos"] = torch.as_tensor(np.asarray(pos, dtype=np.int32), device="cuda")
        idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
        check_status(ws)
        want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"],
                                            x["q_pos"].cpu())
        np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
        assert_close(out.cpu().numpy(), want_out, f"forward, positions {pos}")


def test_device_status_reports_bad_arguments():
    B, L = 2, 3000
    x = gen_small(B, 1, L, [[L - 1], [L - 1]])
    ws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD)
    bad_pos = torch.tensor([[L - 1], [L]], dtype=torch.int32, device="cuda")
    sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], bad_pos, ws=ws)
    assert sga.device_status(ws) == 6
    sga.clear_device_status(ws)
    assert sga.device_status(ws) == 0
    idx = torch.full((B, 1, 2048), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, 5] = L + 10
    ws2 = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_SPARSE_MLA_ATTEND)
    sga.sparse_mla_attend(x["q"], x["kv"], idx, x["gate"], ws=ws2)
    assert sga.device_status(ws2) == 6


# ----------------------------------------------------------------------------- full-size workloads


def sampled_rows(wl, count):
    rows = wl.batch * wl.n_q
    if rows <= count:
        return list(range(rows))
    rng = np.random.default_rng(0)
    pick = set(rng.choice(rows, count - 2, replace=False).tolist()) | {0, rows - 1}
    return sorted(pick)


@pytest.mark.parametrize("name,count", [("decode_b4_ctx8k", 4), ("decode_b64_ctx32k", 6), ("decode_b32_ctx128k", 4),
                                        ("prefill_t4096_ctx128k", 64), ("decode_b8_ctx256k_ties", 3)])
def test_workload_sampled_parity(name, count):
    wl = synth.WORKLOADS[name]
    x = synth.make_inputs(wl, device="cuda", seed=0)
    dims = sga.make_dims(wl.batch, wl.n_q, wl.ctx, wl.top_k)
    ws = sga.alloc_workspace(dims, sga.OP_FORWARD)
    idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    torch.cuda.synchronize()
    check_status(ws)
    # invariants on every row: exactly min(t+1, K) ascending positions <= t, then -1
    idx_all = idx.reshape(-1, wl.top_k)
    pos_all = x["q_pos"].reshape(-1, 1)
    valid = idx_all >= 0
    n_expect = torch.clamp(pos_all[:, 0] + 1, max=wl.top_k)
    assert torch.equal(valid.sum(dim=1), n_expect)
    assert bool(((idx_all <= pos_all) | ~valid).all())
    d = idx_all[:, 1:] - idx_all[:, :-1]
    assert bool(((d > 0) | ~valid[:, 1:]).all())
    # sampled queries against the oracle, one sequence at a time
    rows = sampled_rows(wl, count)
    by_seq = {}
    for r in rows:
        by_seq.setdefault(r // wl.n_q, []).append(r % wl.n_q)
    for b, ts in by_seq.items():
        ts = torch.as_tensor(ts)
        sel = lambda t: t[b:b + 1, ts].contiguous().cpu()  # noqa: E731
        want_idx, want_out = oracle.forward(sel(x["q_idx"]), sel(x["w"]), x["k_idx"][b:b + 1].cpu(), sel(x["q"]),
                                            x["kv"][b:b + 1].cpu(), sel(x["gate"]), sel(x["q_pos"]))
        np.testing.assert_array_equal(idx[b, ts].cpu().numpy(), want_idx[0])
        assert_close(out[b, ts].cpu().numpy(), want_out[0], f"{name} seq {b}")


# ----------------------------------------------------------------------------- E4M3 indexer-key variant
# sga_index_scores_fp8 / sga_forward_fp8 read the indexer queries and keys as
# E4M3 codes; the oracle decodes each code to its exact value.


@pytest.mark.parametrize("B,T,L,pos", INDEX_CASES)
def test_index_scores_fp8_bit_exact(B, T, L, pos):
    x = gen_small(B, T, L, pos)
    qf, kf = synth.to_e4m3(x["q_idx"]), synth.to_e4m3(x["k_idx"])
    scores = torch.full((B, T, L), float("nan"), device="cuda")
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_INDEX_SCORES)
    sga.index_scores_fp8(qf, x["w"], kf, x["q_pos"], scores=scores, ws=ws)
    check_status(ws)
    want = oracle.index_scores_e4m3(qf, x["w"], kf, x["q_pos"].cpu())
    got = scores.cpu().numpy().astype(np.float64)
    pos = np.asarray(pos)
    for b in range(B):
        for t in range(T):
            p = pos[b, t]
            np.testing.assert_array_equal(got[b, t, : p + 1], want[b, t, : p + 1])


@pytest.mark.parametrize("B,T,L,pos", PREFILL_INDEX_CASES)
def test_index_scores_prefill_fp8_bit_exact(B, T, L, pos):
    x = gen_small(B, T, L, pos)
    qf, kf = synth.to_e4m3(x["q_idx"]), synth.to_e4m3(x["k_idx"])
    scores = torch.full((B, T, L), float("nan"), device="cuda")
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_INDEX_SCORES)
    sga.index_scores_fp8(qf, x["w"], kf, x["q_pos"], scores=scores, ws=ws)
    check_status(ws)
    want = oracle.index_scores_e4m3(qf, x["w"], kf, x["q_pos"].cpu())
    got = scores.cpu().numpy().astype(np.float64)
    pos = np.asarray(pos)
    for b in range(B):
        for t in range(T):
            p = pos[b, t]
            np.testing.assert_array_equal(got[b, t, : p + 1], want[b, t, : p + 1])


def test_index_scores_fp8_general_codes():
    """Random finite E4M3 codes (magnitudes 2^-9 .. 448, both signs): every
    product is exact in fp32, only the order of the fp32 sums differs."""
    B, T, L = 2, 2, 3000
    g = torch.Generator(device="cuda").manual_seed(3)
    codes = lambda shape: torch.randint(0, 0x7F, shape, generator=g, device="cuda", dtype=torch.int32)  # noqa: E731
    sign = lambda shape: torch.randint(0, 2, shape, generator=g, device="cuda", dtype=torch.int32) * 0x80  # noqa: E731
    qf = (codes((B, T, 64, 128)) | sign((B, T, 64, 128))).to(torch.uint8)
    kf = (codes((B, L, 128)) | sign((B, L, 128))).to(torch.uint8)
    w = torch.rand((B, T, 64), generator=g, device="cuda").to(torch.bfloat16)
    q_pos = torch.tensor([[L - 1, 1000], [2999, 17]], dtype=torch.int32, device="cuda")
    scores = sga.index_scores_fp8(qf, w, kf, q_pos)
    want = oracle.index_scores_e4m3(qf, w, kf, q_pos.cpu())
    got = scores.cpu().numpy().astype(np.float64)
    for b in range(B):
        for t in range(T):
            p = int(q_pos[b, t])
            err = np.abs(got[b, t, : p + 1] - want[b, t, : p + 1])
            assert err.max() <= 1e-5 * max(np.abs(want[b, t, : p + 1]).max(), 1.0)


@pytest.mark.parametrize("B,T,L,pos", [(2, 1, 1500, [[1499], [700]]), (2, 2, 6000, [[5999, 3000], [2500, 2047]])])
def test_forward_fp8_matches_oracle(B, T, L, pos):
    x = gen_small(B, T, L, pos)
    qf, kf = synth.to_e4m3(x["q_idx"]), synth.to_e4m3(x["k_idx"])
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_FORWARD)
    idx, out = sga.forward_fp8(qf, x["w"], kf, x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    check_status(ws)
    want_idx, want_out = oracle.forward_e4m3(qf, x["w"], kf, x["q"], x["kv"], x["gate"], x["q_pos"].cpu())
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    assert_close(out.cpu().numpy(), want_out, "forward fp8")


def test_workload_fp8_sampled_parity():
    """The 128K decode workload with an E4M3 indexer-key cache, as the bench runs it."""
    wl = synth.WORKLOADS["decode_b32_ctx128k"]
    x = synth.make_inputs_fp8(wl, device="cuda", seed=0)
    ws = sga.alloc_workspace(sga.make_dims(wl.batch, wl.n_q, wl.ctx, wl.top_k), sga.OP_FORWARD)
    idx, out = sga.forward_fp8(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    torch.cuda.synchronize()
    check_status(ws)
    for b in sampled_rows(wl, 3):
        sel = lambda t: t[b:b + 1].contiguous().cpu()  # noqa: E731
        want_idx, want_out = oracle.forward_e4m3(sel(x["q_idx"]), sel(x["w"]), sel(x["k_idx"]), sel(x["q"]),
                                                 sel(x["kv"]), sel(x["gate"]), sel(x["q_pos"]))
        np.testing.assert_array_equal(idx[b].cpu().numpy(), want_idx[0])
        assert_close(out[b].cpu().numpy(), want_out[0], f"fp8 workload seq {b}")
