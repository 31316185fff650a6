"""The top-k entry point that needs no caller workspace.

Some callers cannot allocate device memory, such as a custom operator inside
another inference engine that is handed only its input and output buffers.
sga_topk_select_noalloc serves them from a static scratch array inside the
library.  This file checks, through the C ABI, that it selects exactly what
sga_topk_select (with a caller workspace) and the fp64 oracle select, on two
different calls in a row, so the second call also shows that state left behind
by the first does not leak into its result.  Rows longer than 8 x 65,536
positions keep their selection and tie bitmaps in the scratch array itself
(shorter rows keep them in shared memory and use only its status word), so the
long cases exercise the array.  The file sits last in collection order so that
a failure here comes after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sparse_gated_attention_b200 as sga

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_gated_attention_b200 import build

    build.build()
    oracle.build()
    return sga.load_library()


def call_noalloc(lib, scores, q_pos, k):
    B, T, L = scores.shape
    idx = torch.full((B, T, k), -7, dtype=torch.int32, device=scores.device)
    dims = sga.make_dims(B, T, L, k)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.sga_topk_select_noalloc(ctypes.byref(dims), ctypes.c_void_p(scores.data_ptr()),
                                     ctypes.c_void_p(q_pos.data_ptr()), ctypes.c_void_p(idx.data_ptr()), stream)
    assert rc == 0, f"sga_topk_select_noalloc returned {rc}"
    return idx


def case(seed, B, L, hi, k=2048):
    g = torch.Generator(device="cuda").manual_seed(seed)
    scores = torch.randint(0, hi, (B, 1, L), generator=g, device="cuda", dtype=torch.int32).to(torch.float32)
    q_pos = torch.randint(k // 2, L, (B, 1), generator=g, device="cuda", dtype=torch.int32)
    q_pos[0, 0] = L - 1
    return scores, q_pos


def check_against_both(lib, scores, q_pos, k=2048):
    got = call_noalloc(lib, scores, q_pos, k)
    want = sga.topk_select(scores, q_pos, top_k=k)
    torch.cuda.synchronize()
    got_np = got.cpu().numpy()
    np.testing.assert_array_equal(got_np, want.cpu().numpy())
    B, T, L = scores.shape
    ref = oracle.topk(scores.cpu().numpy().astype(np.float64).reshape(B * T, L),
                      q_pos.cpu().numpy().reshape(B * T), k=k)
    np.testing.assert_array_equal(got_np.reshape(B * T, k), ref)


def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    for seed, B, L, hi in [(1, 12, 100000, 40), (2, 5, 131072, 5000)]:
        scores, q_pos = case(seed, B, L, hi)
        check_against_both(lib, scores, q_pos)


@pytest.mark.parametrize("L", [600004, 600001])
def test_noalloc_bitmaps_in_the_scratch_array_on_two_calls(lib, L):
    """Two rows of ~600K positions: 2 x 2 x 18,751 words x 4 B = 300 KB of
    bitmaps in the library's array.  The second call (other seed, other
    positions) reuses the words the first one left behind."""
    for seed, hi in [(11, 9), (12, 3000)]:
        scores, q_pos = case(seed, 2, L, hi)
        q_pos[1, 0] = L - 2 - seed  # both rows long enough for the array
        check_against_both(lib, scores, q_pos)


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # 40 rows x 2 bitmaps x (262144 / 32) words x 4 B = 2.6 MB fits; 100 rows do not.
    dims = sga.make_dims(100, 1, 262144, 2048)
    P = ctypes.c_void_p
    assert lib.sga_topk_select_noalloc(ctypes.byref(dims), P(0x100000), P(0x100000), P(0x100000), None) == 3
