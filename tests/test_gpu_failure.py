"""The device-side failure path of the kernels, on the GPU, without a fault.

Every wait inside the path's kernels gives up after a cycle budget, records
SGA_ERR_TIMEOUT in the workspace status word, raises its CTA's abort flag (which
releases the CTA's other waits) and unwinds: tensor memory freed, kernel
returned, CUDA context usable.  sga_selftest_bounded_wait runs that sequence on
a barrier that nothing completes: one wait with a budget of a few thousand
cycles, a second with the kernels' own budget (about one second), released by
the abort flag.  Nothing faults, traps or hangs.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gated_attention_b200 as sga

pytestmark = pytest.mark.gpu
SGA_ERR_TIMEOUT = 5


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_gated_attention_b200 import build

    build.build()
    sga.load_library()
    oracle.build()


def test_bounded_wait_gives_up_reports_timeout_and_unwinds():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    sga.selftest_bounded_wait(1000, ws)  # first launch: module load outside the timed call
    torch.cuda.synchronize()
    ws.zero_()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    sga.selftest_bounded_wait(20000, ws)
    stop.record()
    torch.cuda.synchronize()
    words = ws.view(torch.int32).cpu().numpy()
    assert words[0] == SGA_ERR_TIMEOUT
    assert words[1] == 2, "both waits gave up (the second through the abort flag)"
    assert sga.device_status(ws) == SGA_ERR_TIMEOUT
    # the second wait's own budget is ~1 s: it ended because the first raised the flag
    assert start.elapsed_time(stop) < 200.0


def test_context_usable_after_a_timeout():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    sga.selftest_bounded_wait(5000, ws)
    torch.cuda.synchronize()
    assert sga.device_status(ws) == SGA_ERR_TIMEOUT
    sga.clear_device_status(ws)
    assert sga.device_status(ws) == 0
    g = torch.Generator(device="cuda").manual_seed(1)
    B, L = 2, 3000
    q_idx = torch.randint(-3, 4, (B, 1, 64, 128), generator=g, device="cuda", dtype=torch.int32).to(torch.bfloat16)
    w = torch.randint(0, 4, (B, 1, 64), generator=g, device="cuda", dtype=torch.int32).to(torch.bfloat16)
    k_idx = torch.randint(-3, 4, (B, L, 128), generator=g, device="cuda", dtype=torch.int32).to(torch.bfloat16)
    q = torch.randn((B, 1, 64, 576), generator=g, device="cuda").to(torch.bfloat16)
    kv = torch.randn((B, L, 576), generator=g, device="cuda").to(torch.bfloat16)
    gate = torch.randn((B, 1, 64), generator=g, device="cuda").to(torch.bfloat16)
    q_pos = torch.tensor([[L - 1], [2500]], dtype=torch.int32, device="cuda")
    fws = sga.alloc_workspace(sga.make_dims(B, 1, L), sga.OP_FORWARD)
    idx, out = sga.forward(q_idx, w, k_idx, q, kv, gate, q_pos, ws=fws)
    assert sga.device_status(fws) == 0
    want_idx, want_out = oracle.forward(q_idx, w, k_idx, q, kv, gate, q_pos.cpu())
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    err = out.cpu().numpy().astype(np.float64) - want_out
    assert np.linalg.norm(err) / np.linalg.norm(want_out) <= 1e-3 and np.abs(err).max() <= 1e-2
