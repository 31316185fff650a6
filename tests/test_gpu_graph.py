"""sga_forward and sga_layer_forward captured in a CUDA graph.

Every call is asynchronous, allocates nothing and does not synchronise, so once
the one-time set-up has run (the first call on the device), a call can be
captured into a CUDA graph and replayed: its launches become kernel nodes with
their programmatic dependencies.  A replay reads whatever the captured input
buffers hold at that moment, and the workspace's histograms and counters are
left zeroed by every call, so replays may repeat.  The results are checked
against the oracle, for the captured inputs and for new inputs copied into the
same buffers."""
import numpy as np
import pytest
import torch

import oracle
from oracle import layer as layer_oracle
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


def close(got, want, rel=1e-3, abs_=1e-2):
    err = got.astype(np.float64) - want
    return np.linalg.norm(err) / np.linalg.norm(want) <= rel and np.abs(err).max() <= abs_


def test_forward_replays_from_a_cuda_graph():
    wl = synth.custom(batch=3, n_q=1, ctx=9000, first_pos=8999)
    x = synth.make_inputs(wl, device="cuda", seed=30)
    ws = sga.alloc_workspace(sga.make_dims(wl.batch, 1, wl.ctx), sga.OP_FORWARD)
    idx = torch.empty((wl.batch, 1, wl.top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((wl.batch, 1, 64, 512), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()

    def call():
        sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], idx_out=idx, out=out,
                    ws=ws, stream=stream)

    with torch.cuda.stream(stream):
        call()  # the one-time set-up happens outside the capture
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call()
    for seed in (30, 31):
        if seed != 30:  # new inputs in the captured buffers
            for k, v in synth.make_inputs(wl, device="cuda", seed=seed).items():
                x[k].copy_(v)
        idx.fill_(-7)
        out.zero_()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        assert sga.device_status(ws) == 0
        want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"],
                                            x["q_pos"].cpu())
        np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
        assert close(out.cpu().numpy(), want_out)


def test_layer_forward_replays_from_a_cuda_graph():
    """One whole layer (GEMMs, prep kernels, the path, the output projections)
    at ctx <= 2048, where every causal position is selected, so the indices
    are exact; y within the layer's bound."""
    wts = synth.make_layer_weights(device="cuda", seed=0)
    wl = synth.custom(batch=2, n_q=2, ctx=1500, first_pos=1000)
    x = synth.make_inputs(wl, device="cuda", seed=32)
    h = torch.randn((2, 2, synth.D_MODEL), generator=torch.Generator(device="cuda").manual_seed(33),
                    device="cuda").to(torch.bfloat16)
    q_pos = torch.tensor([[1000, 1001], [1498, 1499]], dtype=torch.int32, device="cuda")
    kv_in, ki_in = x["kv"].clone(), x["k_idx"].clone()
    ws = sga.alloc_layer_workspace(sga.make_dims(2, 2, 1500), sga.layer_weights(wts))
    idx = torch.empty((2, 2, wl.top_k), dtype=torch.int32, device="cuda")
    y = torch.empty((2, 2, synth.D_MODEL), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()

    def call():
        sga.layer_forward(wts, h, q_pos, x["kv"], x["k_idx"], idx_out=idx, y=y, ws=ws, stream=stream)

    with torch.cuda.stream(stream):
        call()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call()
    x["kv"].copy_(kv_in)  # the layer writes its new tokens' cache rows in place: start from the inputs again
    x["k_idx"].copy_(ki_in)
    y.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert sga.device_status(ws) == 0
    want = layer_oracle.layer_forward(h, q_pos, kv_in, ki_in, wts)
    np.testing.assert_array_equal(idx.cpu().numpy(), want["idx"])
    err = y.cpu().numpy().astype(np.float64) - want["y"]
    assert np.linalg.norm(err) / np.linalg.norm(want["y"]) <= 1e-2
