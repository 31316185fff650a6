"""Concurrent calls on distinct workspaces.

The ABI allows calls on distinct workspaces from several host threads and
streams at once.  Two threads, each with its own stream, workspace and inputs,
run sga_forward twenty times while the other does the same, so their kernels
(persistent indexers, cluster top-k and attention) share the GPU.  Every
result must equal the oracle's (indices bit-exact, outputs within the path's
tolerance) and repeat bit for bit from call to call."""
import threading

import numpy as np
import pytest
import torch

import oracle
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


def test_forward_from_two_threads_on_two_streams():
    cases = [synth.custom(batch=3, n_q=1, ctx=9000, first_pos=8999),
             synth.custom(batch=2, n_q=1, ctx=20000, first_pos=19999)]
    xs = [synth.make_inputs(wl, device="cuda", seed=20 + i) for i, wl in enumerate(cases)]
    wants = [oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"].cpu())
             for x in xs]
    results = [[] for _ in cases]
    errors = []
    start = threading.Barrier(len(cases))

    def worker(i):
        try:
            wl, x = cases[i], xs[i]
            stream = torch.cuda.Stream()
            ws = sga.alloc_workspace(sga.make_dims(wl.batch, 1, wl.ctx), sga.OP_FORWARD)
            torch.cuda.synchronize()
            start.wait()
            outs = []
            with torch.cuda.stream(stream):
                for _ in range(20):
                    outs.append(sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"],
                                            ws=ws, stream=stream))
            stream.synchronize()
            if sga.device_status(ws, stream) != 0:
                errors.append((i, "device status"))
            results[i] = [(idx.cpu().numpy(), out.cpu().numpy()) for idx, out in outs]
        except Exception as exc:  # reported below, with the thread's index
            errors.append((i, repr(exc)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for i, (want_idx, want_out) in enumerate(wants):
        assert len(results[i]) == 20
        idx0, out0 = results[i][0]
        np.testing.assert_array_equal(idx0, want_idx)
        err = out0.astype(np.float64) - want_out
        assert np.linalg.norm(err) / np.linalg.norm(want_out) <= 1e-3 and np.abs(err).max() <= 1e-2
        for idx, out in results[i][1:]:
            assert np.array_equal(idx, idx0) and np.array_equal(out, out0)
