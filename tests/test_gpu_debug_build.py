"""The SGA_DEBUG build on the GPU: libsga_debug.so (the same kernels with their
device-side invariant checks compiled in: gathered rows inside their sequence,
emitted slots and positions inside their row, the selection's candidate list
within its capacity, GEMM work items inside their tensors, prefill query blocks
inside their sequence) runs a forward, a prefill-shaped forward, the fused
selection with bf16 and E4M3 keys, the indexer's warm-up objective, a long-row
top-k and a layer forward in a process of its own.  Every check must hold
(the workspace status stays SGA_OK) and the results must match the oracle as
the release build's do."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import sys
sys.path.insert(0, ROOT)
import numpy as np
import torch
import oracle
import sparse_gated_attention_b200 as sga
from sparse_gated_attention_b200 import synth
from oracle import layer as layer_oracle

lib = sga.load_library()
assert lib._name.endswith("libsga_debug.so"), lib._name
oracle.build()

def close(got, want):
    err = np.asarray(got, np.float64) - want
    return np.linalg.norm(err) / np.linalg.norm(want) <= 1e-3 and np.abs(err).max() <= 1e-2

# decode forward and a prefill-shaped forward (12 queries per sequence)
for B, T, L, seed in [(3, 1, 9000, 0), (2, 12, 6000, 1)]:
    wl = synth.custom(batch=B, n_q=T, ctx=L, first_pos=L - T)
    x = synth.make_inputs(wl, device="cuda", seed=seed)
    ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_FORWARD)
    idx, out = sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    assert sga.device_status(ws) == 0, ("forward", B, T, sga.device_status(ws))
    want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"].cpu())
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    assert close(out.cpu().numpy(), want_out)

# the fused selection (candidate lists within their capacity), bf16 and E4M3 keys, on the decode case
B, T, L = 3, 1, 9000
wl = synth.custom(batch=B, n_q=T, ctx=L, first_pos=L - T)
x = synth.make_inputs(wl, device="cuda", seed=0)
want_idx, want_out = oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"].cpu())
ws = sga.alloc_workspace(sga.make_dims(B, T, L), sga.OP_FORWARD_FUSED)
for fp8 in (False, True):
    qi, ki = (synth.to_e4m3(x["q_idx"]), synth.to_e4m3(x["k_idx"])) if fp8 else (x["q_idx"], x["k_idx"])
    call = sga.forward_fused_fp8 if fp8 else sga.forward_fused
    idx, out = call(qi, x["w"], ki, x["q"], x["kv"], x["gate"], x["q_pos"], ws=ws)
    assert sga.device_status(ws) == 0, ("fused", fp8, sga.device_status(ws))
    assert np.array_equal(idx.cpu().numpy(), want_idx), ("fused", fp8)  # integer inputs: E4M3 codes are exact
    assert close(out.cpu().numpy(), want_out), ("fused", fp8)

# the indexer's warm-up objective over the oracle's selection
from oracle import warmup as warmup_oracle
want = warmup_oracle.warmup_loss(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["q_pos"].cpu())
wws = torch.zeros(sga.indexer_warmup_workspace_size(sga.make_dims(B, T, L)), dtype=torch.uint8, device="cuda")
got = sga.indexer_warmup(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], torch.as_tensor(want["idx"], device="cuda"),
                         ws=wws)
assert sga.device_status(wws) == 0
assert np.allclose(got["loss"].cpu().numpy(), want["per_query"], rtol=1e-4, atol=0)
for k in ("grad_q_idx", "grad_w", "grad_k_idx"):
    g_ = got[k].cpu().numpy().astype(np.float64)
    assert np.linalg.norm(g_ - want[k]) <= 1e-3 * np.linalg.norm(want[k]), k

# a long row: the streaming top-k with its words in the workspace
g = torch.Generator(device="cuda").manual_seed(2)
L = 600004
sc = torch.randint(0, 3000, (2, 1, L), generator=g, device="cuda", dtype=torch.int32).to(torch.float32)
qp = torch.tensor([[L - 1], [L - 2]], dtype=torch.int32, device="cuda")
ws = sga.alloc_workspace(sga.make_dims(2, 1, L), sga.OP_TOPK_SELECT)
idx = sga.topk_select(sc, qp, ws=ws)
assert sga.device_status(ws) == 0
want = oracle.topk(sc.cpu().numpy().astype(np.float64).reshape(2, L), qp.cpu().numpy().reshape(2))
assert np.array_equal(idx.cpu().numpy().reshape(2, -1), want)

# one layer (its GEMMs) at ctx <= 2048, where every causal position is selected
wts = synth.make_layer_weights(device="cuda", seed=0)
wl = synth.custom(batch=2, n_q=2, ctx=1500, first_pos=1000)
x = synth.make_inputs(wl, device="cuda", seed=3)
h = torch.randn((2, 2, synth.D_MODEL), generator=torch.Generator(device="cuda").manual_seed(4),
                device="cuda").to(torch.bfloat16)
q_pos = torch.tensor([[1000, 1001], [1498, 1499]], dtype=torch.int32, device="cuda")
kv_in, ki_in = x["kv"].clone(), x["k_idx"].clone()
ws = sga.alloc_layer_workspace(sga.make_dims(2, 2, 1500), sga.layer_weights(wts))
idx, y = sga.layer_forward(wts, h, q_pos, x["kv"], x["k_idx"], ws=ws)
assert sga.device_status(ws) == 0
want = layer_oracle.layer_forward(h, q_pos, kv_in, ki_in, wts)
assert np.array_equal(idx.cpu().numpy(), want["idx"])
err = y.cpu().numpy().astype(np.float64) - want["y"]
assert np.linalg.norm(err) / np.linalg.norm(want["y"]) <= 1e-2
print("debug build ok")
'''


def test_debug_build_runs_clean_and_matches_the_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_gated_attention_b200 import build

    build.build(debug=True)
    env = dict(os.environ, SGA_LIBRARY="debug")
    res = subprocess.run([sys.executable, "-c", SCRIPT.replace("ROOT", repr(ROOT))], env=env, capture_output=True,
                         text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    assert "debug build ok" in res.stdout
