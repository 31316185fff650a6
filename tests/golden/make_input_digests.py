"""Writes input_digests.json: sha256 of every tensor the seeded input recipe
draws on the CPU for the tiny decode workload (batch 4 at 8K context, seed 0),
the same inputs with E4M3 indexer keys, and a small layer case.  The digests
pin the recipe's bytes (generator, distributions and drawing order), so a
change in any of them shows up in tests/test_input_digests.py.  Only the input
generator is called here; no expected output is stored.

    python tests/golden/make_input_digests.py
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import torch  # noqa: E402

from sparse_gated_attention_b200 import synth  # noqa: E402


def digest(t: torch.Tensor) -> str:
    t = t.detach().cpu().contiguous()
    raw = t.view(torch.uint8) if t.dtype in (torch.bfloat16, torch.float8_e4m3fn) else t
    return hashlib.sha256(raw.numpy().tobytes()).hexdigest()


def cases() -> dict:
    out = {}
    wl = synth.WORKLOADS["decode_b4_ctx8k"]
    out["decode_b4_ctx8k"] = {k: digest(v) for k, v in synth.make_inputs(wl, device="cpu", seed=0).items()}
    out["decode_b4_ctx8k_fp8"] = {k: digest(v) for k, v in synth.make_inputs_fp8(wl, device="cpu", seed=0).items()
                                  if k in ("q_idx", "k_idx")}
    lw = synth.custom(batch=2, n_q=2, ctx=300, first_pos=150, name="layer_small")
    x = synth.make_layer_inputs(lw, d_model=256, q_rank=96, device="cpu", seed=3)
    out["layer_small"] = {"h": digest(x["h"]), **{k: digest(v) for k, v in x["weights"].items()}}
    return out


if __name__ == "__main__":
    data = {"torch": torch.__version__, "device": "cpu", "digests": cases()}
    with open(os.path.join(HERE, "input_digests.json"), "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
    print("wrote", os.path.join(HERE, "input_digests.json"))
