"""Seeded synthetic workloads for the SGA hot path.

This module draws random inputs and nothing else: it holds none of the method's
arithmetic.  Both the CUDA path and the fp64 oracle consume the tensors it
returns (the oracle gets a host copy of the same bytes).

Recipe (one ``torch.Generator`` seeded with ``seed`` on the target device; the
tensors are drawn in the order listed, one sequence ``b`` at a time so that peak
memory stays at one sequence's worth of fp32 temporaries):

* ``q_idx``  [B,T,64,128]  integers uniform in [-3, 3], stored bf16 (exact)
* ``w``      [B,T,64]      integers uniform in [0, 3], stored bf16
* ``k_idx``  [B,L,128]     integers uniform in [-r, r] (r = 3, or 1 for the tie
                           stress workload), stored bf16
* ``q``      [B,T,64,576]  N(0,1) rounded to bf16 (round to nearest even)
* ``kv``     [B,L,576]     N(0,1) rounded to bf16
* ``gate``   [B,T,64]      N(0,1) rounded to bf16
* ``q_pos``  [B,T] int32   decode: L-1 (one query at the last position);
                           chunked prefill: first_pos .. first_pos+T-1

One SGA layer around the path (``make_layer_inputs``) adds, from a second
generator seeded with ``seed + LAYER_SEED_OFFSET`` and drawn in this order:

* ``h``      [B,T,D]       the new tokens' hidden states, N(0,1) rounded to bf16
* the packed projection weights (the layout of ``sga_layer_weights_t``), each
  N(0,1) / sqrt(fan_in) rounded to bf16 so activations stay O(1):
  ``w_hq`` [R+768, D] (fan_in D), ``w_cq`` [20544, R] (fan_in R),
  ``w_uk`` [64,128,512] and ``w_uv`` [64,128,512] (fan_in 512), ``w_o`` [D, 8192]
  (fan_in 8192); D = 7168 and R = 1536 are the archdb "A.X K2" residual width
  and q low-rank width.
The caches (``kv``, ``k_idx``) and ``q_pos`` are those of ``make_inputs``; the
layer overwrites the rows at ``q_pos`` with the new tokens' projected rows.

Integer indexer inputs make every indexer score an exact integer in fp32, so
the selected positions can be compared bit for bit.  The shapes follow the
indexer and attention fields of the archdb "A.X K2" page (64 indexer heads of
dim 128; 64 heads over a 512 + 64 latent).  CUDA and CPU generators give
different streams for the same seed; a workload is identified by (name, seed,
device type).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

INDEX_HEADS = 64
INDEX_DIM = 128
HEADS = 64
QK_DIM = 576
V_DIM = 512
TOP_K = 2048


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int
    ctx: int  # L: cache rows per sequence
    first_pos: int  # position of the first query of each sequence
    k_range: int = 3  # k_idx drawn from [-k_range, k_range]
    top_k: int = TOP_K

    @property
    def decode(self) -> bool:
        return self.n_q == 1


WORKLOADS = {
    w.name: w
    for w in [
        Workload("decode_b4_ctx8k", batch=4, n_q=1, ctx=8192, first_pos=8191),
        Workload("decode_b64_ctx32k", batch=64, n_q=1, ctx=32768, first_pos=32767),
        Workload("decode_b32_ctx128k", batch=32, n_q=1, ctx=131072, first_pos=131071),
        Workload("prefill_t4096_ctx128k", batch=1, n_q=4096, ctx=131072, first_pos=126976),
        Workload("decode_b8_ctx256k_ties", batch=8, n_q=1, ctx=262144, first_pos=262143, k_range=1),
    ]
}

HEADLINE = "decode_b32_ctx128k"


def custom(batch: int, n_q: int, ctx: int, first_pos: int | None = None, k_range: int = 3,
           top_k: int = TOP_K, name: str = "custom") -> Workload:
    if first_pos is None:
        first_pos = ctx - n_q
    return Workload(name, batch, n_q, ctx, first_pos, k_range, top_k)


def _ints(g, lo, hi, shape, device):
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.int32).to(torch.bfloat16)


def _normal(g, shape, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(wl: Workload, device="cpu", seed: int = 0) -> dict:
    """Draw every input of ``wl`` on ``device`` (see the module docstring)."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    B, T, L = wl.batch, wl.n_q, wl.ctx
    if wl.first_pos < 0 or wl.first_pos + T > L:
        raise ValueError("query positions must lie inside the cache")
    q_idx = torch.empty((B, T, INDEX_HEADS, INDEX_DIM), dtype=torch.bfloat16, device=device)
    w = torch.empty((B, T, INDEX_HEADS), dtype=torch.bfloat16, device=device)
    k_idx = torch.empty((B, L, INDEX_DIM), dtype=torch.bfloat16, device=device)
    q = torch.empty((B, T, HEADS, QK_DIM), dtype=torch.bfloat16, device=device)
    kv = torch.empty((B, L, QK_DIM), dtype=torch.bfloat16, device=device)
    gate = torch.empty((B, T, HEADS), dtype=torch.bfloat16, device=device)
    for b in range(B):
        q_idx[b] = _ints(g, -3, 3, (T, INDEX_HEADS, INDEX_DIM), device)
    for b in range(B):
        w[b] = _ints(g, 0, 3, (T, INDEX_HEADS), device)
    for b in range(B):
        k_idx[b] = _ints(g, -wl.k_range, wl.k_range, (L, INDEX_DIM), device)
    for b in range(B):
        q[b] = _normal(g, (T, HEADS, QK_DIM), device)
    for b in range(B):
        kv[b] = _normal(g, (L, QK_DIM), device)
    for b in range(B):
        gate[b] = _normal(g, (T, HEADS), device)
    pos = torch.arange(wl.first_pos, wl.first_pos + T, dtype=torch.int32, device=device)
    q_pos = pos.unsqueeze(0).expand(B, T).contiguous()
    return dict(q_idx=q_idx, w=w, k_idx=k_idx, q=q, kv=kv, gate=gate, q_pos=q_pos)


def to_e4m3(x: torch.Tensor) -> torch.Tensor:
    """bf16 tensor -> float8_e4m3fn storage (exact for the integer-valued indexer inputs)."""
    return x.to(torch.float8_e4m3fn)


def make_inputs_fp8(wl: Workload, device="cpu", seed: int = 0) -> dict:
    """The inputs of ``make_inputs`` with the indexer queries and keys stored as E4M3
    (the FP8 indexer-key cache variant); the integer values in [-3, 3] are kept exactly."""
    x = make_inputs(wl, device, seed)
    x["q_idx"] = to_e4m3(x["q_idx"])
    x["k_idx"] = to_e4m3(x["k_idx"])
    return x


def input_bytes(wl: Workload) -> dict:
    """Bytes of each input tensor (for reporting)."""
    B, T, L = wl.batch, wl.n_q, wl.ctx
    return dict(q_idx=B * T * INDEX_HEADS * INDEX_DIM * 2, w=B * T * INDEX_HEADS * 2, k_idx=B * L * INDEX_DIM * 2,
                q=B * T * HEADS * QK_DIM * 2, kv=B * L * QK_DIM * 2, gate=B * T * HEADS * 2, q_pos=B * T * 4)


D_MODEL = 7168
Q_RANK = 1536
LAYER_SEED_OFFSET = 0x5EED
HQ_EXTRA = QK_DIM + INDEX_DIM + INDEX_HEADS  # rows of w_hq after W_DQ
CQ_ROWS = HEADS * 192 + HEADS + INDEX_HEADS * INDEX_DIM


def _scaled(g, shape, fan_in, device):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * fan_in ** -0.5).to(torch.bfloat16)


def make_layer_weights(d_model: int = D_MODEL, q_rank: int = Q_RANK, device="cpu", seed: int = 0) -> dict:
    """Packed bf16 projection weights of one layer (see the module docstring)."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed + LAYER_SEED_OFFSET)
    return {
        "w_hq": _scaled(g, (q_rank + HQ_EXTRA, d_model), d_model, device),
        "w_cq": _scaled(g, (CQ_ROWS, q_rank), q_rank, device),
        "w_uk": _scaled(g, (HEADS, 128, V_DIM), V_DIM, device),
        "w_uv": _scaled(g, (HEADS, 128, V_DIM), V_DIM, device),
        "w_o": _scaled(g, (d_model, HEADS * 128), HEADS * 128, device),
    }


def make_layer_inputs(wl: Workload, d_model: int = D_MODEL, q_rank: int = Q_RANK, device="cpu",
                      seed: int = 0) -> dict:
    """The workload's caches and positions, the new tokens' hidden states h and
    the layer's packed weights (see the module docstring)."""
    x = make_inputs(wl, device, seed)
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed + 2 * LAYER_SEED_OFFSET)
    h = torch.randn((wl.batch, wl.n_q, d_model), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return {"h": h, "q_pos": x["q_pos"], "kv": x["kv"], "k_idx": x["k_idx"],
            "weights": make_layer_weights(d_model, q_rank, device, seed)}
