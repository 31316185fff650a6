"""fp64 oracle of one SGA attention layer: the projections either side of the hot path.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's CPU
baseline leg call this module; the product path never does, and the two share
no code.  Plain numpy in double precision; the hot path in the middle is the
C++ oracle of this package (``oracle.forward``).

The layer, in the terms of the archdb "A.X K2" attention fields (64 heads; qk
head dim 192 = 128 nope + 64 rope; v head dim 128; KV latent 512; q low-rank
width 1536; a 64-dim decoupled RoPE key shared across heads; RoPE base 1e6; no
per-head QK norm; no projection bias), its gate field (a head-specific sigmoid
gate on the attention output before o_proj, projected jointly with the query)
and its token-selection field (a DSA-style indexer with 64 heads of dim 128):

    c_q                  = W_DQ h                  query latent (width R = 1536)
    [q_h^nope, q_h^rope] = W_UQ,h c_q              per head 128 + 64
    g                    = W_G c_q                 one gate logit per head
    [c_kv, k^rope]       = W_DKV h                 the 576-wide cache row
    q^rope, k^rope       <- RoPE at the token's position (base 1e6)
    q_h^lat              = W_UK,h^T q_h^nope       W_UK absorbed into the query:
                           q_h^nope . (W_UK,h c_kv) = q_h^lat . c_kv
    q_idx = W_IQ c_q,  k_idx = W_IK h,  w = W_IW h indexer projections
    (the new tokens' cache rows are written at their positions)
    idx, out_h           = sga_forward(...)        indexer, top-2048, latent
                                                   attention, sigmoid gate
    o_h                  = W_UV,h out_h            value head dim 128
    y                    = W_O [o_1; ...; o_64]    o_proj

Readings where the pages are silent:
* no norm on the query or KV latents (the pages list none for these layers);
* RoPE rotates interleaved pairs (2i, 2i+1) by p * base^(-i/32), i < 32, the
  form of the original rotary-embedding paper; no YaRN factor (none is given);
* the indexer query is projected from the query latent c_q, the indexer key
  and the head weights from h, with no RoPE, norm or scale (as DSA-style
  indexers project them; the pages name only the head count and width);
* every activation between two contractions is rounded to bf16 (round to
  nearest, ties to even), the precision of the cached KV and indexer-key rows;
  the contractions themselves are exact fp64, and y is returned unrounded.

Weights are passed in one packed layout (row-major, torch Linear convention
``out = W @ in``), which this module only slices into the named matrices:

    w_hq [R + 576 + 128 + 64, D]    rows: W_DQ | W_DKV | W_IK | W_IW
    w_cq [64*192 + 64 + 64*128, R]  rows: W_UQ (head h: rows 192 h .. 192 h + 191,
                                    nope first) | W_G | W_IQ (head j: rows 128 j ..)
    w_uk [64, 128, 512]             k_h^nope = w_uk[h] @ c_kv
    w_uv [64, 128, 512]             o_h = w_uv[h] @ out_h
    w_o  [D, 64*128]
"""
from __future__ import annotations

import numpy as np

from . import forward as _path_forward

HEADS = 64
NOPE = 128
ROPE = 64
LATENT = 512
KV_DIM = LATENT + ROPE  # 576
V_HEAD = 128
INDEX_HEADS = 64
INDEX_DIM = 128
ROPE_BASE = 1.0e6
Q_ROWS = HEADS * (NOPE + ROPE)  # 12,288
CQ_ROWS = Q_ROWS + HEADS + INDEX_HEADS * INDEX_DIM  # 20,544
HQ_EXTRA = KV_DIM + INDEX_DIM + INDEX_HEADS  # rows of w_hq after W_DQ: 768


def to_f64(a) -> np.ndarray:
    """bf16 torch tensor (or uint16 bit patterns) -> float64 values."""
    if hasattr(a, "detach"):
        import torch

        a = a.detach().cpu()
        if a.dtype == torch.bfloat16:
            a = a.view(torch.int16).numpy().view(np.uint16)
        else:
            return a.numpy().astype(np.float64)
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (8 significant bits), ties to even, from
    the definition: x = m 2^e with 0.5 <= |m| < 1, keep m to 2^-8.  Values here
    stay far inside bf16's normal range, so neither overflow nor subnormals arise."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)  # np.round: half to even


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16-representable float64 values -> their uint16 bit patterns (exact)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def rope(x: np.ndarray, pos: np.ndarray, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate interleaved pairs of the last axis (64 dims) by pos * base^(-i/32).
    x [..., 64]; pos broadcasts against x[..., 0]."""
    d = x.shape[-1]
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x, dtype=np.float64)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def split_weights(wts: dict) -> dict:
    """The named matrices of the packed layout (views, no arithmetic)."""
    w_hq, w_cq = to_f64(wts["w_hq"]), to_f64(wts["w_cq"])
    R = w_hq.shape[0] - HQ_EXTRA
    assert w_cq.shape == (CQ_ROWS, R), w_cq.shape
    o = R
    return {
        "W_DQ": w_hq[:R], "W_DKV": w_hq[o:o + KV_DIM], "W_IK": w_hq[o + KV_DIM:o + KV_DIM + INDEX_DIM],
        "W_IW": w_hq[o + KV_DIM + INDEX_DIM:],
        "W_UQ": w_cq[:Q_ROWS].reshape(HEADS, NOPE + ROPE, R), "W_G": w_cq[Q_ROWS:Q_ROWS + HEADS],
        "W_IQ": w_cq[Q_ROWS + HEADS:].reshape(INDEX_HEADS, INDEX_DIM, R),
        "W_UK": to_f64(wts["w_uk"]), "W_UV": to_f64(wts["w_uv"]), "W_O": to_f64(wts["w_o"]),
    }


def project(h, q_pos, wts: dict, rounding: bool = True) -> dict:
    """The projections in front of the path for tokens h [B,T,D] at positions q_pos [B,T].

    Returns float64 arrays (bf16 values when ``rounding``): c_q [B,T,R], kv_row
    [B,T,576] (c_kv, rotated k^rope), k_idx_row [B,T,128], w [B,T,64], q [B,T,64,576]
    (q^lat, rotated q^rope), gate [B,T,64], q_idx [B,T,64,128]."""
    rb = round_bf16 if rounding else (lambda v: v)
    W = split_weights(wts)
    H = to_f64(h)
    pos = np.asarray(q_pos.cpu() if hasattr(q_pos, "cpu") else q_pos, dtype=np.int64)
    c_q = rb(H @ W["W_DQ"].T)
    kv_pre = H @ W["W_DKV"].T
    c_kv = rb(kv_pre[..., :LATENT])
    k_rope = rb(rope(rb(kv_pre[..., LATENT:]), pos))
    k_idx_row = rb(H @ W["W_IK"].T)
    w = rb(H @ W["W_IW"].T)
    qh = np.einsum("btr,hdr->bthd", c_q, W["W_UQ"])
    q_nope = rb(qh[..., :NOPE])
    q_rope = rb(rope(rb(qh[..., NOPE:]), pos[..., None]))
    gate = rb(c_q @ W["W_G"].T)
    q_idx = rb(np.einsum("btr,jdr->btjd", c_q, W["W_IQ"]))
    q_lat = rb(np.einsum("bthd,hdj->bthj", q_nope, W["W_UK"]))
    return {"c_q": c_q, "kv_row": np.concatenate([c_kv, k_rope], axis=-1), "k_idx_row": k_idx_row, "w": w,
            "q": np.concatenate([q_lat, q_rope], axis=-1), "gate": gate, "q_idx": q_idx, "q_nope": q_nope}


def write_cache(cache, rows: np.ndarray, q_pos) -> np.ndarray:
    """A copy of cache [B,L,C] (float64 values) with rows [B,T,C] stored at their positions."""
    out = to_f64(cache).copy()
    pos = np.asarray(q_pos.cpu() if hasattr(q_pos, "cpu") else q_pos, dtype=np.int64)
    for b in range(pos.shape[0]):
        for t in range(pos.shape[1]):
            out[b, pos[b, t]] = rows[b, t]
    return out


def output_projection(out: np.ndarray, wts: dict, rounding: bool = True) -> np.ndarray:
    """o_h = W_UV,h out_h, y = W_O [o_1; ...; o_64] for out [B,T,64,512]; y [B,T,D] unrounded."""
    rb = round_bf16 if rounding else (lambda v: v)
    W = split_weights(wts)
    o = rb(np.einsum("bthj,hij->bthi", rb(out), W["W_UV"]))
    B, T = o.shape[:2]
    return o.reshape(B, T, HEADS * V_HEAD) @ W["W_O"].T


def layer_forward(h, q_pos, kv_cache, k_idx_cache, wts: dict, k: int = 2048, n_threads: int = 0) -> dict:
    """One SGA layer over new tokens h [B,T,D] (bf16) at positions q_pos [B,T].

    The new tokens' cache rows are written first (so a token attends to itself
    and to the earlier tokens of its chunk), then the hot path runs on the
    updated caches.  Returns idx [B,T,k], y [B,T,D] (float64), the updated
    caches kv [B,L,576] and k_idx [B,L,128] (float64 bf16 values) and the
    projected activations of ``project``."""
    p = project(h, q_pos, wts)
    kv = write_cache(kv_cache, p["kv_row"], q_pos)
    ki = write_cache(k_idx_cache, p["k_idx_row"], q_pos)
    pos = np.asarray(q_pos.cpu() if hasattr(q_pos, "cpu") else q_pos, dtype=np.int32)
    idx, out = _path_forward(bf16_bits(p["q_idx"]), bf16_bits(p["w"]), bf16_bits(ki), bf16_bits(p["q"]),
                             bf16_bits(kv), bf16_bits(p["gate"]), pos, k=k, n_threads=n_threads)
    y = output_projection(out, wts)
    return dict(p, idx=idx, y=y, kv=kv, k_idx=ki, out=out)
