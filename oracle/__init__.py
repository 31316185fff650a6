"""fp64 CPU oracle for the Sparse Gated Attention (SGA) hot path.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's CPU
baseline leg call this package; the product path (the CUDA library and its
Python binding) never does, and the two share no code.

The arithmetic lives in ``sga_oracle.cpp`` (plain C++17, double precision,
std::thread over independent queries).  This module only compiles it with g++
and marshals numpy arrays through ctypes.  bf16 inputs are passed as their raw
uint16 bit patterns.

Each function follows one step of the method:

* ``index_scores`` - the DSA-style indexer (archdb "A.X K2", token-selection
  field: 64 indexer heads of dim 128, ReLU-scored; indexer-key-width field: 128).
* ``topk`` - top-2048 selection per query (same field; arXiv abstract "A.X K2
  Technical Report": each query reads only 2,048 positions), ties to the lower
  position, output ascending and padded with -1.
* ``attend`` - MLA attention in latent form over the selected rows (archdb
  "A.X K2" attention fields: 64 heads, qk head dim 192, latent 512 + rope 64)
  followed by the head-specific sigmoid output gate (archdb "A.X K2" gate field).
* ``forward`` - the three in sequence.
* ``e4m3_to_float64`` / ``index_scores_e4m3`` / ``forward_e4m3`` - the same
  path with an FP8 (E4M3) indexer-key cache (archdb "A.X K2": E4M3 matmuls in
  its pretraining-precision field; nlp.com.ai "A.X K2 FP8"), reading each
  E4M3 code as its exact value with no block scale.  Every finite E4M3 value is
  a bf16 value, so the codes are converted exactly and the bf16 oracle runs
  unchanged.

Two modules build on these steps in plain numpy fp64:

* ``oracle.layer`` - one SGA attention layer: the projections either side of
  the path (q low-rank path, decoupled RoPE, the gate projected with the query,
  W_UK absorption, the cache update, W_UV and o_proj; archdb "A.X K2"
  attention and gate fields).
* ``oracle.warmup`` - the indexer's sparse warm-up objective (a KL divergence
  from the frozen attention's distribution over the indexer's own top-k) and
  its gradients (arXiv abstract "A.X K2 Technical Report": the indexer is
  optimised against its own sparse top-k selection).

Pins: every function is checked against closed forms, invariants, a
hand-worked fixture and library routines (numpy matmul, torch SDPA and softmax
in fp64, torch's bf16 conversion, Python's sort, finite differences), not
against itself: ``tests/test_oracle_pins.py``, ``tests/test_layer_oracle.py``
and ``tests/test_warmup_oracle.py``, with planted mistakes in the
``*_mutants.py`` tests.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sga_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

# Model constants of the method (archdb "A.X K2" attention and indexer fields).
INDEX_HEADS = 64
INDEX_DIM = 128
HEADS = 64
QK_DIM = 576  # 512 latent + 64 rope, absorbed form
V_DIM = 512
TOP_K = 2048
SCALE = 192.0 ** -0.5  # qk head dim 192 = 128 nope + 64 rope


def build(force: bool = False) -> str:
    """Compile the oracle into ``liboracle.so`` next to its source."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        d = ctypes.c_double
        lib.oracle_index_scores.argtypes = [i, i, i, i, i, P, P, P, P, P, i]
        lib.oracle_topk.argtypes = [i, i, P, P, i, P, i]
        lib.oracle_attend.argtypes = [i, i, i, i, i, i, d, P, P, P, i, P, P, i]
        lib.oracle_forward.argtypes = [i, i, i, i, i, i, i, i, d, i, P, P, P, P, P, P, P, P, P, i]
        lib.oracle_hardware_threads.argtypes = []
        for f in (lib.oracle_index_scores, lib.oracle_topk, lib.oracle_attend, lib.oracle_forward,
                  lib.oracle_hardware_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def hardware_threads() -> int:
    return _load().oracle_hardware_threads()


def _bits(a) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 bit patterns."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch

        return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    arr = np.ascontiguousarray(a)
    if arr.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns (uint16), got {arr.dtype}")
    return arr


def _i32(a) -> np.ndarray:
    if hasattr(a, "cpu"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def index_scores(q_idx, w, k_idx, q_pos, n_threads: int = 0) -> np.ndarray:
    """Indexer scores, fp64.  q_idx [B,T,Hi,Di], w [B,T,Hi], k_idx [B,L,Di], q_pos [B,T].

    Returns scores [B,T,L]; positions after q_pos are -inf.
    """
    qb, wb, kb, pos = _bits(q_idx), _bits(w), _bits(k_idx), _i32(q_pos)
    B, T, Hi, Di = qb.shape
    L = kb.shape[1]
    assert wb.shape == (B, T, Hi) and kb.shape == (B, L, Di) and pos.shape == (B, T)
    out = np.empty((B, T, L), dtype=np.float64)
    rc = _load().oracle_index_scores(B, T, L, Hi, Di, _ptr(qb), _ptr(wb), _ptr(kb), _ptr(pos), _ptr(out), n_threads)
    if rc:
        raise ValueError("oracle_index_scores: position out of range")
    return out


def e4m3_to_float64(codes) -> np.ndarray:
    """FP8 E4M3 bit patterns -> exact values.

    The format: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  An
    exponent field e > 0 gives (1 + m/8) * 2^(e-7); e = 0 is subnormal,
    (m/8) * 2^-6.  There are no infinities; S.1111.111 is NaN, so the largest
    finite value is 1.75 * 2^8 = 448.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    return np.where((e == 15) & (c & 0x7 == 7), np.nan, sign * mag)


def e4m3_to_bf16_bits(codes) -> np.ndarray:
    """FP8 E4M3 codes -> bf16 bit patterns of the same values.  Exact: a finite
    E4M3 value has at most 4 significant bits and an exponent in [-9, 8]."""
    v = e4m3_to_float64(codes).astype(np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)


def _codes(a) -> np.ndarray:
    if hasattr(a, "cpu"):
        a = a.detach().cpu().contiguous()
        if str(a.dtype) == "torch.float8_e4m3fn":
            import torch

            a = a.view(torch.uint8)
        a = a.numpy()
    arr = np.ascontiguousarray(a)
    if arr.dtype != np.uint8:
        raise TypeError(f"expected E4M3 codes (uint8), got {arr.dtype}")
    return arr


def index_scores_e4m3(q_idx, w, k_idx, q_pos, n_threads: int = 0) -> np.ndarray:
    """index_scores with E4M3 indexer queries [B,T,Hi,Di] and keys [B,L,Di] (codes)."""
    return index_scores(e4m3_to_bf16_bits(_codes(q_idx)), w, e4m3_to_bf16_bits(_codes(k_idx)), q_pos, n_threads)


def topk(scores, q_pos, k: int = TOP_K, n_threads: int = 0) -> np.ndarray:
    """Top-k positions per row (ties -> lower position), ascending, -1 padded.

    scores [..., L] fp64, q_pos [...] -> idx [..., k] int32.
    """
    sc = np.ascontiguousarray(scores, dtype=np.float64)
    pos = _i32(q_pos)
    lead = sc.shape[:-1]
    L = sc.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    assert pos.size == rows
    out = np.empty(lead + (k,), dtype=np.int32)
    rc = _load().oracle_topk(rows, L, _ptr(sc), _ptr(pos.reshape(-1)), k, _ptr(out), n_threads)
    if rc:
        raise ValueError("oracle_topk: bad arguments")
    return out


def attend(q, kv, idx, gate=None, scale: float = SCALE, v_dim: int = V_DIM, n_threads: int = 0) -> np.ndarray:
    """Sparse latent attention + sigmoid head gate, fp64.

    q [B,T,H,Dq], kv [B,L,Dq], idx [B,T,K] (-1 = empty slot), gate [B,T,H] or None.
    Returns out [B,T,H,Dv].
    """
    qb, kvb, ix = _bits(q), _bits(kv), _i32(idx)
    B, T, H, Dq = qb.shape
    L = kvb.shape[1]
    K = ix.shape[-1]
    assert kvb.shape == (B, L, Dq) and ix.shape == (B, T, K)
    gb = None if gate is None else _bits(gate)
    if gb is not None:
        assert gb.shape == (B, T, H)
    out = np.empty((B, T, H, v_dim), dtype=np.float64)
    rc = _load().oracle_attend(B, T, L, H, Dq, v_dim, float(scale), _ptr(qb), _ptr(kvb), _ptr(ix), K,
                               None if gb is None else _ptr(gb), _ptr(out), n_threads)
    if rc:
        raise ValueError("oracle_attend: index out of range")
    return out


def forward(q_idx, w, k_idx, q, kv, gate, q_pos, k: int = TOP_K, scale: float = SCALE,
            v_dim: int = V_DIM, n_threads: int = 0):
    """Indexer -> top-k -> attention + gate.  Returns (idx [B,T,k], out [B,T,H,Dv])."""
    qib, wb, kib = _bits(q_idx), _bits(w), _bits(k_idx)
    qb, kvb, pos = _bits(q), _bits(kv), _i32(q_pos)
    gb = None if gate is None else _bits(gate)
    B, T, Hi, Di = qib.shape
    L = kib.shape[1]
    H, Dq = qb.shape[2], qb.shape[3]
    idx = np.empty((B, T, k), dtype=np.int32)
    out = np.empty((B, T, H, v_dim), dtype=np.float64)
    rc = _load().oracle_forward(B, T, L, Hi, Di, H, Dq, v_dim, float(scale), k, _ptr(qib), _ptr(wb), _ptr(kib),
                                _ptr(qb), _ptr(kvb), None if gb is None else _ptr(gb), _ptr(pos), _ptr(idx),
                                _ptr(out), n_threads)
    if rc:
        raise ValueError("oracle_forward: bad arguments")
    return idx, out


def forward_e4m3(q_idx, w, k_idx, q, kv, gate, q_pos, k: int = TOP_K, scale: float = SCALE, v_dim: int = V_DIM,
                 n_threads: int = 0):
    """forward with E4M3 indexer queries and keys (codes); returns (idx, out) as forward does."""
    return forward(e4m3_to_bf16_bits(_codes(q_idx)), w, e4m3_to_bf16_bits(_codes(k_idx)), q, kv, gate, q_pos, k=k,
                   scale=scale, v_dim=v_dim, n_threads=n_threads)
