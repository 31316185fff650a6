"""ctypes binding of libsga (include/sga.h): argument marshalling only.

Every step of the path runs in the CUDA library; this module checks tensor
shapes, dtypes and devices, allocates outputs and workspaces with PyTorch when
the caller does not pass them, and forwards raw pointers and the current CUDA
stream.  There is no fallback: if libsga.so is missing or the device is not an
sm_100 GPU the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsga.so")
# The SGA_DEBUG build (device invariant checks compiled in); load_library takes it
# when the environment sets SGA_LIBRARY=debug.
LIB_DEBUG_PATH = os.path.join(_PKG, "libsga_debug.so")

INDEX_HEADS = 64
INDEX_DIM = 128
HEADS = 64
QK_DIM = 576
V_DIM = 512
TOP_K = 2048

OP_INDEX_SCORES, OP_TOPK_SELECT, OP_SPARSE_MLA_ATTEND, OP_FORWARD, OP_FORWARD_FUSED = 0, 1, 2, 3, 4
LAYER_PROJECT, LAYER_OUTPUT, LAYER_FORWARD = 0, 1, 2
# packed layer weights (see sga_layer_weights_t): rows of w_hq after W_DQ, rows of w_cq
HQ_EXTRA = QK_DIM + INDEX_DIM + INDEX_HEADS  # 768
CQ_ROWS = HEADS * 192 + HEADS + INDEX_HEADS * INDEX_DIM  # 20,544
V_HEAD = 128
STATUS_NAMES = {0: "SGA_OK", 1: "SGA_ERR_INVALID_ARG", 2: "SGA_ERR_UNSUPPORTED", 3: "SGA_ERR_WORKSPACE",
                4: "SGA_ERR_CUDA", 5: "SGA_ERR_TIMEOUT", 6: "SGA_ERR_DEVICE_ARG", 7: "SGA_ERR_INTERNAL"}

EXPORTED = ["sga_abi_version", "sga_status_string", "sga_workspace_size", "sga_index_scores", "sga_topk_select",
            "sga_sparse_mla_attend", "sga_forward", "sga_get_device_status", "sga_clear_device_status",
            "sga_topk_select_noalloc", "sga_index_scores_fp8", "sga_forward_fp8", "sga_layer_workspace_size",
            "sga_layer_project", "sga_layer_output", "sga_layer_forward", "sga_indexer_warmup_workspace_size",
            "sga_indexer_warmup", "sga_selftest_bounded_wait", "sga_forward_fused", "sga_forward_fused_fp8"]
NOALLOC_SCRATCH_BYTES = 256 + 4 * 1024 * 1024


class SGAError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("kv_stride", ctypes.c_int32),
                ("top_k", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("q_rank", ctypes.c_int32), ("w_hq", ctypes.c_void_p),
                ("w_cq", ctypes.c_void_p), ("w_uk", ctypes.c_void_p), ("w_uv", ctypes.c_void_p),
                ("w_o", ctypes.c_void_p)]


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Loads libsga.so (built in-tree by ``sparse_gated_attention_b200.build``), or
    libsga_debug.so when the environment sets SGA_LIBRARY=debug."""
    global _lib
    if _lib is not None:
        return _lib
    if path is None:
        path = LIB_DEBUG_PATH if os.environ.get("SGA_LIBRARY") == "debug" else LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libsga.so not found at {path}: build it with `python -m sparse_gated_attention_b200.build`")
    lib = ctypes.CDLL(path)
    P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D = ctypes.POINTER(Dims)
    sig = {
        "sga_abi_version": (i32, []),
        "sga_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "sga_workspace_size": (ctypes.c_int, [D, ctypes.c_int, ctypes.POINTER(sz)]),
        "sga_index_scores": (ctypes.c_int, [D, P, P, P, P, P, P, sz, P]),
        "sga_topk_select": (ctypes.c_int, [D, P, P, P, P, sz, P]),
        "sga_sparse_mla_attend": (ctypes.c_int, [D, P, P, P, P, P, P, sz, P]),
        "sga_forward": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, P, sz, P]),
        "sga_get_device_status": (ctypes.c_int, [P, P, ctypes.POINTER(i32)]),
        "sga_clear_device_status": (ctypes.c_int, [P, P]),
        "sga_topk_select_noalloc": (ctypes.c_int, [D, P, P, P, P]),
        "sga_index_scores_fp8": (ctypes.c_int, [D, P, P, P, P, P, P, sz, P]),
        "sga_forward_fp8": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, P, sz, P]),
        "sga_forward_fused": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, P, sz, P]),
        "sga_forward_fused_fp8": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, P, sz, P]),
        "sga_layer_workspace_size": (ctypes.c_int, [D, ctypes.POINTER(LayerWeights), ctypes.c_int,
                                                    ctypes.POINTER(sz)]),
        "sga_layer_project": (ctypes.c_int, [D, ctypes.POINTER(LayerWeights), P, P, P, P, P, P, P, P, P, sz, P]),
        "sga_layer_output": (ctypes.c_int, [D, ctypes.POINTER(LayerWeights), P, P, P, sz, P]),
        "sga_layer_forward": (ctypes.c_int, [D, ctypes.POINTER(LayerWeights), P, P, P, P, P, P, P, sz, P]),
        "sga_indexer_warmup_workspace_size": (ctypes.c_int, [D, ctypes.POINTER(sz)]),
        "sga_indexer_warmup": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, P, P, sz, P]),
        "sga_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_int64, P, sz, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(call: str, status: int) -> None:
    if status != 0:
        raise SGAError(call, status)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _need_fp8(t, name, shape):
    """An E4M3 tensor (torch.float8_e4m3fn, or its bytes as uint8), returned as uint8."""
    if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    return _need(t, name, torch.uint8, shape)


def make_dims(batch: int, n_q: int, kv_stride: int, top_k: int = TOP_K) -> Dims:
    return Dims(int(batch), int(n_q), int(kv_stride), int(top_k))


def workspace_size(dims: Dims, op: int = OP_FORWARD) -> int:
    out = ctypes.c_size_t(0)
    _check("sga_workspace_size", load_library().sga_workspace_size(ctypes.byref(dims), int(op), ctypes.byref(out)))
    return int(out.value)


def alloc_workspace(dims: Dims, op: int = OP_FORWARD, device=None) -> torch.Tensor:
    """A zero-filled workspace (zero = clear device status)."""
    n = workspace_size(dims, op)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def device_status(ws: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("sga_get_device_status", load_library().sga_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(v)))
    return int(v.value)


def clear_device_status(ws: torch.Tensor, stream=None) -> None:
    _check("sga_clear_device_status", load_library().sga_clear_device_status(_ptr(ws), _stream(stream)))


def index_scores(q_idx, w, k_idx, q_pos, scores=None, ws=None, stream=None):
    """Indexer scores [B,T,L] fp32 (entries after each query's position are not written)."""
    B, T = q_idx.shape[0], q_idx.shape[1]
    L = k_idx.shape[1]
    _need(q_idx, "q_idx", torch.bfloat16, (B, T, INDEX_HEADS, INDEX_DIM))
    _need(w, "w", torch.bfloat16, (B, T, INDEX_HEADS))
    _need(k_idx, "k_idx", torch.bfloat16, (B, L, INDEX_DIM))
    _need(q_pos, "q_pos", torch.int32, (B, T))
    dims = make_dims(B, T, L)
    if scores is None:
        scores = torch.empty((B, T, L), dtype=torch.float32, device=q_idx.device)
    _need(scores, "scores", torch.float32, (B, T, L))
    if ws is None:
        ws = alloc_workspace(dims, OP_INDEX_SCORES, q_idx.device)
    _check("sga_index_scores", load_library().sga_index_scores(
        ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(q_pos), _ptr(scores), _ptr(ws), ws.numel(),
        _stream(stream)))
    return scores


def index_scores_fp8(q_idx, w, k_idx, q_pos, scores=None, ws=None, stream=None):
    """Indexer scores [B,T,L] fp32 with E4M3 indexer queries and keys (see sga_index_scores_fp8)."""
    B, T = q_idx.shape[0], q_idx.shape[1]
    L = k_idx.shape[1]
    q_idx = _need_fp8(q_idx, "q_idx", (B, T, INDEX_HEADS, INDEX_DIM))
    k_idx = _need_fp8(k_idx, "k_idx", (B, L, INDEX_DIM))
    _need(w, "w", torch.bfloat16, (B, T, INDEX_HEADS))
    _need(q_pos, "q_pos", torch.int32, (B, T))
    dims = make_dims(B, T, L)
    if scores is None:
        scores = torch.empty((B, T, L), dtype=torch.float32, device=q_idx.device)
    _need(scores, "scores", torch.float32, (B, T, L))
    if ws is None:
        ws = alloc_workspace(dims, OP_INDEX_SCORES, q_idx.device)
    _check("sga_index_scores_fp8", load_library().sga_index_scores_fp8(
        ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(q_pos), _ptr(scores), _ptr(ws), ws.numel(),
        _stream(stream)))
    return scores


def topk_select(scores, q_pos, top_k: int = TOP_K, idx=None, ws=None, stream=None):
    """Top-k positions [B,T,K] int32, ascending, -1 padded (ties -> lower position)."""
    B, T, L = scores.shape
    _need(scores, "scores", torch.float32, (B, T, L))
    _need(q_pos, "q_pos", torch.int32, (B, T))
    dims = make_dims(B, T, L, top_k)
    if idx is None:
        idx = torch.empty((B, T, top_k), dtype=torch.int32, device=scores.device)
    _need(idx, "idx", torch.int32, (B, T, top_k))
    if ws is None:
        ws = alloc_workspace(dims, OP_TOPK_SELECT, scores.device)
    _check("sga_topk_select", load_library().sga_topk_select(
        ctypes.byref(dims), _ptr(scores), _ptr(q_pos), _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)))
    return idx


def topk_select_noalloc(scores, q_pos, top_k: int = TOP_K, idx=None, stream=None):
    """Top-k without a workspace (the library's own static scratch; see sga.h)."""
    B, T, L = scores.shape
    _need(scores, "scores", torch.float32, (B, T, L))
    _need(q_pos, "q_pos", torch.int32, (B, T))
    dims = make_dims(B, T, L, top_k)
    if idx is None:
        idx = torch.empty((B, T, top_k), dtype=torch.int32, device=scores.device)
    _need(idx, "idx", torch.int32, (B, T, top_k))
    _check("sga_topk_select_noalloc", load_library().sga_topk_select_noalloc(
        ctypes.byref(dims), _ptr(scores), _ptr(q_pos), _ptr(idx), _stream(stream)))
    return idx


def sparse_mla_attend(q, kv, idx, gate=None, out=None, ws=None, stream=None):
    """Sparse latent attention + sigmoid head gate -> out [B,T,64,512] fp32."""
    B, T = q.shape[0], q.shape[1]
    L = kv.shape[1]
    K = idx.shape[-1]
    _need(q, "q", torch.bfloat16, (B, T, HEADS, QK_DIM))
    _need(kv, "kv", torch.bfloat16, (B, L, QK_DIM))
    _need(idx, "idx", torch.int32, (B, T, K))
    if gate is not None:
        _need(gate, "gate", torch.bfloat16, (B, T, HEADS))
    dims = make_dims(B, T, L, K)
    if out is None:
        out = torch.empty((B, T, HEADS, V_DIM), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, T, HEADS, V_DIM))
    if ws is None:
        ws = alloc_workspace(dims, OP_SPARSE_MLA_ATTEND, q.device)
    _check("sga_sparse_mla_attend", load_library().sga_sparse_mla_attend(
        ctypes.byref(dims), _ptr(q), _ptr(kv), _ptr(idx), _ptr(gate), _ptr(out), _ptr(ws), ws.numel(),
        _stream(stream)))
    return out


def _forward_call(call: str, fp8: bool, op: int, q_idx, w, k_idx, q, kv, gate, q_pos, top_k, idx_out, out, ws,
                  stream, return_idx):
    B, T = q_idx.shape[0], q_idx.shape[1]
    L = k_idx.shape[1]
    if fp8:
        q_idx = _need_fp8(q_idx, "q_idx", (B, T, INDEX_HEADS, INDEX_DIM))
        k_idx = _need_fp8(k_idx, "k_idx", (B, L, INDEX_DIM))
    else:
        _need(q_idx, "q_idx", torch.bfloat16, (B, T, INDEX_HEADS, INDEX_DIM))
        _need(k_idx, "k_idx", torch.bfloat16, (B, L, INDEX_DIM))
    _need(w, "w", torch.bfloat16, (B, T, INDEX_HEADS))
    _need(q, "q", torch.bfloat16, (B, T, HEADS, QK_DIM))
    _need(kv, "kv", torch.bfloat16, (B, L, QK_DIM))
    if gate is not None:
        _need(gate, "gate", torch.bfloat16, (B, T, HEADS))
    _need(q_pos, "q_pos", torch.int32, (B, T))
    dims = make_dims(B, T, L, top_k)
    if idx_out is None and return_idx:
        idx_out = torch.empty((B, T, top_k), dtype=torch.int32, device=q.device)
    if idx_out is not None:
        _need(idx_out, "idx_out", torch.int32, (B, T, top_k))
    if out is None:
        out = torch.empty((B, T, HEADS, V_DIM), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, T, HEADS, V_DIM))
    if ws is None:
        ws = alloc_workspace(dims, op, q.device)
    _check(call, getattr(load_library(), call)(
        ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(q), _ptr(kv), _ptr(gate), _ptr(q_pos),
        _ptr(idx_out), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, out


def forward(q_idx, w, k_idx, q, kv, gate, q_pos, top_k: int = TOP_K, idx_out=None, out=None, ws=None,
            stream=None, return_idx: bool = True):
    """The whole path.  Returns (idx [B,T,K] or None, out [B,T,64,512])."""
    return _forward_call("sga_forward", False, OP_FORWARD, q_idx, w, k_idx, q, kv, gate, q_pos, top_k, idx_out,
                         out, ws, stream, return_idx)


def forward_fp8(q_idx, w, k_idx, q, kv, gate, q_pos, top_k: int = TOP_K, idx_out=None, out=None, ws=None,
                stream=None, return_idx: bool = True):
    """The whole path with E4M3 indexer queries and keys (see sga_forward_fp8)."""
    return _forward_call("sga_forward_fp8", True, OP_FORWARD, q_idx, w, k_idx, q, kv, gate, q_pos, top_k, idx_out,
                         out, ws, stream, return_idx)


def forward_fused(q_idx, w, k_idx, q, kv, gate, q_pos, top_k: int = TOP_K, idx_out=None, out=None, ws=None,
                  stream=None, return_idx: bool = True):
    """The whole path with the selection fused into the indexer (see
    sga_forward_fused): the results of `forward`.  A workspace passed in is
    sized for OP_FORWARD_FUSED."""
    return _forward_call("sga_forward_fused", False, OP_FORWARD_FUSED, q_idx, w, k_idx, q, kv, gate, q_pos, top_k,
                         idx_out, out, ws, stream, return_idx)


def forward_fused_fp8(q_idx, w, k_idx, q, kv, gate, q_pos, top_k: int = TOP_K, idx_out=None, out=None, ws=None,
                      stream=None, return_idx: bool = True):
    """`forward_fused` with E4M3 indexer queries and keys: the results of `forward_fp8`."""
    return _forward_call("sga_forward_fused_fp8", True, OP_FORWARD_FUSED, q_idx, w, k_idx, q, kv, gate, q_pos,
                         top_k, idx_out, out, ws, stream, return_idx)


# ----------------------------------------------------------------------------- one SGA layer
def layer_weights(wts: dict) -> LayerWeights:
    """The C struct for packed bf16 weights {w_hq, w_cq, w_uk, w_uv, w_o} (see sga_layer_weights_t).
    The tensors must stay alive while the struct is in use."""
    w_hq, w_cq, w_o = wts["w_hq"], wts["w_cq"], wts["w_o"]
    D = w_hq.shape[1]
    R = w_hq.shape[0] - HQ_EXTRA
    _need(w_hq, "w_hq", torch.bfloat16, (R + HQ_EXTRA, D))
    _need(w_cq, "w_cq", torch.bfloat16, (CQ_ROWS, R))
    _need(wts["w_uk"], "w_uk", torch.bfloat16, (HEADS, 128, V_DIM))
    _need(wts["w_uv"], "w_uv", torch.bfloat16, (HEADS, V_HEAD, V_DIM))
    _need(w_o, "w_o", torch.bfloat16, (D, HEADS * V_HEAD))
    return LayerWeights(int(D), int(R), w_hq.data_ptr(), w_cq.data_ptr(), wts["w_uk"].data_ptr(),
                        wts["w_uv"].data_ptr(), w_o.data_ptr())


def layer_workspace_size(dims: Dims, lw: LayerWeights, op: int = LAYER_FORWARD) -> int:
    out = ctypes.c_size_t(0)
    _check("sga_layer_workspace_size", load_library().sga_layer_workspace_size(
        ctypes.byref(dims), ctypes.byref(lw), int(op), ctypes.byref(out)))
    return int(out.value)


def alloc_layer_workspace(dims: Dims, lw: LayerWeights, op: int = LAYER_FORWARD, device=None) -> torch.Tensor:
    """A zero-filled layer workspace (ready for the first sga_layer_forward)."""
    return torch.zeros(layer_workspace_size(dims, lw, op), dtype=torch.uint8, device=device or "cuda")


def _layer_common(wts, h, q_pos, kv_cache, k_idx_cache):
    lw = layer_weights(wts)
    B, T, D = h.shape
    L = kv_cache.shape[1]
    _need(h, "h", torch.bfloat16, (B, T, lw.d_model))
    _need(q_pos, "q_pos", torch.int32, (B, T))
    _need(kv_cache, "kv_cache", torch.bfloat16, (B, L, QK_DIM))
    _need(k_idx_cache, "k_idx_cache", torch.bfloat16, (B, L, INDEX_DIM))
    return lw, B, T, L


def layer_project(wts, h, q_pos, kv_cache, k_idx_cache, ws=None, stream=None):
    """The projections in front of the path (sga_layer_project).  Writes the new tokens'
    rows into the caches in place; returns dict(q, gate, q_idx, w), bf16."""
    lw, B, T, L = _layer_common(wts, h, q_pos, kv_cache, k_idx_cache)
    dev = h.device
    q = torch.empty((B, T, HEADS, QK_DIM), dtype=torch.bfloat16, device=dev)
    gate = torch.empty((B, T, HEADS), dtype=torch.bfloat16, device=dev)
    q_idx = torch.empty((B, T, INDEX_HEADS, INDEX_DIM), dtype=torch.bfloat16, device=dev)
    w = torch.empty((B, T, INDEX_HEADS), dtype=torch.bfloat16, device=dev)
    dims = make_dims(B, T, L)
    if ws is None:
        ws = alloc_layer_workspace(dims, lw, LAYER_PROJECT, dev)
    _check("sga_layer_project", load_library().sga_layer_project(
        ctypes.byref(dims), ctypes.byref(lw), _ptr(h), _ptr(q_pos), _ptr(kv_cache), _ptr(k_idx_cache), _ptr(q),
        _ptr(gate), _ptr(q_idx), _ptr(w), _ptr(ws), ws.numel(), _stream(stream)))
    return {"q": q, "gate": gate, "q_idx": q_idx, "w": w}


def layer_output(wts, out, y=None, ws=None, stream=None):
    """The projections after the path (sga_layer_output): out [B,T,64,512] fp32 -> y [B,T,D] fp32."""
    lw = layer_weights(wts)
    B, T = out.shape[0], out.shape[1]
    _need(out, "out", torch.float32, (B, T, HEADS, V_DIM))
    if y is None:
        y = torch.empty((B, T, lw.d_model), dtype=torch.float32, device=out.device)
    _need(y, "y", torch.float32, (B, T, lw.d_model))
    dims = make_dims(B, T, 1)
    if ws is None:
        ws = alloc_layer_workspace(dims, lw, LAYER_OUTPUT, out.device)
    _check("sga_layer_output", load_library().sga_layer_output(
        ctypes.byref(dims), ctypes.byref(lw), _ptr(out), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def layer_forward(wts, h, q_pos, kv_cache, k_idx_cache, top_k: int = TOP_K, idx_out=None, y=None, ws=None,
                  stream=None, return_idx: bool = True):
    """One SGA layer (sga_layer_forward).  Writes the new tokens' cache rows in place;
    returns (idx [B,T,K] or None, y [B,T,D] fp32)."""
    lw, B, T, L = _layer_common(wts, h, q_pos, kv_cache, k_idx_cache)
    dims = make_dims(B, T, L, top_k)
    if idx_out is None and return_idx:
        idx_out = torch.empty((B, T, top_k), dtype=torch.int32, device=h.device)
    if idx_out is not None:
        _need(idx_out, "idx_out", torch.int32, (B, T, top_k))
    if y is None:
        y = torch.empty((B, T, lw.d_model), dtype=torch.float32, device=h.device)
    _need(y, "y", torch.float32, (B, T, lw.d_model))
    if ws is None:
        ws = alloc_layer_workspace(dims, lw, LAYER_FORWARD, h.device)
    _check("sga_layer_forward", load_library().sga_layer_forward(
        ctypes.byref(dims), ctypes.byref(lw), _ptr(h), _ptr(q_pos), _ptr(kv_cache), _ptr(k_idx_cache),
        _ptr(idx_out), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, y


# ----------------------------------------------------------------------------- indexer warm-up objective
def indexer_warmup_workspace_size(dims: Dims) -> int:
    out = ctypes.c_size_t(0)
    _check("sga_indexer_warmup_workspace_size",
           load_library().sga_indexer_warmup_workspace_size(ctypes.byref(dims), ctypes.byref(out)))
    return int(out.value)


def indexer_warmup(q_idx, w, k_idx, q, kv, idx, grad_k_idx=None, ws=None, stream=None):
    """The indexer's sparse warm-up objective over the selection idx (sga_indexer_warmup).
    Returns dict(loss [B,T], grad_q_idx [B,T,64,128], grad_w [B,T,64], grad_k_idx [B,L,128]),
    fp32; grad_k_idx is added to (a zero-filled tensor is made when none is passed)."""
    B, T = q_idx.shape[0], q_idx.shape[1]
    L = k_idx.shape[1]
    K = idx.shape[-1]
    _need(q_idx, "q_idx", torch.bfloat16, (B, T, INDEX_HEADS, INDEX_DIM))
    _need(w, "w", torch.bfloat16, (B, T, INDEX_HEADS))
    _need(k_idx, "k_idx", torch.bfloat16, (B, L, INDEX_DIM))
    _need(q, "q", torch.bfloat16, (B, T, HEADS, QK_DIM))
    _need(kv, "kv", torch.bfloat16, (B, L, QK_DIM))
    _need(idx, "idx", torch.int32, (B, T, K))
    dev = q_idx.device
    dims = make_dims(B, T, L, K)
    loss = torch.empty((B, T), dtype=torch.float32, device=dev)
    grad_q_idx = torch.empty((B, T, INDEX_HEADS, INDEX_DIM), dtype=torch.float32, device=dev)
    grad_w = torch.empty((B, T, INDEX_HEADS), dtype=torch.float32, device=dev)
    if grad_k_idx is None:
        grad_k_idx = torch.zeros((B, L, INDEX_DIM), dtype=torch.float32, device=dev)
    _need(grad_k_idx, "grad_k_idx", torch.float32, (B, L, INDEX_DIM))
    if ws is None:
        ws = torch.zeros(indexer_warmup_workspace_size(dims), dtype=torch.uint8, device=dev)
    _check("sga_indexer_warmup", load_library().sga_indexer_warmup(
        ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(q), _ptr(kv), _ptr(idx), _ptr(loss),
        _ptr(grad_q_idx), _ptr(grad_w), _ptr(grad_k_idx), _ptr(ws), ws.numel(), _stream(stream)))
    return {"loss": loss, "grad_q_idx": grad_q_idx, "grad_w": grad_w, "grad_k_idx": grad_k_idx}


def selftest_bounded_wait(budget_cycles: int, ws: torch.Tensor, stream=None) -> None:
    """Runs the bounded-wait diagnostic (sga_selftest_bounded_wait) on ``ws``
    (a uint8 device tensor of at least 256 bytes); asynchronous on the stream."""
    _need(ws, "ws", torch.uint8)
    _check("sga_selftest_bounded_wait", load_library().sga_selftest_bounded_wait(
        int(budget_cycles), _ptr(ws), ws.numel(), _stream(stream)))
