"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/sga.h declares, sizes workspaces and rejects bad arguments before
touching the GPU.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import sparse_gated_attention_b200 as sga
from sparse_gated_attention_b200 import build as sga_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    sga_build.build()
    return sga.load_library()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "sga.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"SGA_API\s+[\w\s\*]+?\b(sga_\w+)\s*\(", text)))


def test_header_declares_the_four_steps():
    names = declared_symbols()
    for n in ["sga_index_scores", "sga_topk_select", "sga_sparse_mla_attend", "sga_forward"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert names and set(names) == set(sga.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings(lib):
    assert lib.sga_abi_version() == 1
    assert lib.sga_status_string(0) == b"SGA_OK"
    assert lib.sga_status_string(5) == b"SGA_ERR_TIMEOUT"
    assert lib.sga_status_string(7) == b"SGA_ERR_INTERNAL"
    assert lib.sga_status_string(99) == b"SGA_ERR_UNKNOWN"


def test_debug_library_builds_and_exports_the_same_calls():
    """libsga_debug.so: the same sources with the SGA_DEBUG invariant checks."""
    path = sga_build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for n in sga.EXPORTED:
        assert hasattr(dbg, n), n
    dbg.sga_status_string.restype = ctypes.c_char_p
    dbg.sga_status_string.argtypes = [ctypes.c_int]
    assert dbg.sga_status_string(7) == b"SGA_ERR_INTERNAL"


def test_workspace_sizes(lib):
    d = sga.make_dims(32, 1, 131072)
    idx_ws = sga.workspace_size(d, sga.OP_INDEX_SCORES)
    topk_ws = sga.workspace_size(d, sga.OP_TOPK_SELECT)
    att_ws = sga.workspace_size(d, sga.OP_SPARSE_MLA_ATTEND)
    fwd_ws = sga.workspace_size(d, sga.OP_FORWARD)
    assert idx_ws == 256
    assert topk_ws == 256 + 2 * 32 * (131072 // 32) * 4
    # the splits of a query merge on chip: the attention needs only the status word
    assert att_ws == 256
    assert fwd_ws >= topk_ws + 32 * 131072 * 4 + 32 * 2048 * 4
    # prefill: 4096 queries fill the GPU without splitting
    p = sga.make_dims(1, 4096, 131072)
    assert sga.workspace_size(p, sga.OP_SPARSE_MLA_ATTEND) == 256
    # the fused selection: no scores and no bitmaps; 8-byte candidates, the
    # histograms and one 128-byte counter line per query
    fused_ws = sga.workspace_size(d, sga.OP_FORWARD_FUSED)
    assert fused_ws == 256 + 32 * 2048 * 4 + 32 * 4096 * 4 + 32 * 131072 * 8 + 32 * 128
    # rows the fused selection does not take (prefill; L above 262,144) use the plain layout
    assert sga.workspace_size(p, sga.OP_FORWARD_FUSED) == sga.workspace_size(p, sga.OP_FORWARD)
    big = sga.make_dims(2, 1, 262144 + 32)
    assert sga.workspace_size(big, sga.OP_FORWARD_FUSED) == sga.workspace_size(big, sga.OP_FORWARD)
    edge = sga.make_dims(2, 1, 262144)
    assert sga.workspace_size(edge, sga.OP_FORWARD_FUSED) != sga.workspace_size(edge, sga.OP_FORWARD)
    with pytest.raises(sga.SGAError):
        sga.workspace_size(d, sga.OP_FORWARD_FUSED + 1)


@pytest.mark.parametrize("dims", [(0, 1, 100, 2048), (1, 0, 100, 2048), (1, 1, 0, 2048), (1, 1, 100, 100),
                                  (1, 1, 100, 4096), (1, 1, 100, 0), (70000, 1, 1 << 20, 2048)])
def test_bad_dims_rejected(lib, dims):
    d = sga.make_dims(*dims)
    out = ctypes.c_size_t(0)
    assert lib.sga_workspace_size(ctypes.byref(d), 3, ctypes.byref(out)) == 1


def test_null_and_misaligned_pointers_rejected_on_host(lib):
    d = sga.make_dims(1, 1, 4096)
    P = ctypes.c_void_p
    good = P(0x100000)
    odd = P(0x100002)
    ws = P(0x200000)
    # null inputs
    assert lib.sga_index_scores(ctypes.byref(d), None, good, good, good, good, ws, 1 << 20, None) == 1
    assert lib.sga_topk_select(ctypes.byref(d), good, good, None, ws, 1 << 20, None) == 1
    assert lib.sga_sparse_mla_attend(ctypes.byref(d), good, None, good, None, good, ws, 1 << 20, None) == 1
    # misaligned bf16 input (TMA needs 16-byte alignment)
    assert lib.sga_index_scores(ctypes.byref(d), good, good, odd, good, good, ws, 1 << 20, None) == 1
    assert lib.sga_sparse_mla_attend(ctypes.byref(d), odd, good, good, None, good, ws, 1 << 20, None) == 1
    # workspace: null, misaligned, too small
    assert lib.sga_topk_select(ctypes.byref(d), good, good, good, None, 1 << 20, None) == 3
    assert lib.sga_topk_select(ctypes.byref(d), good, good, good, P(0x200010), 1 << 20, None) == 3
    assert lib.sga_topk_select(ctypes.byref(d), good, good, good, ws, 64, None) == 3
    assert lib.sga_get_device_status(None, None, None) == 1
    assert lib.sga_clear_device_status(None, None) == 1
    # the bounded-wait diagnostic: budget out of range, workspace null / misaligned / too small
    assert lib.sga_selftest_bounded_wait(0, ws, 256, None) == 1
    assert lib.sga_selftest_bounded_wait(1 << 31, ws, 256, None) == 1
    assert lib.sga_selftest_bounded_wait(1000, None, 256, None) == 3
    assert lib.sga_selftest_bounded_wait(1000, P(0x200010), 256, None) == 3
    assert lib.sga_selftest_bounded_wait(1000, ws, 128, None) == 3


def test_binding_refuses_cpu_tensors():
    import torch

    q = torch.zeros((1, 1, 64, 576), dtype=torch.bfloat16)
    kv = torch.zeros((1, 8, 576), dtype=torch.bfloat16)
    idx = torch.zeros((1, 1, 64), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sga.sparse_mla_attend(q, kv, idx)


def test_binding_fails_loudly_without_library(tmp_path):
    from sparse_gated_attention_b200 import _binding

    saved = _binding._lib
    _binding._lib = None
    try:
        with pytest.raises(RuntimeError, match="libsga.so not found"):
            _binding.load_library(str(tmp_path / "missing.so"))
    finally:
        _binding._lib = saved


# ----------------------------------------------------------------------------- one SGA layer
def _layer_weights(d_model=7168, q_rank=1536, w_hq=0x300000, w_cq=0x400000, w_uk=0x500000, w_uv=0x600000,
                   w_o=0x700000):
    return sga.LayerWeights(d_model, q_rank, w_hq, w_cq, w_uk, w_uv, w_o)


def test_layer_workspace_sizes(lib):
    d = sga.make_dims(32, 1, 131072)
    lw = _layer_weights()
    proj = sga.layer_workspace_size(d, lw, sga.LAYER_PROJECT)
    outp = sga.layer_workspace_size(d, lw, sga.LAYER_OUTPUT)
    fwd = sga.layer_workspace_size(d, lw, sga.LAYER_FORWARD)
    rows = 32
    # 32 tokens: G1 (18 weight tiles of 128 rows) splits K eight ways for 148 SMs
    # and keeps eight fp32 partials, G2 (161 tiles) three; c_q and q_nope in bf16
    assert proj >= 256 + rows * 4 * (8 * (1536 + 768) + 3 * 20544) + rows * 2 * (1536 + 64 * 128)
    # the output side keeps out and o in bf16 and G5's five K-split fp32 partials
    assert outp >= 256 + rows * 2 * (64 * 512 + 8192) + 5 * rows * 7168 * 4
    # the whole layer also holds the path's workspace and the path's inputs and output
    assert fwd >= sga.workspace_size(d, sga.OP_FORWARD) + proj - 256 + outp - 256
    assert sga.layer_workspace_size(d, _layer_weights(q_rank=1024), sga.LAYER_FORWARD) < fwd


@pytest.mark.parametrize("d_model,q_rank", [(7170, 1536), (7168, 1530), (0, 1536), (7168, 0)])
def test_layer_bad_widths_rejected(lib, d_model, q_rank):
    d = sga.make_dims(2, 1, 1000)
    out = ctypes.c_size_t(0)
    lw = _layer_weights(d_model=d_model, q_rank=q_rank)
    assert lib.sga_layer_workspace_size(ctypes.byref(d), ctypes.byref(lw), sga.LAYER_FORWARD, ctypes.byref(out)) == 1


def test_layer_bad_arguments_rejected_on_host(lib):
    d = sga.make_dims(2, 1, 1000)
    P = ctypes.c_void_p
    good, odd, ws = P(0x100000), P(0x100002), P(0x20000000)
    big = 1 << 30
    out = ctypes.c_size_t(0)
    lw = _layer_weights()
    assert lib.sga_layer_workspace_size(ctypes.byref(d), ctypes.byref(lw), 7, ctypes.byref(out)) == 1
    assert lib.sga_layer_workspace_size(ctypes.byref(d), None, sga.LAYER_FORWARD, ctypes.byref(out)) == 1
    # null or misaligned weights and activations
    for bad in (_layer_weights(w_hq=0), _layer_weights(w_cq=0x400002), _layer_weights(w_uk=0)):
        assert lib.sga_layer_project(ctypes.byref(d), ctypes.byref(bad), good, good, good, good, good, good, good,
                                     good, ws, big, None) == 1
    for bad in (_layer_weights(w_uv=0), _layer_weights(w_o=0x700008)):
        assert lib.sga_layer_output(ctypes.byref(d), ctypes.byref(bad), good, good, ws, big, None) == 1
    assert lib.sga_layer_project(ctypes.byref(d), ctypes.byref(lw), odd, good, good, good, good, good, good, good,
                                 ws, big, None) == 1
    assert lib.sga_layer_forward(ctypes.byref(d), ctypes.byref(lw), good, good, good, good, None, odd, ws, big,
                                 None) == 1
    # workspace: null, misaligned, too small
    assert lib.sga_layer_output(ctypes.byref(d), ctypes.byref(lw), good, good, None, big, None) == 3
    assert lib.sga_layer_output(ctypes.byref(d), ctypes.byref(lw), good, good, P(0x20000010), big, None) == 3
    assert lib.sga_layer_forward(ctypes.byref(d), ctypes.byref(lw), good, good, good, good, None, good, ws, 4096,
                                 None) == 3
    # the whole layer checks the path's top_k too
    bad_k = sga.make_dims(2, 1, 1000, 100)
    assert lib.sga_layer_workspace_size(ctypes.byref(bad_k), ctypes.byref(lw), sga.LAYER_FORWARD,
                                        ctypes.byref(out)) == 1


# ----------------------------------------------------------------------------- indexer warm-up objective
def test_warmup_workspace_size(lib):
    d = sga.make_dims(2, 3, 5000, 2048)
    rows, K = 6, 2048
    # status block, then z and a ([rows][64][K] fp32 each), the scores ([rows][K] fp32), each 64-slot
    # chunk's softmax statistics per head ([rows][64][K / 64] float pairs) and of its scores ([rows][K / 64]
    # float pairs), and its loss term ([rows][K / 64])
    assert sga.indexer_warmup_workspace_size(d) == (256 + 2 * rows * 64 * K * 4 + rows * K * 4 + rows * 64 * 32 * 8
                                                    + rows * 32 * 8 + rows * 32 * 4)


@pytest.mark.parametrize("dims", [(1, 1, 100, 100), (1, 1, 100, 0), (70000, 1, 100, 2048), (0, 1, 100, 2048)])
def test_warmup_bad_dims_rejected(lib, dims):
    d = sga.make_dims(*dims)
    out = ctypes.c_size_t(0)
    assert lib.sga_indexer_warmup_workspace_size(ctypes.byref(d), ctypes.byref(out)) == 1


def test_warmup_bad_arguments_rejected_on_host(lib):
    d = sga.make_dims(2, 1, 1000, 2048)
    P = ctypes.c_void_p
    g, odd, ws = P(0x100000), P(0x100002), P(0x20000000)
    big = 1 << 30
    call = lib.sga_indexer_warmup
    assert call(ctypes.byref(d), None, g, g, g, g, g, g, g, g, g, ws, big, None) == 1   # q_idx null
    assert call(ctypes.byref(d), g, g, g, odd, g, g, g, g, g, g, ws, big, None) == 1    # q misaligned
    assert call(ctypes.byref(d), g, g, g, g, g, g, g, g, g, None, ws, big, None) == 1   # grad_k_idx null
    assert call(ctypes.byref(d), g, g, g, g, g, g, g, g, g, g, None, big, None) == 3    # workspace null
    assert call(ctypes.byref(d), g, g, g, g, g, g, g, g, g, g, P(0x20000010), big, None) == 3
    assert call(ctypes.byref(d), g, g, g, g, g, g, g, g, g, g, ws, 1024, None) == 3      # too small


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "sga.h"

int main(void) {
  sga_dims_t d = {32, 1, 131072, 2048};
  size_t fwd = 0, att = 0, warm = 0, layer = 0;
  sga_layer_weights_t lw = {7168, 1536, 0, 0, 0, 0, 0};
  if (sga_abi_version() != 1) return 1;
  if (strcmp(sga_status_string(SGA_OK), "SGA_OK") != 0) return 2;
  if (sga_workspace_size(&d, SGA_OP_FORWARD, &fwd) != SGA_OK || fwd == 0) return 3;
  if (sga_workspace_size(&d, SGA_OP_SPARSE_MLA_ATTEND, &att) != SGA_OK || att != 256) return 4;
  if (sga_indexer_warmup_workspace_size(&d, &warm) != SGA_OK || warm == 0) return 5;
  if (sga_layer_workspace_size(&d, &lw, SGA_LAYER_FORWARD, &layer) != SGA_OK || layer <= fwd) return 6;
  /* rejected on the host, before any device call */
  if (sga_index_scores(&d, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) != SGA_ERR_INVALID_ARG) return 7;
  d.top_k = 100;
  if (sga_workspace_size(&d, SGA_OP_FORWARD, &fwd) != SGA_ERR_INVALID_ARG) return 8;
  printf("ok %zu %zu %zu\n", att, warm, layer);
  return 0;
}
"""


def test_the_header_is_a_c_abi(lib, tmp_path):
    """A C99 program includes include/sga.h, links libsga.so and calls the host-only entry points."""
    import subprocess

    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(sga.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), os.path.join(libdir, "libsga.so"),
                           "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("ok 256 ")
