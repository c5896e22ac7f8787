"""Python binding of the B200 SpotAttention decode-path library.

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libspot_b200.so`` behind the C ABI of ``include/spot.h``; this module turns
torch CUDA tensors into device pointers and the current torch stream into a
``cudaStream_t``.  There is no CPU fallback: a missing library or a tensor
that is not on a CUDA device raises.

Functions (names as in the C ABI, without the ``spot_`` prefix):
``workspace_size``, ``append_selector_keys``, ``select``, ``sparse_decode``,
``decode_step``, ``read_device_status``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspot_b200.so")

SEL_FMT = {"bf16": 0, "int4": 1, "mxfp4": 2, "fp8": 3, "int8": 4}
MODE = {"topp": 0, "topk": 1}
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace too small",
          4: "CUDA error", 5: "device: index out of range", 6: "device: bounded wait timed out"}


class SpotError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")
        self.code = code


class LayerDesc(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("sel_dim", ctypes.c_int32), ("sel_fmt", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


class SelectParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("sink_blocks", ctypes.c_int32),
                ("recency_blocks", ctypes.c_int32), ("kmin_blocks", ctypes.c_int32),
                ("topk_blocks", ctypes.c_int32), ("temperature", ctypes.c_float),
                ("quantize_queries", ctypes.c_int32)]


class TokLayerDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_q_heads", "num_kv_heads", "head_dim", "page_size", "idx_heads", "idx_dim",
        "sel_block", "num_pages", "sel_fmt")]


def tok_layer_desc(num_q_heads, num_kv_heads, num_pages, head_dim=128, page_size=64,
                   idx_heads=4, idx_dim=128, sel_block=16, sel_fmt="bf16") -> TokLayerDesc:
    return TokLayerDesc(num_q_heads, num_kv_heads, head_dim, page_size, idx_heads, idx_dim,
                        sel_block, num_pages,
                        SEL_FMT[sel_fmt] if isinstance(sel_fmt, str) else int(sel_fmt))


def layer_desc(num_q_heads, num_kv_heads, num_pages, sel_fmt="bf16", head_dim=128,
               block_size=64, sel_dim=64) -> LayerDesc:
    return LayerDesc(num_q_heads, num_kv_heads, head_dim, block_size, sel_dim,
                     SEL_FMT[sel_fmt] if isinstance(sel_fmt, str) else int(sel_fmt), num_pages)


def select_params(mode="topp", sink_blocks=1, recency_blocks=4, kmin_blocks=8, topk_blocks=0,
                  temperature=1.0, quantize_queries=False) -> SelectParams:
    return SelectParams(MODE[mode] if isinstance(mode, str) else int(mode), sink_blocks,
                        recency_blocks, kmin_blocks, topk_blocks, float(temperature),
                        1 if quantize_queries else 0)


_lib = None


def lib():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "block_sparse_long_spot_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
        L.spot_workspace_size.argtypes = [P, i32, i32]
        L.spot_workspace_size.restype = sz
        L.spot_append_selector_keys.argtypes = [P, P, P, P, i32, i32, P, P, P, i32, P, P]
        L.spot_select.argtypes = [P, P, P, P, P, P, P, i32, P, P, i32, P, P, i32, P, sz, P]
        L.spot_sparse_decode.argtypes = [P, P, P, P, P, i32, P, P, P, i32, i32, f32, P, P, P, sz,
                                         P]
        L.spot_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, P, P, i32, f32, P, P,
                                       i32, P, P, P, sz, P]
        L.spot_sparse_decode_noalloc.argtypes = [P, P, P, P, P, i32, P, P, P, i32, i32, f32, P,
                                                 P, P]
        L.spot_tok_workspace_size.argtypes = [P, i32, i32]
        L.spot_tok_workspace_size.restype = sz
        L.spot_tok_append_selector_keys.argtypes = [P, P, P, P, i32, i32, P, P, P, i32, P, P]
        L.spot_tok_select.argtypes = [P, P, P, P, P, P, P, i32, P, P, i32, P, P, i32, P, sz, P]
        L.spot_tok_sparse_decode.argtypes = [P, P, P, P, P, i32, P, P, P, i32, i32, f32, P, P,
                                             P, sz, P]
        L.spot_tok_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, P, P, i32, f32, P,
                                           P, i32, P, P, P, sz, P]
        L.spot_prefill_num_tiles.argtypes = [P, P, i32]
        L.spot_prefill_num_tiles.restype = ctypes.c_int64
        L.spot_prefill_workspace_size.argtypes = [P, i32, i32, i32]
        L.spot_prefill_workspace_size.restype = sz
        L.spot_prefill.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, P, P, P, i32, i32, f32, P,
                                   P, i32, P, P, P, sz, P]
        L.spot_prefill.restype = ctypes.c_int
        L.spot_read_device_status.argtypes = [P, P]
        L.spot_check_wait_timeout.argtypes = [P, P]
        L.spot_check_wait_timeout.restype = ctypes.c_int
        L.spot_status_string.restype = ctypes.c_char_p
        for name in ("spot_append_selector_keys", "spot_select", "spot_sparse_decode",
                     "spot_decode_step", "spot_read_device_status",
                     "spot_sparse_decode_noalloc", "spot_tok_append_selector_keys",
                     "spot_tok_select", "spot_tok_sparse_decode", "spot_tok_decode_step"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code, where):
    if code != 0:
        raise SpotError(int(code), where)


def workspace_size(desc: LayerDesc, batch: int, max_blocks: int) -> int:
    n = lib().spot_workspace_size(ctypes.byref(desc), batch, max_blocks)
    if n == 0:
        raise SpotError(2, "workspace_size")
    return int(n)


def new_workspace(desc: LayerDesc, batch: int, max_blocks: int, device=None) -> torch.Tensor:
    """Zero-filled workspace of the required size (uint8, 256-byte aligned)."""
    n = workspace_size(desc, batch, max_blocks)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def append_selector_keys(desc: LayerDesc, sel_data, sel_scales, page_table, seq_ids, block_ids,
                         keys, status_ws=None, stream=None):
    """Write / quantise keys bf16 [n, Hkv, sel_dim] into the selector pool."""
    pt = page_table
    code = lib().spot_append_selector_keys(
        ctypes.byref(desc), _ptr(sel_data, name="sel_data"), _ptr(sel_scales, name="sel_scales"),
        _ptr(pt, torch.int32, "page_table"), int(pt.shape[0]), int(pt.shape[-1]),
        _ptr(seq_ids, torch.int32, "seq_ids"),
        _ptr(block_ids, torch.int32, "block_ids"), _ptr(keys, torch.bfloat16, "keys"),
        int(keys.shape[0]), _ptr(status_ws, name="status_ws"), _stream(stream))
    _check(code, "append_selector_keys")


def select(desc: LayerDesc, params: SelectParams, q_sel, w, sel_data, sel_scales, page_table,
           seq_lens, top_p, sel_idx, sel_cnt, workspace, stream=None):
    """Block selection into sel_idx int32 [B, Hkv, max_blocks], sel_cnt int32 [B, Hkv]."""
    B, max_blocks = int(q_sel.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_select(
        ctypes.byref(desc), ctypes.byref(params), _ptr(q_sel, torch.bfloat16, "q_sel"),
        _ptr(w, torch.float32, "w"), _ptr(sel_data, name="sel_data"),
        _ptr(sel_scales, name="sel_scales"), _ptr(page_table, torch.int32, "page_table"),
        int(page_table.shape[-1]), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(top_p, torch.float32, "top_p"), B, _ptr(sel_idx, torch.int32, "sel_idx"),
        _ptr(sel_cnt, torch.int32, "sel_cnt"), max_blocks, _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "select")


def sparse_decode(desc: LayerDesc, q, k_pool, v_pool, page_table, seq_lens, sel_idx, sel_cnt,
                  softmax_scale, out, lse, workspace, stream=None):
    """Attention over the selected blocks into out fp32 [B, Hq, D] (+ lse fp32 [B, Hq])."""
    B, max_blocks = int(q.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_sparse_decode(
        ctypes.byref(desc), _ptr(q, torch.bfloat16, "q"), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(v_pool, torch.bfloat16, "v_pool"), _ptr(page_table, torch.int32, "page_table"),
        int(page_table.shape[-1]), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"), max_blocks,
        B, float(softmax_scale), _ptr(out, torch.float32, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(code, "sparse_decode")


def sparse_decode_noalloc(desc: LayerDesc, q, k_pool, v_pool, page_table, seq_lens, sel_idx,
                          sel_cnt, softmax_scale, out, lse, stream=None):
    """sparse_decode without a workspace, for callers that cannot allocate
    device memory: the scratch is an 8 MiB array inside the library, shared
    by all calls (calls that overlap on the GPU race).  Shapes needing more
    raise SpotError(3).  Make the first call on a device before any stream
    capture."""
    B, max_blocks = int(q.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_sparse_decode_noalloc(
        ctypes.byref(desc), _ptr(q, torch.bfloat16, "q"), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(v_pool, torch.bfloat16, "v_pool"), _ptr(page_table, torch.int32, "page_table"),
        int(page_table.shape[-1]), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"), max_blocks,
        B, float(softmax_scale), _ptr(out, torch.float32, "out"), _ptr(lse, torch.float32, "lse"),
        _stream(stream))
    _check(code, "sparse_decode_noalloc")


def decode_step(desc: LayerDesc, params: SelectParams, q_sel, w, sel_data, sel_scales, q, k_pool,
                v_pool, page_table, seq_lens, top_p, softmax_scale, sel_idx, sel_cnt, out, lse,
                workspace, stream=None):
    """select followed by sparse_decode on one stream."""
    B, max_blocks = int(q.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_decode_step(
        ctypes.byref(desc), ctypes.byref(params), _ptr(q_sel, torch.bfloat16, "q_sel"),
        _ptr(w, torch.float32, "w"), _ptr(sel_data, name="sel_data"),
        _ptr(sel_scales, name="sel_scales"), _ptr(q, torch.bfloat16, "q"),
        _ptr(k_pool, torch.bfloat16, "k_pool"), _ptr(v_pool, torch.bfloat16, "v_pool"),
        _ptr(page_table, torch.int32, "page_table"), int(page_table.shape[-1]),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(top_p, torch.float32, "top_p"), B,
        float(softmax_scale), _ptr(sel_idx, torch.int32, "sel_idx"),
        _ptr(sel_cnt, torch.int32, "sel_cnt"), max_blocks, _ptr(out, torch.float32, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "decode_step")


# ---------------------------------------------- token-level, layer-shared selector

def tok_workspace_size(desc: TokLayerDesc, batch: int, max_blocks: int) -> int:
    n = lib().spot_tok_workspace_size(ctypes.byref(desc), batch, max_blocks)
    if n == 0:
        raise SpotError(2, "tok_workspace_size")
    return int(n)


def new_tok_workspace(desc: TokLayerDesc, batch: int, max_blocks: int, device=None):
    """Zero-filled workspace for the token selector's calls."""
    n = tok_workspace_size(desc, batch, max_blocks)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def tok_selector_pool(num_pages: int, fmt: str = "bf16", page_size=64, idx_heads=4, idx_dim=128,
                      device="cuda"):
    """Empty per-token selector pool (data, scales) for a format: key rows
    [pages, page_size, idx_heads, row] and their scales (None for bf16 /
    FP8)."""
    lead = (num_pages, page_size, idx_heads)
    if fmt == "bf16":
        return torch.zeros(*lead, idx_dim, dtype=torch.bfloat16, device=device), None
    if fmt == "fp8":
        return torch.zeros(*lead, idx_dim, dtype=torch.uint8, device=device), None
    if fmt == "int8":
        return (torch.zeros(*lead, idx_dim, dtype=torch.int8, device=device),
                torch.zeros(*lead, 1, dtype=torch.float16, device=device))
    data = torch.zeros(*lead, idx_dim // 2, dtype=torch.uint8, device=device)
    sdt = torch.float16 if fmt == "int4" else torch.uint8
    return data, torch.zeros(*lead, idx_dim // 32, dtype=sdt, device=device)


def tok_append_selector_keys(desc: TokLayerDesc, sel_data, sel_scales, page_table, seq_ids,
                             positions, keys, status_ws=None, stream=None):
    """Write (quantising to the pool's format) per-token selector keys bf16
    [n, idx_heads, idx_dim] by position."""
    pt = page_table
    code = lib().spot_tok_append_selector_keys(
        ctypes.byref(desc), _ptr(sel_data, name="sel_data"), _ptr(sel_scales, name="sel_scales"),
        _ptr(pt, torch.int32, "page_table"), int(pt.shape[0]), int(pt.shape[-1]),
        _ptr(seq_ids, torch.int32, "seq_ids"), _ptr(positions, torch.int32, "positions"),
        _ptr(keys, torch.bfloat16, "keys"), int(keys.shape[0]),
        _ptr(status_ws, name="status_ws"), _stream(stream))
    _check(code, "tok_append_selector_keys")


def tok_select(desc: TokLayerDesc, params: SelectParams, q_idx, w_idx, sel_data, sel_scales,
               page_table, seq_lens, top_p, sel_idx, sel_cnt, workspace, stream=None):
    """One selection per sequence into sel_idx int32 [B, max_blocks], sel_cnt int32 [B]."""
    B, max_blocks = int(q_idx.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_tok_select(
        ctypes.byref(desc), ctypes.byref(params), _ptr(q_idx, torch.bfloat16, "q_idx"),
        _ptr(w_idx, torch.float32, "w_idx"), _ptr(sel_data, name="sel_data"),
        _ptr(sel_scales, name="sel_scales"),
        _ptr(page_table, torch.int32, "page_table"), int(page_table.shape[-1]),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(top_p, torch.float32, "top_p"), B,
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"),
        max_blocks, _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "tok_select")


def tok_sparse_decode(desc: TokLayerDesc, q, k_pool, v_pool, page_table, seq_lens, sel_idx,
                      sel_cnt, softmax_scale, out, lse, workspace, stream=None):
    """Attention of every head over its sequence's selected 16-token blocks."""
    B, max_blocks = int(q.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_tok_sparse_decode(
        ctypes.byref(desc), _ptr(q, torch.bfloat16, "q"), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(v_pool, torch.bfloat16, "v_pool"), _ptr(page_table, torch.int32, "page_table"),
        int(page_table.shape[-1]), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"), max_blocks,
        B, float(softmax_scale), _ptr(out, torch.float32, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(code, "tok_sparse_decode")


def tok_decode_step(desc: TokLayerDesc, params: SelectParams, q_idx, w_idx, sel_data,
                    sel_scales, q, k_pool, v_pool, page_table, seq_lens, top_p, softmax_scale,
                    sel_idx, sel_cnt, out, lse, workspace, stream=None):
    """tok_select followed by tok_sparse_decode on one stream."""
    B, max_blocks = int(q.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_tok_decode_step(
        ctypes.byref(desc), ctypes.byref(params), _ptr(q_idx, torch.bfloat16, "q_idx"),
        _ptr(w_idx, torch.float32, "w_idx"), _ptr(sel_data, name="sel_data"),
        _ptr(sel_scales, name="sel_scales"),
        _ptr(q, torch.bfloat16, "q"), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(v_pool, torch.bfloat16, "v_pool"), _ptr(page_table, torch.int32, "page_table"),
        int(page_table.shape[-1]), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(top_p, torch.float32, "top_p"), B, float(softmax_scale),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_cnt, torch.int32, "sel_cnt"), max_blocks,
        _ptr(out, torch.float32, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(code, "tok_decode_step")


# ---------------------------------------------------------------- sparse prefill

def prefill_num_tiles(seq_lens, q_lens) -> int:
    """Query tiles of a batch (host lists / arrays of seq_lens and q_lens)."""
    import numpy as _np
    a = _np.ascontiguousarray(_np.asarray(seq_lens, dtype=_np.int32))
    b = _np.ascontiguousarray(_np.asarray(q_lens, dtype=_np.int32))
    n = lib().spot_prefill_num_tiles(a.ctypes.data_as(ctypes.c_void_p),
                                     b.ctypes.data_as(ctypes.c_void_p), int(a.size))
    if n < 0:
        raise SpotError(1, "prefill_num_tiles")
    return int(n)


def prefill_workspace_size(desc: LayerDesc, batch: int, max_tiles: int, max_blocks: int) -> int:
    n = lib().spot_prefill_workspace_size(ctypes.byref(desc), batch, max_tiles, max_blocks)
    if n == 0:
        raise SpotError(2, "prefill_workspace_size")
    return int(n)


def new_prefill_workspace(desc: LayerDesc, batch: int, max_tiles: int, max_blocks: int,
                          device=None) -> torch.Tensor:
    n = prefill_workspace_size(desc, batch, max_tiles, max_blocks)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def prefill(desc: LayerDesc, params: SelectParams, q_sel, w, sel_data, sel_scales, q, k_pool,
            v_pool, page_table, seq_lens, q_lens, top_p, softmax_scale, sel_idx, sel_cnt, out,
            lse, workspace, stream=None):
    """Sparse prefill of packed chunk queries: per (tile, KV head) selection
    into sel_idx int32 [max_tiles, Hkv, max_blocks] / sel_cnt [max_tiles, Hkv],
    causal attention into out fp32 [rows, Hq, D] (+ lse [rows, Hq]).  The
    selector pool (sel_data, sel_scales) is in the descriptor's format."""
    B = int(seq_lens.shape[0])
    max_tiles, max_blocks = int(sel_idx.shape[0]), int(sel_idx.shape[-1])
    code = lib().spot_prefill(
        ctypes.byref(desc), ctypes.byref(params), _ptr(q_sel, torch.bfloat16, "q_sel"),
        _ptr(w, torch.float32, "w"), _ptr(sel_data, name="sel_data"),
        _ptr(sel_scales, name="sel_scales"),
        _ptr(q, torch.bfloat16, "q"), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(v_pool, torch.bfloat16, "v_pool"), _ptr(page_table, torch.int32, "page_table"),
        int(page_table.shape[-1]), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(q_lens, torch.int32, "q_lens"), _ptr(top_p, torch.float32, "top_p"), B, max_tiles,
        float(softmax_scale), _ptr(sel_idx, torch.int32, "sel_idx"),
        _ptr(sel_cnt, torch.int32, "sel_cnt"), max_blocks, _ptr(out, torch.float32, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "prefill")


def check_wait_timeout(workspace, stream=None):
    """Run the failure-path check kernel (a wait nothing satisfies); the
    timeout is then visible through read_device_status."""
    _check(lib().spot_check_wait_timeout(_ptr(workspace, name="workspace"), _stream(stream)),
           "check_wait_timeout")


def read_device_status(workspace, stream=None) -> int:
    """Status recorded by kernels since the last read (0 = ok); clears it."""
    return int(lib().spot_read_device_status(_ptr(workspace, name="workspace"), _stream(stream)))


# ---------------------------------------------------------------- helpers

def selector_pool(fmt: str, num_pages: int, num_kv_heads: int, sel_dim: int = 64, device="cuda"):
    """Empty selector pool (data, scales) for a format."""
    if fmt == "bf16":
        return (torch.zeros(num_pages, num_kv_heads, sel_dim, dtype=torch.bfloat16, device=device),
                None)
    if fmt == "fp8":
        return (torch.zeros(num_pages, num_kv_heads, sel_dim, dtype=torch.uint8, device=device),
                None)
    if fmt == "int8":
        return (torch.zeros(num_pages, num_kv_heads, sel_dim, dtype=torch.int8, device=device),
                torch.zeros(num_pages, num_kv_heads, 1, dtype=torch.float16, device=device))
    data = torch.zeros(num_pages, num_kv_heads, sel_dim // 2, dtype=torch.uint8, device=device)
    sdt = torch.float16 if fmt == "int4" else torch.uint8
    return data, torch.zeros(num_pages, num_kv_heads, sel_dim // 32, dtype=sdt, device=device)


def selector_bytes_per_element(fmt: str) -> float:
    """Stored bits / 8 per selector-key element, scales included."""
    return {"bf16": 2.0, "int4": (4 + 16 / 32) / 8, "mxfp4": (4 + 8 / 32) / 8, "fp8": 1.0,
            "int8": (8 + 16 / 64) / 8}[fmt]
