"""fp64 CPU oracle for the SpotAttention decode hot path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module; the
product package never does.  It shares no code with the CUDA library: the C
source next to this file is compiled with gcc into ``liboracle.so`` and called
through ctypes with numpy arrays.

Source of every definition: "SpotAttention: Plug-In Block-Sparse Routing for
Pretrained Long-Context Transformers" (arXiv HTML), §2.1 (selector score),
§2.3 Eqs. 6-8 (block score, residual softmax, dual top-p with sink / recency
reservation and the K_min floor), §5.3 and App. G (group-32 INT4 / FP4
selector K-cache), App. A Tab. 3 (temperature 1.0).

bf16 tensors are passed as their uint16 bit patterns; the oracle widens each
value exactly to fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spot_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

FMT = {"bf16": 0, "int4": 1, "mxfp4": 2, "fp8": 3, "int8": 4}
MODE = {"topp": 0, "topk": 1}
_FMT_NAME = {v: k for k, v in FMT.items()}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain IEEE fp64: no fast-math, no FMA
    contraction) and OpenMP; returns the library path."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "num_kv_heads", "head_dim", "block_size", "sel_dim",
        "sel_fmt", "num_pages", "max_blocks")]


class Params(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("sink_blocks", ctypes.c_int32),
                ("recency_blocks", ctypes.c_int32), ("kmin_blocks", ctypes.c_int32),
                ("topk_blocks", ctypes.c_int32), ("temperature", ctypes.c_double),
                ("quantize_queries", ctypes.c_int32)]


class TokShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "num_kv_heads", "head_dim", "page_size", "idx_heads", "idx_dim",
        "sel_block", "num_pages", "max_pages", "max_blocks", "sel_fmt")]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_dequant_selector.argtypes = [ctypes.c_int, i64, ctypes.c_int, P, P, P]
        lib.oracle_quantize_selector.argtypes = [ctypes.c_int, i64, ctypes.c_int, P, P, P]
        lib.oracle_block_scores.argtypes = [P, P, P, P, P, P, P, P, P]
        lib.oracle_select_from_scores.argtypes = [P, i32, i32, P, dbl, P, P]
        lib.oracle_select_from_scores.restype = i32
        lib.oracle_sparse_attention.argtypes = [P, P, P, P, P, P, P, P, dbl, P, P]
        lib.oracle_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, dbl, P, i32,
                                           P, P, P, P, P]
        lib.oracle_tok_block_scores.argtypes = [P, P, P, P, P, P, P, P, P]
        lib.oracle_tok_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, dbl, P, i32,
                                               P, P, P, P, P]
        lib.oracle_prefill_num_tiles.argtypes = [P, P, P]
        lib.oracle_prefill_num_tiles.restype = i64
        lib.oracle_prefill_scores.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, P]
        lib.oracle_prefill_step.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, dbl, P, i32,
                                            P, P, P, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> int:
    """Threads for later oracle calls; returns the count in effect."""
    return int(_load().oracle_set_num_threads(int(n)))


def make_shape(batch, num_q_heads, num_kv_heads, head_dim, block_size, sel_dim, sel_fmt,
               num_pages, max_blocks) -> Shape:
    return Shape(batch, num_q_heads, num_kv_heads, head_dim, block_size, sel_dim,
                 FMT[sel_fmt] if isinstance(sel_fmt, str) else sel_fmt, num_pages, max_blocks)


def make_params(mode="topp", sink_blocks=1, recency_blocks=4, kmin_blocks=8, topk_blocks=0,
                temperature=1.0, quantize_queries=False) -> Params:
    return Params(MODE[mode] if isinstance(mode, str) else mode, sink_blocks, recency_blocks,
                  kmin_blocks, topk_blocks, float(temperature), 1 if quantize_queries else 0)


def _data_dtype(fmt):
    return {"bf16": np.uint16, "int8": np.int8}.get(fmt, np.uint8)


def _scale_dtype(fmt):
    return np.uint16 if fmt in ("int4", "int8") else np.uint8


def _row_elems(fmt, ds):
    return {"bf16": ds, "fp8": ds, "int8": ds}.get(fmt, ds // 2)


def _scales_per_row(fmt, ds):
    return {"int4": ds // 32, "mxfp4": ds // 32, "int8": 1}.get(fmt, 0)


def dequant_selector(fmt: str, data: np.ndarray, scales, ds: int) -> np.ndarray:
    """Exact fp64 values of selector keys stored as `fmt` ([rows, ds])."""
    rows = data.size // _row_elems(fmt, ds)
    data = _c(data, _data_dtype(fmt))
    if scales is not None:
        scales = _c(scales, _scale_dtype(fmt))
    out = np.empty((rows, ds), np.float64)
    rc = _load().oracle_dequant_selector(FMT[fmt], rows, ds, _ptr(data), _ptr(scales), _ptr(out))
    assert rc == 0
    return out


def quantize_selector(fmt: str, keys_bits: np.ndarray):
    """Quantise bf16 keys (uint16 bit patterns, [..., ds]) -> (data, scales)."""
    ds = keys_bits.shape[-1]
    lead = keys_bits.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    keys = _c(keys_bits, np.uint16)
    data = np.empty(lead + (_row_elems(fmt, ds),), _data_dtype(fmt))
    nsc = _scales_per_row(fmt, ds)
    scales = np.empty(lead + (nsc,), _scale_dtype(fmt)) if nsc else None
    rc = _load().oracle_quantize_selector(FMT[fmt], rows, ds, _ptr(keys), _ptr(data),
                                          _ptr(scales))
    assert rc == 0
    return data, scales


def select_from_scores(scores, nb=None, n_full=None, params=None, p=0.9):
    """Selection for one (sequence, KV head) -> (ascending block ids, nucleus mass)."""
    s = _c(scores, np.float64)
    nb = s.size if nb is None else nb
    n_full = nb if n_full is None else n_full
    params = params or make_params()
    sel = np.empty(max(nb, 1), np.int32)
    mass = ctypes.c_double(0.0)
    cnt = _load().oracle_select_from_scores(_ptr(s), nb, n_full, ctypes.byref(params), float(p),
                                            _ptr(sel), ctypes.byref(mass))
    return sel[:cnt].copy(), mass.value


def block_scores(shape: Shape, params: Params, q_sel, w, sel_data, sel_scales, page_table,
                 seq_lens) -> np.ndarray:
    """Selector block scores [B, Hkv, max_blocks] (NaN where no complete block)."""
    scores = np.full((shape.batch, shape.num_kv_heads, shape.max_blocks), np.nan)
    fmt = shape.sel_fmt
    rc = _load().oracle_block_scores(
        ctypes.byref(shape), ctypes.byref(params), _ptr(_c(q_sel, np.uint16)),
        _ptr(_c(w, np.float32)), _ptr(_c(sel_data, _data_dtype(_FMT_NAME[fmt]))),
        _ptr(_c(sel_scales, _scale_dtype(_FMT_NAME[fmt]))),
        _ptr(_c(page_table, np.int32)), _ptr(_c(seq_lens, np.int32)), _ptr(scores))
    assert rc == 0
    return scores


def sparse_attention(shape: Shape, q, k_pool, v_pool, page_table, seq_lens, sel_idx, sel_cnt,
                     sm_scale):
    """Exact attention over given block selections -> (out [B,Hq,D], lse [B,Hq])."""
    out = np.zeros((shape.batch, shape.num_q_heads, shape.head_dim))
    lse = np.zeros((shape.batch, shape.num_q_heads))
    _load().oracle_sparse_attention(
        ctypes.byref(shape), _ptr(_c(q, np.uint16)), _ptr(_c(k_pool, np.uint16)),
        _ptr(_c(v_pool, np.uint16)), _ptr(_c(page_table, np.int32)),
        _ptr(_c(seq_lens, np.int32)), _ptr(_c(sel_idx, np.int32)), _ptr(_c(sel_cnt, np.int32)),
        float(sm_scale), _ptr(out), _ptr(lse))
    return out, lse


def decode_step(shape: Shape, params: Params, q_sel, w, sel_data, sel_scales, q, k_pool, v_pool,
                page_table, seq_lens, top_p, sm_scale, units=None):
    """Whole decode step (scores, selection, attention) for `units` (list of
    b*Hkv+g, default all).  Entries of units not listed are left at zero."""
    B, Hkv, Hq = shape.batch, shape.num_kv_heads, shape.num_q_heads
    sel_idx = np.full((B, Hkv, max(shape.max_blocks, 1)), -1, np.int32)
    sel_cnt = np.zeros((B, Hkv), np.int32)
    mass = np.zeros((B, Hkv))
    out = np.zeros((B, Hq, shape.head_dim))
    lse = np.zeros((B, Hq))
    fmt = shape.sel_fmt
    u = None if units is None else _c(units, np.int32)
    rc = _load().oracle_decode_step(
        ctypes.byref(shape), ctypes.byref(params), _ptr(_c(q_sel, np.uint16)),
        _ptr(_c(w, np.float32)), _ptr(_c(sel_data, _data_dtype(_FMT_NAME[fmt]))),
        _ptr(_c(sel_scales, _scale_dtype(_FMT_NAME[fmt]))), _ptr(_c(q, np.uint16)),
        _ptr(_c(k_pool, np.uint16)), _ptr(_c(v_pool, np.uint16)), _ptr(_c(page_table, np.int32)),
        _ptr(_c(seq_lens, np.int32)), _ptr(_c(top_p, np.float32)), float(sm_scale), _ptr(u),
        0 if u is None else len(u), _ptr(sel_idx), _ptr(sel_cnt), _ptr(mass), _ptr(out),
        _ptr(lse))
    assert rc == 0
    return {"sel_idx": sel_idx, "sel_cnt": sel_cnt, "nuc_mass": mass, "out": out, "lse": lse}


# ---------------------------------------------------------------------------
# Token-level, layer-shared selector (§2.1 / §2.3 / App. A Tab. 3 as written)

def make_tok_shape(batch, num_q_heads, num_kv_heads, num_pages, max_pages, head_dim=128,
                   page_size=64, idx_heads=4, idx_dim=128, sel_block=16,
                   max_blocks=None, sel_fmt="bf16") -> TokShape:
    mb = max_pages * (page_size // sel_block) if max_blocks is None else max_blocks
    return TokShape(batch, num_q_heads, num_kv_heads, head_dim, page_size, idx_heads, idx_dim,
                    sel_block, num_pages, max_pages, mb,
                    FMT[sel_fmt] if isinstance(sel_fmt, str) else sel_fmt)


def _tok_pool(shape, sel_tok, sel_scales):
    fmt = _FMT_NAME[shape.sel_fmt]
    return (_c(sel_tok, _data_dtype(fmt)),
            None if sel_scales is None else _c(sel_scales, _scale_dtype(fmt)))


def tok_block_scores(shape: TokShape, params: Params, q_idx, w, sel_tok, page_table,
                     seq_lens, sel_scales=None) -> np.ndarray:
    """Block scores [B, max_blocks] of the token-level selector (max over
    each block's token scores; NaN where no complete block).  sel_tok /
    sel_scales: the per-token key pool in the shape's format."""
    scores = np.full((shape.batch, shape.max_blocks), np.nan)
    data, scales = _tok_pool(shape, sel_tok, sel_scales)
    rc = _load().oracle_tok_block_scores(
        ctypes.byref(shape), ctypes.byref(params), _ptr(_c(q_idx, np.uint16)),
        _ptr(_c(w, np.float32)), _ptr(data), _ptr(scales), _ptr(_c(page_table, np.int32)),
        _ptr(_c(seq_lens, np.int32)), _ptr(scores))
    assert rc == 0
    return scores


def tok_decode_step(shape: TokShape, params: Params, q_idx, w, sel_tok, q, k_pool, v_pool,
                    page_table, seq_lens, top_p, sm_scale, seqs=None, sel_scales=None):
    """Decode step of the token-level selector for sequences `seqs` (default
    all): one selection per sequence shared by every head."""
    B, Hq = shape.batch, shape.num_q_heads
    sel_idx = np.full((B, max(shape.max_blocks, 1)), -1, np.int32)
    sel_cnt = np.zeros(B, np.int32)
    mass = np.zeros(B)
    out = np.zeros((B, Hq, shape.head_dim))
    lse = np.zeros((B, Hq))
    sq = None if seqs is None else _c(seqs, np.int32)
    data, scales = _tok_pool(shape, sel_tok, sel_scales)
    rc = _load().oracle_tok_decode_step(
        ctypes.byref(shape), ctypes.byref(params), _ptr(_c(q_idx, np.uint16)),
        _ptr(_c(w, np.float32)), _ptr(data), _ptr(scales), _ptr(_c(q, np.uint16)),
        _ptr(_c(k_pool, np.uint16)), _ptr(_c(v_pool, np.uint16)), _ptr(_c(page_table, np.int32)),
        _ptr(_c(seq_lens, np.int32)), _ptr(_c(top_p, np.float32)), float(sm_scale), _ptr(sq),
        0 if sq is None else len(sq), _ptr(sel_idx), _ptr(sel_cnt), _ptr(mass), _ptr(out),
        _ptr(lse))
    assert rc == 0
    return {"sel_idx": sel_idx, "sel_cnt": sel_cnt, "nuc_mass": mass, "out": out, "lse": lse}


# ---------------------------------------------------------------------------
# Sparse prefill (§2.3 applied to a chunk of queries; tiles of one KV block)

def prefill_tiles(seq_lens, q_lens, block_size=64):
    """(b, first position, last position, first row) of every query tile."""
    out, row = [], 0
    for b, (L, T) in enumerate(zip(np.asarray(seq_lens).tolist(), np.asarray(q_lens).tolist())):
        if T <= 0:
            continue
        q0 = L - T
        for m in range(q0 // block_size, (L - 1) // block_size + 1):
            lo, hi = max(q0, m * block_size), min(L - 1, m * block_size + block_size - 1)
            out.append((b, lo, hi, row + lo - q0))
        row += T
    return out


def prefill_scores(shape: Shape, params: Params, q_sel, w, sel_data, sel_scales, page_table,
                   seq_lens, q_lens, tiles=None) -> np.ndarray:
    """Block scores [tiles, Hkv, max_blocks] of the query tiles (max over
    the tile's queries; NaN where no complete block or tile not listed)."""
    lens, ql = _c(seq_lens, np.int32), _c(q_lens, np.int32)
    nt = int(_load().oracle_prefill_num_tiles(ctypes.byref(shape), _ptr(lens), _ptr(ql)))
    scores = np.full((max(nt, 1), shape.num_kv_heads, shape.max_blocks), np.nan)
    fmt = shape.sel_fmt
    tl = None if tiles is None else _c(tiles, np.int32)
    rc = _load().oracle_prefill_scores(
        ctypes.byref(shape), ctypes.byref(params), _ptr(_c(q_sel, np.uint16)),
        _ptr(_c(w, np.float32)), _ptr(_c(sel_data, _data_dtype(_FMT_NAME[fmt]))),
        _ptr(_c(sel_scales, _scale_dtype(_FMT_NAME[fmt]))), _ptr(_c(page_table, np.int32)),
        _ptr(lens), _ptr(ql), _ptr(tl), 0 if tl is None else len(tl), _ptr(scores))
    assert rc == 0
    return scores[:nt]


def prefill_step(shape: Shape, params: Params, q_sel, w, sel_data, sel_scales, q, k_pool, v_pool,
                 page_table, seq_lens, q_lens, top_p, sm_scale, tiles=None):
    """Sparse prefill of the chunks' query rows (packed [rows, Hq, ...]):
    selection per (tile, KV head) and causal attention over it.  `tiles`
    restricts the work to some tiles (their rows of out / lse are filled)."""
    lens, ql = _c(seq_lens, np.int32), _c(q_lens, np.int32)
    nt = int(_load().oracle_prefill_num_tiles(ctypes.byref(shape), _ptr(lens), _ptr(ql)))
    rows = int(np.maximum(ql, 0).sum())
    Hkv, Hq = shape.num_kv_heads, shape.num_q_heads
    sel_idx = np.full((max(nt, 1), Hkv, max(shape.max_blocks, 1)), -1, np.int32)
    sel_cnt = np.zeros((max(nt, 1), Hkv), np.int32)
    out = np.zeros((max(rows, 1), Hq, shape.head_dim))
    lse = np.zeros((max(rows, 1), Hq))
    fmt = shape.sel_fmt
    tl = None if tiles is None else _c(tiles, np.int32)
    rc = _load().oracle_prefill_step(
        ctypes.byref(shape), ctypes.byref(params), _ptr(_c(q_sel, np.uint16)),
        _ptr(_c(w, np.float32)), _ptr(_c(sel_data, _data_dtype(_FMT_NAME[fmt]))),
        _ptr(_c(sel_scales, _scale_dtype(_FMT_NAME[fmt]))), _ptr(_c(q, np.uint16)),
        _ptr(_c(k_pool, np.uint16)), _ptr(_c(v_pool, np.uint16)), _ptr(_c(page_table, np.int32)),
        _ptr(lens), _ptr(ql), _ptr(_c(top_p, np.float32)), float(sm_scale), _ptr(tl),
        0 if tl is None else len(tl), _ptr(sel_idx), _ptr(sel_cnt), _ptr(out), _ptr(lse))
    assert rc == 0
    return {"sel_idx": sel_idx[:nt], "sel_cnt": sel_cnt[:nt], "out": out[:rows], "lse": lse[:rows],
            "tiles": prefill_tiles(lens, ql, shape.block_size)}
