"""Shared helpers of the GPU parity tests: run a workload through the CUDA
library (C ABI via the Python binding) and through the fp64 oracle, and
compare them under the parity rules.

Parity rules (tolerances of the bf16-in / fp32-accumulate path):
  * selection: on integer-valued inputs the selected sets must be identical;
    on real-valued inputs every block whose oracle score lies more than 1e-6
    (relative) from the cut -- the lowest score the oracle kept in the
    nucleus -- must be treated identically, and any differing block must
    leave the GPU's set valid in fp64: nucleus mass >= p - 1e-5 and the mass
    without its lowest-ranked block < p + 1e-5;
  * attention outputs: |gpu - oracle| <= 2e-3 + 1e-2 |oracle| element-wise,
    for every (sequence, KV head) whose selection matches exactly.
"""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_long_spot_b200 as spot
import oracle
import workloads

ATOL, RTOL = 2e-3, 1e-2
CUT_REL = 1e-6
MASS_TOL = 1e-5


def gpu_selector_pool(wl, fmt, device):
    """Selector pool in `fmt`, written by the library's append kernel."""
    data, scales = spot.selector_pool(fmt, wl.num_pages, wl.num_kv_heads, device=device)
    pt = wl.page_table
    lens = wl.seq_lens.cpu().numpy()
    seq_ids, blk_ids, pages = [], [], []
    ptn = pt.cpu().numpy()
    for b in range(wl.batch):
        nb = int(lens[b]) // 64               # complete blocks carry keys
        for j in range(nb):
            if 0 <= ptn[b, j] < wl.num_pages:   # a test may corrupt an entry on purpose
                seq_ids.append(b)
                blk_ids.append(j)
                pages.append(int(ptn[b, j]))
    if seq_ids:
        keys = wl.sel_keys[torch.as_tensor(pages, device=device).long()].contiguous()
        desc = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, fmt)
        spot.append_selector_keys(desc, data, scales, pt,
                                  torch.as_tensor(seq_ids, dtype=torch.int32, device=device),
                                  torch.as_tensor(blk_ids, dtype=torch.int32, device=device), keys)
    return data, scales


def oracle_selector_pool(wl, fmt):
    return oracle.quantize_selector(fmt, workloads.bits(wl.sel_keys))


def host_bytes(t):
    if t is None:
        return None
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def run_gpu(wl, fmt="bf16", mode="topp", kmin=None, topk=0, sink=None, rec=None,
            temperature=1.0, pool=None, max_blocks=None, quantize_queries=False):
    dev = wl.q.device
    B, Hq, Hkv = wl.batch, wl.num_q_heads, wl.num_kv_heads
    mb = wl.max_blocks if max_blocks is None else max_blocks
    desc = spot.layer_desc(Hq, Hkv, wl.num_pages, fmt)
    prm = spot.select_params(mode, wl.spec.sink_blocks if sink is None else sink,
                             wl.spec.recency_blocks if rec is None else rec,
                             wl.spec.kmin_blocks if kmin is None else kmin, topk, temperature,
                             quantize_queries)
    data, scales = pool if pool is not None else gpu_selector_pool(wl, fmt, dev)
    ws = spot.new_workspace(desc, B, mb, dev)
    sel_idx = torch.full((B, Hkv, mb), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.full((B, Hkv), -1, dtype=torch.int32, device=dev)
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=dev)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
    spot.decode_step(desc, prm, wl.q_sel, wl.w, data, scales, wl.q, wl.k_pool, wl.v_pool,
                     wl.page_table, wl.seq_lens, wl.top_p, wl.sm_scale, sel_idx, sel_cnt, out, lse,
                     ws)
    torch.cuda.synchronize()
    status = spot.read_device_status(ws)
    return {"sel_idx": sel_idx.cpu().numpy(), "sel_cnt": sel_cnt.cpu().numpy(),
            "out": out.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
            "status": status, "pool": (data, scales)}


def oracle_args(wl, fmt="bf16"):
    data, scales = oracle_selector_pool(wl, fmt)
    return dict(q_sel=workloads.bits(wl.q_sel), w=host_bytes(wl.w), sel_data=data,
                sel_scales=scales, q=workloads.bits(wl.q), k_pool=workloads.bits(wl.k_pool),
                v_pool=workloads.bits(wl.v_pool), page_table=wl.page_table.cpu().numpy(),
                seq_lens=wl.seq_lens.cpu().numpy(), top_p=wl.top_p.cpu().numpy(),
                sm_scale=wl.sm_scale)


def oracle_shape_params(wl, fmt="bf16", mode="topp", kmin=None, topk=0, sink=None, rec=None,
                        temperature=1.0, max_blocks=None, quantize_queries=False):
    sh = oracle.make_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, 128, 64, 64, fmt,
                           wl.num_pages, wl.max_blocks if max_blocks is None else max_blocks)
    pr = oracle.make_params(mode, wl.spec.sink_blocks if sink is None else sink,
                            wl.spec.recency_blocks if rec is None else rec,
                            wl.spec.kmin_blocks if kmin is None else kmin, topk, temperature,
                            quantize_queries)
    return sh, pr


def run_oracle(wl, fmt="bf16", units=None, args=None, **kw):
    sh, pr = oracle_shape_params(wl, fmt, **kw)
    a = args or oracle_args(wl, fmt)
    if kw.get("max_blocks") is not None and kw["max_blocks"] != wl.max_blocks:
        pt = np.full((wl.batch, kw["max_blocks"]), -1, np.int32)
        pt[:, :wl.max_blocks] = a["page_table"]
        a = dict(a, page_table=pt)
    return oracle.decode_step(sh, pr, units=units, **a)


def oracle_scores(wl, fmt="bf16", args=None, **kw):
    sh, pr = oracle_shape_params(wl, fmt, **kw)
    a = args or oracle_args(wl, fmt)
    return oracle.block_scores(sh, pr, a["q_sel"], a["w"], a["sel_data"], a["sel_scales"],
                               a["page_table"], a["seq_lens"])


def unit_selection(res, b, g):
    return res["sel_idx"][b, g, :res["sel_cnt"][b, g]].tolist()


def _reserved_residual(L, bsz, sink, rec):
    """Reserved (sink / recency, incomplete last block) and residual block
    ids of a sequence of L tokens in blocks of bsz."""
    nb, n_full = (L + bsz - 1) // bsz, L // bsz
    r_eff = min(max(rec, nb - n_full), nb)
    s_eff = min(sink, nb)
    reserved = set(range(s_eff)) | set(range(nb - r_eff, nb))
    return reserved, [j for j in range(nb) if j not in reserved]


def _unit_near_cut(sg, so, s, reserved, res, p, kmin, where):
    """Check one unit's GPU set sg against the oracle's so under the
    real-valued rule; returns 1 if they differ (all near the cut), else 0."""
    assert reserved <= sg, where
    if sg == so:
        return 0
    nuc_o = so - reserved
    assert nuc_o, where
    cut = min(s[j] for j in nuc_o)
    for j in sg ^ so:
        assert j in res, (where, j)
        assert abs(s[j] - cut) <= CUT_REL * abs(cut) + 1e-12, (where, j, s[j], cut)
    # the GPU set is itself a valid nucleus in fp64
    sr = np.array([s[j] for j in res])
    e = np.exp(sr - sr.max())
    e /= e.sum()
    mass = {j: e[i] for i, j in enumerate(res)}
    nuc_g = sorted(sg - reserved, key=lambda j: (-s[j], j))
    if len(nuc_g) > max(kmin - len(reserved), 0):
        m_g = sum(mass[j] for j in nuc_g)
        assert m_g >= p - MASS_TOL, (where, m_g, p)
        assert m_g - mass[nuc_g[-1]] < p + MASS_TOL, (where, m_g, p)
    return 1


def check_selection_near_cut(gpu, ora, scores, wl, kmin=None, sink=None, rec=None):
    """Apply the real-valued selection rule to every unit; return the number
    of (sequence, KV head) units whose sets differ (all near the cut)."""
    kmin = wl.spec.kmin_blocks if kmin is None else kmin
    sink = wl.spec.sink_blocks if sink is None else sink
    rec = wl.spec.recency_blocks if rec is None else rec
    lens = wl.seq_lens.cpu().numpy()
    p_all = wl.top_p.cpu().numpy()
    n_diff = 0
    for b in range(wl.batch):
        reserved, res = _reserved_residual(int(lens[b]), 64, sink, rec)
        for g in range(wl.num_kv_heads):
            n_diff += _unit_near_cut(set(unit_selection(gpu, b, g)), set(unit_selection(ora, b, g)),
                                     scores[b, g], reserved, res, float(p_all[b]), kmin, (b, g))
    return n_diff


def check_outputs(gpu, ora, wl, units=None):
    """Element-wise output check on units whose selections agree; returns
    (max abs err, max rel err, units compared)."""
    G = wl.num_q_heads // wl.num_kv_heads
    if units is None:
        units = [(b, g) for b in range(wl.batch) for g in range(wl.num_kv_heads)]
    worst_a, worst_r, n = 0.0, 0.0, 0
    for b, g in units:
        if unit_selection(gpu, b, g) != unit_selection(ora, b, g):
            continue
        o_g = gpu["out"][b, g * G:(g + 1) * G]
        o_r = ora["out"][b, g * G:(g + 1) * G]
        err = np.abs(o_g - o_r)
        bad = err > ATOL + RTOL * np.abs(o_r)
        assert not bad.any(), (b, g, float(err.max()))
        l_g = gpu["lse"][b, g * G:(g + 1) * G]
        l_r = ora["lse"][b, g * G:(g + 1) * G]
        fin = np.isfinite(l_r)
        assert np.array_equal(fin, np.isfinite(l_g)), (b, g)
        assert (np.abs(l_g[fin] - l_r[fin]) <= ATOL + RTOL * np.abs(l_r[fin])).all(), (b, g)
        worst_a = max(worst_a, float(err.max()))
        worst_r = max(worst_r, float((err / np.maximum(np.abs(o_r), 1e-3)).max()))
        n += 1
    return worst_a, worst_r, n


def safe_top_p(wl, fmt="bf16", lo=0.5, hi=0.99, margin=2e-5, **kw):
    """Per-sequence p values at least `margin` away from every cumulative
    residual mass of every KV head of that sequence (from the oracle's own
    scores), so the nucleus size is decided far from the fp boundary."""
    scores = oracle_scores(wl, fmt, **kw)
    lens = wl.seq_lens.cpu().numpy()
    sink, rec = wl.spec.sink_blocks, wl.spec.recency_blocks
    ps = []
    for b in range(wl.batch):
        nb, n_full = (int(lens[b]) + 63) // 64, int(lens[b]) // 64
        r_eff = min(max(rec, nb - n_full), nb)
        res = list(range(min(sink, nb), max(min(sink, nb), nb - r_eff)))
        cums = [lo, hi]
        for g in range(wl.num_kv_heads):
            s = np.array([scores[b, g, j] for j in res])
            if s.size == 0:
                continue
            order = sorted(range(len(res)), key=lambda i: (-s[i], res[i]))
            e = np.exp(s - s.max())
            e /= e.sum()
            cums += np.cumsum(e[order]).tolist()
        c = np.unique(np.clip(np.array(cums), lo, hi))
        gaps = np.diff(c)
        k = int(np.argmax(gaps))
        assert gaps[k] > 2 * margin
        ps.append(0.5 * (c[k] + c[k + 1]))
    return torch.as_tensor(np.array(ps, np.float32), device=wl.top_p.device)


# ------------------------------------------------ token-level, layer-shared selector

def _tok_sel(spec, kmin, sink, rec):
    return (spec.kmin_blocks if kmin is None else kmin, spec.sink_blocks if sink is None else sink,
            spec.recency_blocks if rec is None else rec)


def gpu_tok_pool(wl, fmt, desc):
    """Per-token selector pool in `fmt`, written by the library's append
    kernel from the workload's bf16 keys (every cached token)."""
    dev = wl.q.device
    if fmt == "bf16":
        return wl.sel_tok, None
    data, scales = spot.tok_selector_pool(wl.num_pages, fmt, device=dev)
    lens = wl.seq_lens.cpu().numpy()
    pt = wl.page_table.cpu().numpy()
    seq = np.concatenate([np.full(int(L), b) for b, L in enumerate(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(int(L)) for L in lens]).astype(np.int32)
    if seq.size == 0:
        return data, scales
    pages = torch.as_tensor(pt[seq, pos // 64].astype(np.int64), device=dev)
    keys = wl.sel_tok[pages, torch.as_tensor(pos % 64, device=dev).long()].contiguous()
    spot.tok_append_selector_keys(desc, data, scales, wl.page_table,
                                  torch.as_tensor(seq, device=dev), torch.as_tensor(pos, device=dev),
                                  keys)
    torch.cuda.synchronize()
    return data, scales


def run_gpu_tok(wl, mode="topp", kmin=None, topk=0, sink=None, rec=None, temperature=1.0,
                max_blocks=None, pool=None, fmt="bf16", quantize_queries=False):
    dev = wl.q.device
    B, Hq, Hkv = wl.batch, wl.num_q_heads, wl.num_kv_heads
    mb = wl.max_blocks if max_blocks is None else max_blocks
    kmin, sink, rec = _tok_sel(wl.spec, kmin, sink, rec)
    desc = spot.tok_layer_desc(Hq, Hkv, wl.num_pages, sel_fmt=fmt)
    data, scales = gpu_tok_pool(wl, fmt, desc) if pool is None else pool
    prm = spot.select_params(mode, sink, rec, kmin, topk, temperature, quantize_queries)
    ws = spot.new_tok_workspace(desc, B, mb, dev)
    sel_idx = torch.full((B, mb), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.full((B,), -1, dtype=torch.int32, device=dev)
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=dev)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
    spot.tok_decode_step(desc, prm, wl.q_idx, wl.w_idx, data, scales, wl.q, wl.k_pool, wl.v_pool,
                         wl.page_table, wl.seq_lens, wl.top_p, wl.sm_scale, sel_idx, sel_cnt, out,
                         lse, ws)
    torch.cuda.synchronize()
    status = spot.read_device_status(ws)
    return {"sel_idx": sel_idx.cpu().numpy(), "sel_cnt": sel_cnt.cpu().numpy(),
            "out": out.cpu().double().numpy(), "lse": lse.cpu().double().numpy(),
            "status": status}


def tok_oracle_args(wl, fmt="bf16"):
    bits = workloads.bits(wl.sel_tok)
    if fmt == "bf16":
        data, scales = bits, None
    else:
        data, scales = oracle.quantize_selector(fmt, bits)
    return dict(q_idx=workloads.bits(wl.q_idx), w=host_bytes(wl.w_idx),
                sel_tok=data, sel_scales=scales, q=workloads.bits(wl.q),
                k_pool=workloads.bits(wl.k_pool), v_pool=workloads.bits(wl.v_pool),
                page_table=wl.page_table.cpu().numpy(), seq_lens=wl.seq_lens.cpu().numpy(),
                top_p=wl.top_p.cpu().numpy(), sm_scale=wl.sm_scale)


def tok_oracle_shape_params(wl, mode="topp", kmin=None, topk=0, sink=None, rec=None,
                            temperature=1.0, max_blocks=None, fmt="bf16", quantize_queries=False):
    kmin, sink, rec = _tok_sel(wl.spec, kmin, sink, rec)
    sh = oracle.make_tok_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.num_pages,
                               wl.max_pages, max_blocks=wl.max_blocks if max_blocks is None
                               else max_blocks, sel_fmt=fmt)
    pr = oracle.make_params(mode, sink, rec, kmin, topk, temperature, quantize_queries)
    return sh, pr


def run_oracle_tok(wl, seqs=None, args=None, **kw):
    sh, pr = tok_oracle_shape_params(wl, **kw)
    a = args or tok_oracle_args(wl, kw.get("fmt", "bf16"))
    return oracle.tok_decode_step(sh, pr, seqs=seqs, **a)


def oracle_tok_scores(wl, args=None, **kw):
    sh, pr = tok_oracle_shape_params(wl, **kw)
    a = args or tok_oracle_args(wl, kw.get("fmt", "bf16"))
    return oracle.tok_block_scores(sh, pr, a["q_idx"], a["w"], a["sel_tok"], a["page_table"],
                                   a["seq_lens"], sel_scales=a["sel_scales"])


def tok_selection(res, b):
    return res["sel_idx"][b, :res["sel_cnt"][b]].tolist()


def check_tok_selection_near_cut(gpu, ora, scores, wl, seqs=None, kmin=None, sink=None,
                                 rec=None):
    """The real-valued selection rule per sequence; returns how many
    sequences' shared selections differ (all near the cut)."""
    kmin, sink, rec = _tok_sel(wl.spec, kmin, sink, rec)
    lens = wl.seq_lens.cpu().numpy()
    p_all = wl.top_p.cpu().numpy()
    n_diff = 0
    for b in (range(wl.batch) if seqs is None else seqs):
        reserved, res = _reserved_residual(int(lens[b]), wl.spec.sel_block, sink, rec)
        n_diff += _unit_near_cut(set(tok_selection(gpu, b)), set(tok_selection(ora, b)),
                                 scores[b], reserved, res, float(p_all[b]), kmin, b)
    return n_diff


def check_tok_outputs(gpu, ora, wl, seqs=None):
    """Element-wise output check of every head of the sequences whose
    selections agree; returns (max abs err, sequences compared)."""
    worst, n = 0.0, 0
    for b in (range(wl.batch) if seqs is None else seqs):
        if tok_selection(gpu, b) != tok_selection(ora, b):
            continue
        err = np.abs(gpu["out"][b] - ora["out"][b])
        bad = err > ATOL + RTOL * np.abs(ora["out"][b])
        assert not bad.any(), (b, float(err.max()))
        fin = np.isfinite(ora["lse"][b])
        assert np.array_equal(fin, np.isfinite(gpu["lse"][b])), b
        assert (np.abs(gpu["lse"][b][fin] - ora["lse"][b][fin]) <=
                ATOL + RTOL * np.abs(ora["lse"][b][fin])).all(), b
        worst = max(worst, float(err.max()))
        n += 1
    return worst, n


def safe_top_p_tok(wl, lo=0.5, hi=0.99, margin=2e-5, **kw):
    """Per-sequence p at least `margin` from every cumulative residual mass."""
    scores = oracle_tok_scores(wl, **kw)
    kmin, sink, rec = _tok_sel(wl.spec, kw.get("kmin"), kw.get("sink"), kw.get("rec"))
    lens = wl.seq_lens.cpu().numpy()
    ps = []
    for b in range(wl.batch):
        _, res = _reserved_residual(int(lens[b]), wl.spec.sel_block, sink, rec)
        cums = [lo, hi]
        if res:
            s = np.array([scores[b, j] for j in res])
            order = sorted(range(len(res)), key=lambda i: (-s[i], res[i]))
            e = np.exp(s - s.max())
            e /= e.sum()
            cums += np.cumsum(e[order]).tolist()
        c = np.unique(np.clip(np.array(cums), lo, hi))
        gaps = np.diff(c)
        k = int(np.argmax(gaps))
        assert gaps[k] > 2 * margin
        ps.append(0.5 * (c[k] + c[k + 1]))
    return torch.as_tensor(np.array(ps, np.float32), device=wl.top_p.device)


# ------------------------------------------------------------------ sparse prefill

def _pf_sel(spec, kmin, sink, rec):
    return (spec.kmin_blocks if kmin is None else kmin, spec.sink_blocks if sink is None else sink,
            spec.recency_blocks if rec is None else rec)


def run_gpu_prefill(wl, mode="topp", kmin=None, topk=0, sink=None, rec=None, temperature=1.0,
                    max_tiles=None, fmt="bf16", quantize_queries=False):
    dev = wl.q.device
    Hq, Hkv, mb = wl.num_q_heads, wl.num_kv_heads, wl.max_blocks
    kmin, sink, rec = _pf_sel(wl.spec, kmin, sink, rec)
    nt = spot.prefill_num_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    mt = max(nt, 1) if max_tiles is None else max_tiles
    desc = spot.layer_desc(Hq, Hkv, wl.num_pages, fmt)
    prm = spot.select_params(mode, sink, rec, kmin, topk, temperature, quantize_queries)
    # bf16 keys as they are (a test may corrupt the page table on purpose, so
    # nothing here gathers through it); other formats through the append
    data, scales = (wl.sel_keys, None) if fmt == "bf16" else gpu_selector_pool(wl, fmt, dev)
    ws = spot.new_prefill_workspace(desc, wl.batch, mt, mb, dev)
    rows = int(wl.q.shape[0])
    sel_idx = torch.full((mt, Hkv, mb), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.full((mt, Hkv), -1, dtype=torch.int32, device=dev)
    out = torch.full((max(rows, 1), Hq, 128), float("nan"), dtype=torch.float32, device=dev)
    lse = torch.full((max(rows, 1), Hq), float("nan"), dtype=torch.float32, device=dev)
    spot.prefill(desc, prm, wl.q_sel, wl.w, data, scales, wl.q, wl.k_pool, wl.v_pool,
                 wl.page_table, wl.seq_lens, wl.q_lens, wl.top_p, wl.sm_scale, sel_idx, sel_cnt,
                 out, lse, ws)
    torch.cuda.synchronize()
    status = spot.read_device_status(ws)
    return {"sel_idx": sel_idx.cpu().numpy()[:nt], "sel_cnt": sel_cnt.cpu().numpy()[:nt],
            "out": out.cpu().double().numpy()[:rows], "lse": lse.cpu().double().numpy()[:rows],
            "status": status, "num_tiles": nt}


def prefill_oracle_args(wl, fmt="bf16"):
    data, scales = oracle_selector_pool(wl, fmt)
    return dict(q_sel=workloads.bits(wl.q_sel), w=host_bytes(wl.w),
                sel_data=data, sel_scales=scales, q=workloads.bits(wl.q),
                k_pool=workloads.bits(wl.k_pool), v_pool=workloads.bits(wl.v_pool),
                page_table=wl.page_table.cpu().numpy(), seq_lens=wl.seq_lens.cpu().numpy(),
                q_lens=wl.q_lens.cpu().numpy(), top_p=wl.top_p.cpu().numpy(),
                sm_scale=wl.sm_scale)


def prefill_shape_params(wl, mode="topp", kmin=None, topk=0, sink=None, rec=None,
                         temperature=1.0, fmt="bf16", quantize_queries=False):
    kmin, sink, rec = _pf_sel(wl.spec, kmin, sink, rec)
    sh = oracle.make_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, 128, 64, 64, fmt,
                           wl.num_pages, wl.max_blocks)
    return sh, oracle.make_params(mode, sink, rec, kmin, topk, temperature, quantize_queries)


def run_oracle_prefill(wl, tiles=None, args=None, **kw):
    sh, pr = prefill_shape_params(wl, **kw)
    return oracle.prefill_step(sh, pr, tiles=tiles,
                               **(args or prefill_oracle_args(wl, kw.get("fmt", "bf16"))))


def oracle_prefill_scores(wl, tiles=None, args=None, **kw):
    sh, pr = prefill_shape_params(wl, **kw)
    a = args or prefill_oracle_args(wl, kw.get("fmt", "bf16"))
    return oracle.prefill_scores(sh, pr, a["q_sel"], a["w"], a["sel_data"], a["sel_scales"],
                                 a["page_table"], a["seq_lens"], a["q_lens"], tiles=tiles)


def tile_selection(res, t, g):
    return res["sel_idx"][t, g, :res["sel_cnt"][t, g]].tolist()


def check_prefill_selection_near_cut(gpu, ora, scores, wl, tiles=None, kmin=None, sink=None,
                                     rec=None):
    """The real-valued rule per (tile, KV head); returns how many differ."""
    kmin, sink, rec = _pf_sel(wl.spec, kmin, sink, rec)
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    p_all = wl.top_p.cpu().numpy()
    n_diff = 0
    for t in (range(len(info)) if tiles is None else tiles):
        b, lo, hi, _ = info[t]
        reserved, res = _reserved_residual(hi + 1, 64, sink, rec)
        for g in range(wl.num_kv_heads):
            n_diff += _unit_near_cut(set(tile_selection(gpu, t, g)), set(tile_selection(ora, t, g)),
                                     scores[t, g], reserved, res, float(p_all[b]), kmin, (t, g))
    return n_diff


P_ROUND = 2.0 ** -9          # relative rounding of a softmax weight stored as bf16


def prefill_weighted_abs_v(wl, ora, t, g):
    """sum_i w_i |v_i| per (query row, head, dim) of tile t, KV head g, with
    w the exact (fp64) causal softmax weights over the tile's selected
    tokens: the scale of the error that rounding the weights to bf16 before
    P.V can cause (reading r21 of the design notes)."""
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    b, lo, hi, r0 = info[t]
    G = wl.num_q_heads // wl.num_kv_heads
    sel = ora["sel_idx"][t, g, :ora["sel_cnt"][t, g]]
    pt = wl.page_table[b].cpu().numpy()
    pos = np.concatenate([np.arange(j * 64, j * 64 + 64) for j in sel]) if len(sel) else \
        np.zeros(0, np.int64)
    pos = pos[pos <= hi]
    pages = torch.as_tensor(pt[pos // 64].astype(np.int64))
    rows_in = torch.as_tensor(pos % 64)
    k = wl.k_pool[pages.to(wl.k_pool.device), g, rows_in.to(wl.k_pool.device)].double().cpu()
    v = wl.v_pool[pages.to(wl.v_pool.device), g, rows_in.to(wl.v_pool.device)].double().cpu()
    q = wl.q[r0:r0 + hi - lo + 1, g * G:(g + 1) * G].double().cpu()      # [rows, G, D]
    logits = torch.einsum("rhd,kd->rhk", q, k) * wl.sm_scale
    qpos = torch.arange(lo, hi + 1)[:, None, None]
    logits = logits.masked_fill(torch.as_tensor(pos)[None, None, :] > qpos, float("-inf"))
    w = torch.softmax(logits, dim=-1).nan_to_num(0.0)
    return torch.einsum("rhk,kd->rhd", w, v.abs()).numpy()


def check_prefill_outputs(gpu, ora, wl, tiles=None):
    """Element-wise check of the query rows of every (tile, KV head) whose
    selections agree; returns (max abs err, units compared).

    Tolerance (reading r21): the attention kernel rounds the softmax weights
    to bf16 (relative 2^-9) before the P.V product and divides by the sum of
    the unrounded weights, so an output element can move by up to
    2^-9 * sum_i w_i |v_i| beyond the fp32 error the decode rule covers.  A
    decode row averages hundreds of tokens, where this stays far inside the
    2e-3 term; a prefill row near the start of a sequence may attend a
    handful, so that bound, computed per element from the exact weights, is
    added to the shared 2e-3 + 1e-2 |ref| rule."""
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    G = wl.num_q_heads // wl.num_kv_heads
    worst, n = 0.0, 0
    for t in (range(len(info)) if tiles is None else tiles):
        _, lo, hi, r0 = info[t]
        rows = slice(r0, r0 + hi - lo + 1)
        for g in range(wl.num_kv_heads):
            if tile_selection(gpu, t, g) != tile_selection(ora, t, g):
                continue
            hs = slice(g * G, (g + 1) * G)
            o_g, o_r = gpu["out"][rows, hs], ora["out"][rows, hs]
            err = np.abs(o_g - o_r)
            bound = ATOL + RTOL * np.abs(o_r) + P_ROUND * prefill_weighted_abs_v(wl, ora, t, g)
            assert not (err > bound).any(), (t, g, float(err.max()))
            l_g, l_r = gpu["lse"][rows, hs], ora["lse"][rows, hs]
            fin = np.isfinite(l_r)
            assert np.array_equal(fin, np.isfinite(l_g)), (t, g)
            assert (np.abs(l_g[fin] - l_r[fin]) <= ATOL + RTOL * np.abs(l_r[fin])).all(), (t, g)
            worst = max(worst, float(err.max()) if err.size else 0.0)
            n += 1
    return worst, n


def safe_top_p_prefill(wl, lo=0.5, hi=0.99, margin=2e-5, **kw):
    """Per-sequence p at least `margin` from every cumulative residual mass
    of every (tile, KV head) of that sequence."""
    kmin, sink, rec = _pf_sel(wl.spec, kw.get("kmin"), kw.get("sink"), kw.get("rec"))
    scores = oracle_prefill_scores(wl, **kw)
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    cums = {b: [lo, hi] for b in range(wl.batch)}
    for t, (b, _, hi_pos, _) in enumerate(info):
        _, res = _reserved_residual(hi_pos + 1, 64, sink, rec)
        for g in range(wl.num_kv_heads):
            if not res:
                continue
            s = np.array([scores[t, g, j] for j in res])
            order = sorted(range(len(res)), key=lambda i: (-s[i], res[i]))
            e = np.exp(s - s.max())
            e /= e.sum()
            cums[b] += np.cumsum(e[order]).tolist()
    ps = []
    for b in range(wl.batch):
        c = np.unique(np.clip(np.array(cums[b]), lo, hi))
        gaps = np.diff(c)
        k = int(np.argmax(gaps))
        assert gaps[k] > 2 * margin
        ps.append(0.5 * (c[k] + c[k + 1]))
    return torch.as_tensor(np.array(ps, np.float32), device=wl.top_p.device)
