"""Benchmark of the SpotAttention decode hot path on B200.

One step = one decode step of one sparse attention layer for the whole batch:
selector scoring, residual softmax and dual top-p selection, then exact
attention over the selected KV blocks (spot_select + spot_sparse_decode,
i.e. spot_decode_step).  Steps rotate over several independent layer caches
(each far larger than the 126 MB L2), so every step reads its KV from HBM.

Default workload: the Qwen3-32B-shaped layer at L = 131072 (batch 4, 64 query
/ 8 KV heads, head_dim 128, blocks of 64, bf16 selector keys, top-p 0.95).
Reported: decode tokens/s for the whole model (per-layer time x 64 layers),
us per layer, and the HBM roofline fraction of the sparse-attention kernels
and of the whole step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl spot|reference]

Multi-GPU (torchrun, one process per GPU): every rank decodes its own batch
(data parallel over sequences, no collective on the data path); the time is
the max over ranks and `value` counts the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

HBM_FALLBACK_GBS = 6650.0

# DRAM bytes (read + write) of one launch of each workload's dominant kernel
# (dram__bytes_read.sum + dram__bytes_write.sum from an ncu capture of the
# same workload; where the layer caches rotated per step select different
# amounts, the mean over one launch per cache), valid only while the kernel's
# source files are unchanged (sha256 prefix over them); otherwise the
# roofline's traffic is null.
NCU_TRAFFIC = {
    "qwen3_32b_128k": {"bytes": 735307072 + 1026368, "sel_fmt": "bf16",
                       "files": ["sparse_decode.cu"],
                       "sha256": "e463ade2fe28a806"},
    "qwen3_8b_128k_tok": {"bytes": 307664896 + 965504, "sel_fmt": "bf16",
                          "files": ["sparse_decode.cu"],
                          "sha256": "e463ade2fe28a806"},
    "qwen3_8b_prefill_32k": {"bytes": 411903488 + 499184128, "sel_fmt": "bf16",
                             "files": ["prefill.cu", "tc.cuh"],
                             "sha256": "716d0750e6195d2d"},
}


def measured_traffic(args):
    """The recorded per-launch DRAM bytes, only for the exact capture: same
    workload, selector format and batch, and the kernel source unchanged."""
    import hashlib
    rec = NCU_TRAFFIC.get(args.workload)
    if rec is None or args.batch is not None or args.sel_fmt != rec["sel_fmt"]:
        return None
    h = hashlib.sha256()
    for name in rec["files"]:
        with open(os.path.join(ROOT, "block_sparse_long_spot_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return rec["bytes"] if h.hexdigest()[:16] == rec["sha256"] else None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank timing over all ranks (the only cross-rank traffic)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def layer_seed(rank: int, layer: int) -> int:
    """Seed of a rank's layer cache: every rank decodes its own sequences."""
    return 1000 * rank + layer


def rank_sequences(batch_total: int, world: int, rank: int) -> list:
    """Sequences of a global batch that rank `rank` decodes: a contiguous
    share, the first batch_total % world ranks one more (data parallel over
    sequences; no sequence is split, so no rank needs another's data)."""
    base, extra = divmod(batch_total, world)
    lo = rank * base + min(rank, extra)
    return list(range(lo, lo + base + (1 if rank < extra else 0)))


def shard_summary(batch_per_rank: int, world: int, ms_step_max: float, layers_model: int):
    """Whole-job decode throughput: tokens of all ranks over the slowest rank."""
    return batch_per_rank * world / (ms_step_max / 1e3 * layers_model)


def bench_metric(workload: str) -> str:
    """The metric line of a decode workload (the headline names L = 128K)."""
    if workload == "ragged_hybrid":
        return ("decode tokens/s, ragged L ~ U[8K, 128K] (whole model = per-layer step x "
                "sparse layers)")
    if workload == "qwen3_4b_32k":
        return "decode tokens/s at L=32K (whole model = per-layer step x sparse layers)"
    return "decode tokens/s at L=128K (whole model = per-layer step x sparse layers)"


def unit_counts(wl):
    lens = wl.seq_lens.cpu().numpy().astype(np.int64)
    return (lens + 63) // 64, lens // 64


def step_bytes(wl, sel_cnt: np.ndarray, fmt: str):
    """Algorithmic HBM bytes of one decode step and of its sparse-attention
    part, from the selection actually made."""
    B, Hq, Hkv = wl.batch, wl.num_q_heads, wl.num_kv_heads
    lens = wl.seq_lens.cpu().numpy().astype(np.int64)
    nb, n_full = unit_counts(wl)
    key_bytes = {"bf16": 128, "int4": 32 + 4, "mxfp4": 32 + 2, "fp8": 64, "int8": 64 + 2}[fmt]
    sel_cache = int(Hkv * n_full.sum() * key_bytes)
    # tokens attended per (b, g): full blocks, the last one possibly partial
    kv = 0
    for b in range(B):
        for g in range(Hkv):
            c = int(sel_cnt[b, g])
            kv += c * 64 * 128 * 2 * 2
    part = (lens % 64 != 0)
    # a partial last block is always selected: subtract its missing tokens
    kv -= int((Hkv * (64 - lens[part] % 64) * 128 * 2 * 2).sum())
    idx = int(sel_cnt.sum()) * 4 * 2          # selected list + page-table entry per block
    q_io = B * Hq * (128 * 2 + 128 * 4 + 4) + B * Hkv * 4
    sparse = kv + idx + q_io
    select = sel_cache + B * Hq * 64 * 2 + int(n_full.sum()) * 4 + int(sel_cnt.sum()) * 4
    return {"sparse": sparse, "select": select, "step": sparse + select, "kv": kv,
            "selector": sel_cache}


class CopyPipeline:
    """End-to-end stepping with the host copies overlapped: each step's
    inputs go from pinned host memory to one of two device buffers on an
    upload stream, the step computes on `stream` from that buffer into one of
    two output buffers, and the output goes back to pinned host memory on a
    download stream while the next step computes (uploads and downloads on
    separate streams, so neither queues behind the other's wait).  Events
    order every buffer reuse; time() brackets K steps from the first upload
    to the last download on the device."""

    def __init__(self, dev, host_inputs, out_like, stream):
        self.stream = stream
        self.up = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.host_inputs = host_inputs                    # per layer: tuple of pinned tensors
        self.dev_in = [[torch.empty_like(t, device=dev) for t in host_inputs[0]] for _ in range(2)]
        self.dev_out = [torch.empty_like(out_like) for _ in range(2)]
        self.host_out = [torch.empty(out_like.shape, dtype=out_like.dtype).pin_memory()
                         for _ in range(2)]
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_done = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.h2d = sum(t.numel() * t.element_size() for t in host_inputs[0])
        self.d2h = out_like.numel() * out_like.element_size()

    def step(self, i, compute):
        k = i & 1
        self.up.wait_event(self.ev_done[k])           # step i - 2 is done with dev_in[k]
        with torch.cuda.stream(self.up):
            for d, h in zip(self.dev_in[k], self.host_inputs[i % len(self.host_inputs)]):
                d.copy_(h, non_blocking=True)
            self.ev_in[k].record(self.up)
        self.stream.wait_event(self.ev_in[k])
        self.stream.wait_event(self.ev_out[k])        # dev_out[k] of step i - 2 downloaded
        compute(i, *self.dev_in[k], self.dev_out[k])
        self.ev_done[k].record(self.stream)
        self.down.wait_event(self.ev_done[k])
        with torch.cuda.stream(self.down):
            self.host_out[k].copy_(self.dev_out[k], non_blocking=True)
            self.ev_out[k].record(self.down)

    def time(self, K, warmup, compute):
        for i in range(warmup):
            self.step(i, compute)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        self.up.wait_event(e0)
        self.down.wait_event(e0)
        for i in range(K):
            self.step(i, compute)
        self.stream.wait_event(self.ev_out[(K - 1) & 1])
        self.stream.wait_event(self.ev_out[K & 1])
        e1.record(self.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K


def run_spot(args, world, rank, local):
    import block_sparse_long_spot_b200 as spot
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    fmt = args.sel_fmt
    layers = []
    for l in range(args.layers):
        # layers of one model share sequence lengths and page tables
        wl = workloads.make(args.workload, seed=layer_seed(rank, l), device=dev, sel_fmt=fmt,
                            batch=args.batch, structure_from=layers[0][0] if layers else None)
        desc = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, fmt)
        if fmt == "bf16":
            data, scales = wl.sel_keys, None
        else:
            data, scales = spot.selector_pool(fmt, wl.num_pages, wl.num_kv_heads, device=dev)
            nb, n_full = unit_counts(wl)
            seq = np.concatenate([np.full(n, b) for b, n in enumerate(n_full)]).astype(np.int32)
            blk = np.concatenate([np.arange(n) for n in n_full]).astype(np.int32)
            pages = wl.page_table.cpu().numpy()[seq, blk]
            spot.append_selector_keys(desc, data, scales, wl.page_table,
                                      torch.as_tensor(seq, device=dev),
                                      torch.as_tensor(blk, device=dev),
                                      wl.sel_keys[torch.as_tensor(pages, device=dev).long()])
        layers.append((wl, desc, data, scales))
    wl0, desc0 = layers[0][0], layers[0][1]
    B, Hq, Hkv, mb = wl0.batch, wl0.num_q_heads, wl0.num_kv_heads, wl0.max_blocks
    prm = spot.select_params("topp", wl0.spec.sink_blocks, wl0.spec.recency_blocks,
                             wl0.spec.kmin_blocks)
    ws = spot.new_workspace(desc0, B, mb, dev)
    sel_idx = torch.empty(B, Hkv, mb, dtype=torch.int32, device=dev)
    sel_cnt = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=dev)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None, st=None):
        st = stream if st is None else st
        wl, desc, data, scales = layers[i % len(layers)]
        if ev is not None:
            ev[0].record(st)
        spot.select(desc, prm, wl.q_sel, wl.w, data, scales, wl.page_table, wl.seq_lens,
                    wl.top_p, sel_idx, sel_cnt, ws, st)
        if ev is not None:
            ev[1].record(st)
        spot.sparse_decode(desc, wl.q, wl.k_pool, wl.v_pool, wl.page_table, wl.seq_lens, sel_idx,
                           sel_cnt, wl.sm_scale, out, lse, ws, st)
        if ev is not None:
            ev[2].record(st)

    # selection statistics and algorithmic bytes per layer
    per_layer = []
    for l in range(len(layers)):
        step(l)
        torch.cuda.synchronize()
        cnt = sel_cnt.cpu().numpy().copy()
        wl = layers[l][0]
        nb, _ = unit_counts(wl)
        per_layer.append((step_bytes(wl, cnt, fmt), cnt / np.maximum(nb[:, None], 1)))
    status = spot.read_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t0.record(stream)
        for i in range(K):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_total = t0.elapsed_time(t1)
    ms_step = max_over_ranks(ms_total / K, world)
    # per-kernel durations in a second pass (events between the two calls keep
    # them from overlapping, so this pass is not the step time)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        step(i, evs[i])
    torch.cuda.synchronize()
    ms_sel = [e[0].elapsed_time(e[1]) for e in evs]
    ms_dec = [e[1].elapsed_time(e[2]) for e in evs]

    # ---- the same steps replayed from CUDA graphs (one per layer cache):
    # the host's per-launch work leaves the timed region
    cap = torch.cuda.Stream(dev)
    graphs = []
    for l in range(len(layers)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(l, st=cap)
        graphs.append(g)
    for i in range(args.warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for i in range(K):
        graphs[i % len(graphs)].replay()
    g1.record(stream)
    torch.cuda.synchronize()
    ms_graph = max_over_ranks(g0.elapsed_time(g1) / K, world)
    del graphs

    # ---- end to end through the public call with host buffers
    pipe = CopyPipeline(dev, [(layers[l][0].q.cpu().pin_memory(),
                               layers[l][0].q_sel.cpu().pin_memory()) for l in range(len(layers))],
                        out, stream)

    def e2e_compute(i, q_dev, qs_dev, out_dev):
        wl, desc, data, scales = layers[i % len(layers)]
        spot.decode_step(desc, prm, qs_dev, wl.w, data, scales, q_dev, wl.k_pool, wl.v_pool,
                         wl.page_table, wl.seq_lens, wl.top_p, wl.sm_scale, sel_idx, sel_cnt,
                         out_dev, lse, ws, stream)

    barrier(world)
    ms_e2e = max_over_ranks(pipe.time(K, args.warmup, e2e_compute), world)
    barrier(world)
    status = spot.read_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after timing")

    nl = len(layers)
    b_sparse = np.mean([per_layer[i % nl][0]["sparse"] for i in range(K)])
    b_step = np.mean([per_layer[i % nl][0]["step"] for i in range(K)])
    frac_sel = np.concatenate([x[1].ravel() for x in per_layer])
    dec_ms = float(np.mean(ms_dec))
    sel_ms = float(np.mean(ms_sel))
    peak, peak_kind = peaks()
    layers_model = wl0.spec.layers_sparse
    value = shard_summary(B, world, ms_step, layers_model)
    value_e2e = shard_summary(B, world, ms_e2e, layers_model)
    achieved = b_sparse / (dec_ms / 1e3) / 1e9
    res = {
        "metric": bench_metric(args.workload),
        "value": round(value, 3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "us_per_layer": round(ms_step * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 with planted hot blocks)",
        "config": {
            "workload": args.workload, "batch_per_gpu": B, "q_heads": Hq, "kv_heads": Hkv,
            "head_dim": 128, "context": int(wl0.seq_lens.max().item()), "block": 64,
            "sel_fmt": fmt, "top_p": float(wl0.top_p[0].item()),
            "sink_blocks": wl0.spec.sink_blocks, "recency_blocks": wl0.spec.recency_blocks,
            "kmin_blocks": wl0.spec.kmin_blocks, "layers_in_model": layers_model,
            "layer_caches_rotated": nl,
            "l2": f"inputs larger than L2: {nl} layer caches of "
                  f"{wl0.k_pool.numel() * 4 / 1e9:.2f} GB rotated per step",
            "selected_fraction": {"mean": round(float(frac_sel.mean()), 4),
                                  "min": round(float(frac_sel.min()), 4),
                                  "max": round(float(frac_sel.max()), 4)},
            "parallelism": f"dp{world} (sequences)",
        },
        "roofline": {
            "bound": "hbm", "kernel": "sparse decode (attention + combine)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": measured_traffic(args),
            "peak_source": peak_kind,
            "algorithmic_bytes_per_launch": int(b_sparse), "ms_per_launch": round(dec_ms, 5),
        },
        "step_roofline": {
            "achieved": round(b_step / (ms_step / 1e3) / 1e9, 1), "peak": peak, "unit": "GB/s",
            "frac": round(b_step / (ms_step / 1e3) / 1e9 / peak, 4),
            "algorithmic_bytes_per_step": int(b_step),
            "select_ms": round(sel_ms, 5),
        },
        "e2e": {"value": round(value_e2e, 3), "unit": "tokens/s",
                "ms_per_step": round(ms_e2e, 5),
                "h2d_bytes_per_step": pipe.h2d, "d2h_bytes_per_step": pipe.d2h,
                "copies": "double-buffered; uploads and downloads on a second stream overlap "
                          "the neighbouring steps' compute"},
        "graph": {"ms_per_step": round(ms_graph, 5),
                  "value": round(shard_summary(B, world, ms_graph, layers_model), 3),
                  "note": "the same steps replayed from captured CUDA graphs"},
        "gpu_launches": K * 2,          # scoring + selection (one launch), sparse decode per step
        "clocks": clk.summary(),
    }
    return res, layers


def tok_row_bytes(fmt: str, idx_dim: int = 128) -> int:
    """Bytes of one stored per-token selector key row (codes + scales)."""
    return {"bf16": 2 * idx_dim, "fp8": idx_dim, "int8": idx_dim + 2,
            "int4": idx_dim // 2 + 2 * (idx_dim // 32),
            "mxfp4": idx_dim // 2 + idx_dim // 32}[fmt]


def tok_step_bytes(wl, sel_cnt: np.ndarray, fmt: str = "bf16"):
    """Algorithmic HBM bytes of one token-selector decode step: the
    per-token selector keys of every complete 16-token block (codes and
    scales of the stored format), the K and V rows of the selected tokens
    for every KV head, indices and queries."""
    B, Hq, Hkv, sb = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.spec.sel_block
    lens = wl.seq_lens.cpu().numpy().astype(np.int64)
    n_full = lens // sb
    sel_cache = int(n_full.sum()) * sb * wl.spec.idx_heads * tok_row_bytes(fmt, wl.spec.idx_dim)
    kv = int(sel_cnt.sum()) * sb * Hkv * 128 * 2 * 2
    part = lens % sb != 0                     # the partial last block is always selected
    kv -= int((Hkv * (sb - lens[part] % sb) * 128 * 2 * 2).sum())
    idx = int(sel_cnt.sum()) * 4 * 2 * Hkv    # each KV head reads the list and the page id
    q_io = B * Hq * (128 * 2 + 128 * 4 + 4)
    select = (sel_cache + B * wl.spec.idx_heads * (wl.spec.idx_dim * 2 + 4) +
              int(n_full.sum()) * 4 + int(sel_cnt.sum()) * 4)
    sparse = kv + idx + q_io
    return {"sparse": sparse, "select": select, "step": sparse + select, "kv": kv,
            "selector": sel_cache}


def sel_pool_bytes(pool) -> int:
    return sum(t.numel() * t.element_size() for t in pool if t is not None)


def tok_pool(spot, wl, desc, fmt):
    """The layer's per-token selector pool in `fmt`: the workload's bf16
    keys as they are, or written through the library's quantising append
    (every cached token, by sequence and position)."""
    if fmt == "bf16":
        return wl.sel_tok, None
    dev = wl.q.device
    data, scales = spot.tok_selector_pool(wl.num_pages, fmt, device=dev)
    lens = wl.seq_lens.cpu().numpy()
    pt = wl.page_table.cpu().numpy()
    seq = np.concatenate([np.full(int(L), b) for b, L in enumerate(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(int(L)) for L in lens]).astype(np.int32)
    page = torch.as_tensor(pt[seq, pos // 64].astype(np.int64), device=dev)
    keys = wl.sel_tok[page, torch.as_tensor(pos % 64, device=dev).long()].contiguous()
    spot.tok_append_selector_keys(desc, data, scales, wl.page_table,
                                  torch.as_tensor(seq, device=dev),
                                  torch.as_tensor(pos, device=dev), keys)
    torch.cuda.synchronize()
    return data, scales


def run_spot_tok(args, world, rank, local):
    """The token-level, layer-shared selector path (tok_select, then
    tok_sparse_decode), timed like run_spot."""
    import block_sparse_long_spot_b200 as spot
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    fmt = args.sel_fmt
    layers, pools = [], []
    for l in range(args.layers):
        wl = workloads.make_tok(args.workload, seed=layer_seed(rank, l), device=dev)
        desc = spot.tok_layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, sel_fmt=fmt)
        layers.append((wl, desc))
        pools.append(tok_pool(spot, wl, desc, fmt))
    wl0, desc0 = layers[0]
    B, Hq, mb = wl0.batch, wl0.num_q_heads, wl0.max_blocks
    sp = wl0.spec
    prm = spot.select_params("topp", sp.sink_blocks, sp.recency_blocks, sp.kmin_blocks)
    # one workspace per layer cache: the layers differ in their page counts
    wss = [spot.new_tok_workspace(d, B, mb, dev) for _, d in layers]
    sel_idx = torch.empty(B, mb, dtype=torch.int32, device=dev)
    sel_cnt = torch.empty(B, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=dev)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        wl, desc = layers[i % len(layers)]
        ws = wss[i % len(layers)]
        sd, ss = pools[i % len(layers)]
        if ev is not None:
            ev[0].record(stream)
        spot.tok_select(desc, prm, wl.q_idx, wl.w_idx, sd, ss, wl.page_table, wl.seq_lens,
                        wl.top_p, sel_idx, sel_cnt, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        spot.tok_sparse_decode(desc, wl.q, wl.k_pool, wl.v_pool, wl.page_table, wl.seq_lens,
                               sel_idx, sel_cnt, wl.sm_scale, out, lse, ws, stream)
        if ev is not None:
            ev[2].record(stream)

    per_layer = []
    for l in range(len(layers)):
        step(l)
        torch.cuda.synchronize()
        cnt = sel_cnt.cpu().numpy().copy()
        wl = layers[l][0]
        nb = (wl.seq_lens.cpu().numpy() + sp.sel_block - 1) // sp.sel_block
        per_layer.append((tok_step_bytes(wl, cnt, fmt), cnt / np.maximum(nb, 1)))
    for ws in wss:
        status = spot.read_device_status(ws)
        if status != 0:
            raise RuntimeError(f"device status {status} after warm-up")
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t0.record(stream)
        for i in range(K):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_step = max_over_ranks(t0.elapsed_time(t1) / K, world)
    # per-kernel durations in a second pass (not the step time)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        step(i, evs[i])
    torch.cuda.synchronize()
    sel_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    dec_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))

    pipe = CopyPipeline(dev, [(wl.q.cpu().pin_memory(), wl.q_idx.cpu().pin_memory())
                              for wl, _ in layers], out, stream)

    def e2e_compute(i, q_dev, qi_dev, out_dev):
        wl, desc = layers[i % len(layers)]
        sd, ss = pools[i % len(layers)]
        spot.tok_decode_step(desc, prm, qi_dev, wl.w_idx, sd, ss, q_dev, wl.k_pool,
                             wl.v_pool, wl.page_table, wl.seq_lens, wl.top_p, wl.sm_scale,
                             sel_idx, sel_cnt, out_dev, lse, wss[i % len(layers)], stream)

    barrier(world)
    ms_e2e = max_over_ranks(pipe.time(K, args.warmup, e2e_compute), world)
    barrier(world)
    for ws in wss:
        status = spot.read_device_status(ws)
        if status != 0:
            raise RuntimeError(f"device status {status} after timing")

    nl = len(layers)
    b_sparse = float(np.mean([per_layer[i % nl][0]["sparse"] for i in range(K)]))
    b_select = float(np.mean([per_layer[i % nl][0]["select"] for i in range(K)]))
    b_step = b_sparse + b_select
    frac_sel = np.concatenate([x[1].ravel() for x in per_layer])
    peak, peak_kind = peaks()
    layers_model = sp.layers_sparse
    value = shard_summary(B, world, ms_step, layers_model)
    value_e2e = shard_summary(B, world, ms_e2e, layers_model)
    dom_sparse = b_sparse >= b_select
    kb, kms = (b_sparse, dec_ms) if dom_sparse else (b_select, sel_ms)
    achieved = kb / (kms / 1e3) / 1e9
    return {
        "metric": bench_metric(args.workload),
        "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "us_per_layer": round(ms_step * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 with planted hot 16-token blocks)",
        "config": {
            "workload": args.workload, "selector": "token-level, layer-shared",
            "batch_per_gpu": B, "q_heads": Hq, "kv_heads": wl0.num_kv_heads, "head_dim": 128,
            "idx_heads": sp.idx_heads, "idx_dim": sp.idx_dim, "sel_block": sp.sel_block,
            "context": int(wl0.seq_lens.max().item()), "sel_fmt": fmt,
            "top_p": float(wl0.top_p[0].item()), "sink_blocks": sp.sink_blocks,
            "recency_blocks": sp.recency_blocks, "kmin_blocks": sp.kmin_blocks,
            "layers_in_model": layers_model, "layer_caches_rotated": nl,
            "l2": f"inputs larger than L2: {nl} layer caches of "
                  f"{(wl0.k_pool.numel() * 4 + sel_pool_bytes(pools[0])) / 1e9:.2f} GB rotated",
            "selected_fraction": {"mean": round(float(frac_sel.mean()), 4),
                                  "min": round(float(frac_sel.min()), 4),
                                  "max": round(float(frac_sel.max()), 4)},
            "parallelism": f"dp{world} (sequences)",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "sparse decode (attention + combine)" if dom_sparse else
                      "token selector (scoring + selection)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": measured_traffic(args) if dom_sparse else None,
            "peak_source": peak_kind,
            "algorithmic_bytes_per_launch": int(kb), "ms_per_launch": round(kms, 5),
        },
        "select_roofline": {
            "achieved": round(b_select / (sel_ms / 1e3) / 1e9, 1), "peak": peak,
            "frac": round(b_select / (sel_ms / 1e3) / 1e9 / peak, 4),
            "algorithmic_bytes": int(b_select), "ms": round(sel_ms, 5)},
        "sparse_roofline": {
            "achieved": round(b_sparse / (dec_ms / 1e3) / 1e9, 1), "peak": peak,
            "frac": round(b_sparse / (dec_ms / 1e3) / 1e9 / peak, 4),
            "algorithmic_bytes": int(b_sparse), "ms": round(dec_ms, 5)},
        "step_roofline": {
            "achieved": round(b_step / (ms_step / 1e3) / 1e9, 1), "peak": peak, "unit": "GB/s",
            "frac": round(b_step / (ms_step / 1e3) / 1e9 / peak, 4),
            "algorithmic_bytes_per_step": int(b_step)},
        "e2e": {"value": round(value_e2e, 3), "unit": "tokens/s",
                "ms_per_step": round(ms_e2e, 5),
                "h2d_bytes_per_step": pipe.h2d, "d2h_bytes_per_step": pipe.d2h,
                "copies": "double-buffered; uploads and downloads on a second stream overlap "
                          "the neighbouring steps' compute"},
        "gpu_launches": K * 3,          # token scoring, selection, sparse decode per step
        "clocks": clk.summary(),
    }, layers


def tok_oracle_inputs(wl, fmt="bf16"):
    """(shape, params, arguments) of the oracle's token-selector decode step
    for a workload, the selector keys quantised by the oracle to `fmt`."""
    import oracle
    sp = wl.spec
    sh = oracle.make_tok_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.num_pages,
                               wl.max_pages, sel_fmt=fmt)
    pr = oracle.make_params(sink_blocks=sp.sink_blocks, recency_blocks=sp.recency_blocks,
                            kmin_blocks=sp.kmin_blocks)
    bits = workloads.bits(wl.sel_tok)
    data, scales = (bits, None) if fmt == "bf16" else oracle.quantize_selector(fmt, bits)
    a = dict(q_idx=workloads.bits(wl.q_idx),
             w=None if wl.w_idx is None else wl.w_idx.cpu().numpy(),
             sel_tok=data, sel_scales=scales, q=workloads.bits(wl.q),
             k_pool=workloads.bits(wl.k_pool), v_pool=workloads.bits(wl.v_pool),
             page_table=wl.page_table.cpu().numpy(), seq_lens=wl.seq_lens.cpu().numpy(),
             top_p=wl.top_p.cpu().numpy(), sm_scale=wl.sm_scale)
    return sh, pr, a


def cpu_baseline_tok(wl, fmt="bf16", min_s=10.0, max_s=30.0):
    """The fp64 oracle's token-selector decode step on the host cores, one
    sequence at a time, until about 10 s of work; scaled to the model."""
    import oracle
    sp = wl.spec
    sh, pr, a = tok_oracle_inputs(wl, fmt)
    total, n = 0.0, 0
    while total < min_s and n < 64:
        t = time.perf_counter()
        oracle.tok_decode_step(sh, pr, seqs=[n % wl.batch], **a)
        total += time.perf_counter() - t
        n += 1
        if total > max_s:
            break
    per_seq = total / n
    value = 1.0 / (per_seq * sp.layers_sparse)
    return {"value": round(value, 6), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"fp64 oracle token-selector decode step of one sequence (all heads), "
                      f"{n} runs, {total:.1f} s; x{sp.layers_sparse} layers"}


def prefill_flops(wl, sel_idx: np.ndarray, sel_cnt: np.ndarray):
    """Algorithmic FLOPs of one sparse-prefill layer from the selection made:
    attention 4 * 128 per (query, head, attended key) -- QK^T and PV -- and
    tile scoring 2 * 64 per (query, head, scored block)."""
    import oracle
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    G = wl.num_q_heads // wl.num_kv_heads
    attn = 0
    score = 0
    for t, (_, lo, hi, _) in enumerate(info):
        m = lo // 64
        nq = hi - lo + 1
        pos = np.arange(lo, hi + 1)
        n_full = (hi + 1) // 64
        for g in range(wl.num_kv_heads):
            sel = sel_idx[t, g, :sel_cnt[t, g]]
            before = int((sel < m).sum()) * 64
            keys = before * nq + ((pos - m * 64 + 1).sum() if (sel == m).any() else 0)
            attn += int(keys) * G * 4 * 128
            score += nq * G * n_full * 64 * 2
    return attn, score


def block_pool(spot, wl, desc, fmt):
    """A layer's per-block selector pool in `fmt`: the workload's bf16 keys as
    they are, or written through the library's quantising append (every
    complete block of every sequence)."""
    if fmt == "bf16":
        return wl.sel_keys, None
    dev = wl.q.device
    data, scales = spot.selector_pool(fmt, wl.num_pages, wl.num_kv_heads, device=dev)
    lens = wl.seq_lens.cpu().numpy()
    pt = wl.page_table.cpu().numpy()
    seq = np.concatenate([np.full(int(L) // 64, b) for b, L in enumerate(lens)]).astype(np.int32)
    blk = np.concatenate([np.arange(int(L) // 64) for L in lens]).astype(np.int32)
    if seq.size:
        keys = wl.sel_keys[torch.as_tensor(pt[seq, blk].astype(np.int64), device=dev)].contiguous()
        spot.append_selector_keys(desc, data, scales, wl.page_table,
                                  torch.as_tensor(seq, device=dev), torch.as_tensor(blk, device=dev),
                                  keys)
    torch.cuda.synchronize()
    return data, scales


def run_spot_prefill(args, world, rank, local):
    """One sparse-prefill layer (plan, tile scoring, selection, attention)
    per step over the whole chunk."""
    import block_sparse_long_spot_b200 as spot
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    layers = [workloads.make_prefill(args.workload, seed=layer_seed(rank, l), device=dev)
              for l in range(args.layers)]
    wl0 = layers[0]
    sp = wl0.spec
    Hq, Hkv, mb = wl0.num_q_heads, wl0.num_kv_heads, wl0.max_blocks
    nt = spot.prefill_num_tiles(wl0.seq_lens.cpu().numpy(), wl0.q_lens.cpu().numpy())
    fmt = args.sel_fmt
    descs = [spot.layer_desc(Hq, Hkv, w.num_pages, fmt) for w in layers]
    pools = [block_pool(spot, w, d, fmt) for w, d in zip(layers, descs)]
    prm = spot.select_params("topp", sp.sink_blocks, sp.recency_blocks, sp.kmin_blocks)
    wss = [spot.new_prefill_workspace(d, wl0.batch, nt, mb, dev) for d in descs]
    rows = int(wl0.q.shape[0])
    sel_idx = torch.empty(nt, Hkv, mb, dtype=torch.int32, device=dev)
    sel_cnt = torch.empty(nt, Hkv, dtype=torch.int32, device=dev)
    out = torch.empty(rows, Hq, 128, dtype=torch.float32, device=dev)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, q=None, q_sel=None, o=None):
        w = layers[i % len(layers)]
        sd, ss = pools[i % len(layers)]
        spot.prefill(descs[i % len(layers)], prm, w.q_sel if q_sel is None else q_sel, w.w,
                     sd, ss, w.q if q is None else q, w.k_pool, w.v_pool, w.page_table,
                     w.seq_lens, w.q_lens, w.top_p, w.sm_scale, sel_idx, sel_cnt,
                     out if o is None else o, lse, wss[i % len(layers)], stream)

    flops = []
    sel0 = None
    for l in range(len(layers)):
        step(l)
        torch.cuda.synchronize()
        if l == 0:
            sel0 = (sel_idx.cpu().numpy(), sel_cnt.cpu().numpy())
        flops.append(prefill_flops(layers[l], sel_idx.cpu().numpy(), sel_cnt.cpu().numpy()))
        frac = (sel_cnt.cpu().numpy().astype(np.float64) /
                (np.arange(nt)[:, None] + 1)).mean()
    for ws in wss:
        if spot.read_device_status(ws) != 0:
            raise RuntimeError("device status after warm-up")
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t0.record(stream)
        for i in range(K):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_step = max_over_ranks(t0.elapsed_time(t1) / K, world)
    # end to end: the step's queries (q, q_sel) copied from pinned host memory
    pipe = CopyPipeline(dev, [(w.q.cpu().pin_memory(), w.q_sel.cpu().pin_memory())
                              for w in layers], out, stream)
    ms_e2e = max_over_ranks(pipe.time(K, 1, lambda i, q, qs, o: step(i, q, qs, o)), world)
    for ws in wss:
        if spot.read_device_status(ws) != 0:
            raise RuntimeError("device status after timing")
    nl = len(layers)
    f_attn = float(np.mean([flops[i % nl][0] for i in range(K)]))
    f_score = float(np.mean([flops[i % nl][1] for i in range(K)]))
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, peak_kind = float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        peak, peak_kind = 1400.0, "fallback (sustained)"
    tokens = int(wl0.q_lens.sum().item())
    value = tokens * world / (ms_step / 1e3 * sp_layers(args))
    achieved = (f_attn + f_score) / (ms_step / 1e3) / 1e12
    return {
        "metric": "prefill tokens/s at L=32K (whole model = per-layer time x layers)",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 with planted hot blocks)",
        "config": {"workload": args.workload, "batch_per_gpu": wl0.batch, "q_heads": Hq,
                   "kv_heads": Hkv, "head_dim": 128, "context": int(wl0.seq_lens.max().item()),
                   "chunk": int(wl0.q_lens.max().item()), "tiles": nt, "block": 64,
                   "sel_fmt": fmt,
                   "top_p": sp.top_p, "sink_blocks": sp.sink_blocks,
                   "recency_blocks": sp.recency_blocks, "kmin_blocks": sp.kmin_blocks,
                   "layers_in_model": sp_layers(args), "layer_caches_rotated": nl,
                   "selected_fraction_mean": round(float(frac), 4),
                   "l2": "compute-bound; KV of a layer re-read from L2 by its tiles",
                   "parallelism": f"dp{world} (sequences)"},
        "roofline": {"bound": "tensor", "kernel": "sparse prefill (all four kernels)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": measured_traffic(args),
                     "traffic_kernel": "prefill_attn_kernel (dram read + write of one launch)",
                     "peak_source": peak_kind,
                     "algorithmic_flops_per_step": int(f_attn + f_score),
                     "attention_flops": int(f_attn), "scoring_flops": int(f_score)},
        "e2e": {"value": round(tokens * world / (ms_e2e / 1e3 * sp_layers(args)), 1),
                "unit": "tokens/s", "ms_per_step": round(ms_e2e, 4),
                "h2d_bytes_per_step": pipe.h2d, "d2h_bytes_per_step": pipe.d2h,
                "copies": "double-buffered; uploads and downloads on a second stream overlap "
                          "the neighbouring steps' compute"},
        "gpu_launches": K * 4,          # plan, tile scores, selection, attention per step
        "clocks": clk.summary(),
    }, (layers, sel0[0], sel0[1])


def cpu_baseline_prefill(wl, sel_idx, sel_cnt, layers_model, fmt="bf16"):
    """The fp64 oracle's sparse prefill on the host cores for two tiles (the
    last and a middle one, all KV heads), scaled to the layer by the share of
    the layer's attention FLOPs those tiles hold, then to the model."""
    import oracle
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    nt = len(info)
    tiles = [nt - 1, nt // 2]
    sh = oracle.make_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, 128, 64, 64, fmt,
                           wl.num_pages, wl.max_blocks)
    sp = wl.spec
    pr = oracle.make_params(sink_blocks=sp.sink_blocks, recency_blocks=sp.recency_blocks,
                            kmin_blocks=sp.kmin_blocks)
    bits = workloads.bits(wl.sel_keys)
    sd, ss = (bits, None) if fmt == "bf16" else oracle.quantize_selector(fmt, bits)
    args = dict(q_sel=workloads.bits(wl.q_sel), w=None, sel_data=sd,
                sel_scales=ss, q=workloads.bits(wl.q), k_pool=workloads.bits(wl.k_pool),
                v_pool=workloads.bits(wl.v_pool), page_table=wl.page_table.cpu().numpy(),
                seq_lens=wl.seq_lens.cpu().numpy(), q_lens=wl.q_lens.cpu().numpy(),
                top_p=wl.top_p.cpu().numpy(), sm_scale=wl.sm_scale)
    t = time.perf_counter()
    oracle.prefill_step(sh, pr, tiles=tiles, **args)
    sec = time.perf_counter() - t
    mask = np.zeros(nt, bool)
    mask[tiles] = True
    part = prefill_flops_tiles(wl, sel_idx, sel_cnt, mask)
    total = prefill_flops_tiles(wl, sel_idx, sel_cnt, np.ones(nt, bool))
    layer_s = sec * total / max(part, 1)
    tokens = int(wl.q_lens.sum().item())
    return {"value": round(tokens / (layer_s * layers_model), 3), "unit": "tokens/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"fp64 oracle sparse prefill of tiles {tiles} (all KV heads), {sec:.1f} s, "
                      f"scaled by attention FLOPs to the {nt} tiles of the layer, "
                      f"x{layers_model} layers"}


def prefill_flops_tiles(wl, sel_idx, sel_cnt, mask):
    import oracle
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    G = wl.num_q_heads // wl.num_kv_heads
    total = 0
    for t, (_, lo, hi, _) in enumerate(info):
        if not mask[t]:
            continue
        m, nq = lo // 64, hi - lo + 1
        pos = np.arange(lo, hi + 1)
        for g in range(wl.num_kv_heads):
            sel = sel_idx[t, g, :sel_cnt[t, g]]
            keys = int((sel < m).sum()) * 64 * nq + (int((pos - m * 64 + 1).sum())
                                                     if (sel == m).any() else 0)
            total += keys * G * 4 * 128
    return total


def sp_layers(args):
    return 36 if "qwen3_8b" in args.workload else 1


def prepare_oracle(wl, fmt, seqs):
    """Host copies of sequences `seqs` of a layer, ready for the fp64 oracle."""
    import oracle
    sub = workloads.gather_units(wl, seqs)
    data, scales = oracle.quantize_selector(fmt, workloads.bits(sub.sel_keys))
    sh = oracle.make_shape(sub.batch, sub.num_q_heads, sub.num_kv_heads, 128, 64, 64, fmt,
                           sub.num_pages, sub.max_blocks)
    pr = oracle.make_params(sink_blocks=sub.spec.sink_blocks,
                            recency_blocks=sub.spec.recency_blocks,
                            kmin_blocks=sub.spec.kmin_blocks)
    args = dict(q_sel=workloads.bits(sub.q_sel), w=None, sel_data=data, sel_scales=scales,
                q=workloads.bits(sub.q), k_pool=workloads.bits(sub.k_pool),
                v_pool=workloads.bits(sub.v_pool), page_table=sub.page_table.cpu().numpy(),
                seq_lens=sub.seq_lens.cpu().numpy(), top_p=sub.top_p.cpu().numpy(),
                sm_scale=sub.sm_scale)
    return sh, pr, args


def time_oracle(prep, units=None):
    import oracle
    sh, pr, args = prep
    t = time.perf_counter()
    oracle.decode_step(sh, pr, units=units, **args)
    return time.perf_counter() - t


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleSampler:
    """Bounded samples of one layer for the fp64 oracle: a sample is the
    decode step (scoring, selection, attention) of `per` consecutive
    (sequence, KV head) units of the layer, walking round the layer's units
    from sample to sample.  Host copies are made outside the timed calls and
    kept for the last sequences touched."""

    def __init__(self, wl, fmt, per):
        self.wl, self.fmt = wl, fmt
        self.U = wl.batch * wl.num_kv_heads
        self.per = max(1, min(per, self.U))
        self.next = 0
        self.cache = {}

    def _prep(self, seqs):
        key = tuple(seqs)
        if key not in self.cache:
            self.cache.clear()                    # one sample's sequences on the host at a time
            self.cache[key] = prepare_oracle(self.wl, self.fmt, seqs)
        return self.cache[key]

    def take(self):
        """Runs the next sample; returns (seconds, units run)."""
        Hkv = self.wl.num_kv_heads
        units = [(self.next + k) % self.U for k in range(self.per)]
        self.next = (self.next + self.per) % self.U
        seqs = sorted({u // Hkv for u in units})
        local = [seqs.index(u // Hkv) * Hkv + u % Hkv for u in units]
        return time_oracle(self._prep(seqs), units=local), len(units)


def cpu_baseline(wl, fmt, min_s=10.0, max_s=30.0):
    """The fp64 oracle on the host: samples of as many (sequence, KV head)
    units as there are cores, run in parallel over the units on every core
    until about min_s of work, then single units on one core; the rate in
    units per second becomes decode tokens/s of the model (one token of a
    sequence = its Hkv units in every sparse layer)."""
    import oracle
    cores = host_cores()
    units_per_token = wl.num_kv_heads * wl.spec.layers_sparse
    smp = OracleSampler(wl, fmt, cores)
    oracle.set_num_threads(cores)
    total, done = 0.0, 0
    while total < min_s and done < 64 * smp.U:
        sec, n = smp.take()
        total += sec
        done += n
        if total > max_s:
            break
    rate_all = done / total
    one = OracleSampler(wl, fmt, 1)
    oracle.set_num_threads(1)
    t1, d1 = 0.0, 0
    while t1 < min_s / 2 and d1 < smp.U:
        sec, n = one.take()
        t1 += sec
        d1 += n
    rate_one = d1 / t1
    oracle.set_num_threads(cores)
    return {"value": round(rate_all / units_per_token, 6), "unit": "tokens/s", "cores": cores,
            "kind": "oracle", "cpu": cpu_model(),
            "single_thread": {"value": round(rate_one / units_per_token, 6), "cores": 1,
                              "sample": f"{d1} units one at a time, {t1:.1f} s"},
            "sample": f"fp64 oracle decode step (scoring, selection, attention) over {done} "
                      f"(sequence, KV head) units of the layer in samples of {smp.per} units "
                      f"run in parallel on {cores} threads, {total:.1f} s; tokens/s = "
                      f"units/s / ({wl.num_kv_heads} KV heads x {wl.spec.layers_sparse} sparse "
                      f"layers)"}


def run_reference(args, world, rank):
    """The fp64 CPU oracle as the reference arm, on the same workload: each
    step is one bounded sample of the layer -- the decode step of as many
    (sequence, KV head) units as the host has cores, in parallel on all of
    them -- walking round the layer's units; tokens/s = units per second /
    (KV heads x sparse layers), ms_per_step the measured time of one sample."""
    if rank != 0:
        return None
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = workloads.make(args.workload, seed=0, device=dev, sel_fmt=args.sel_fmt, batch=args.batch)
    cores = host_cores()
    oracle.set_num_threads(cores)
    smp = OracleSampler(wl, args.sel_fmt, cores)
    secs, units = [], 0
    for i in range(args.warmup + args.steps):
        sec, n = smp.take()
        if i >= args.warmup:
            secs.append(sec)
            units += n
    total = float(sum(secs))
    units_per_token = wl.num_kv_heads * wl.spec.layers_sparse
    value = units / total / units_per_token
    sample = (f"each step: the fp64 oracle decode step of {smp.per} consecutive (sequence, KV head) "
              f"units of the {smp.U}-unit layer, in parallel on {cores} threads, walking round "
              f"the layer; tokens/s = units/s / ({wl.num_kv_heads} KV heads x "
              f"{wl.spec.layers_sparse} sparse layers)")
    return {
        "impl": "reference",
        "metric": bench_metric(args.workload),
        "value": round(value, 6), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / len(secs) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 with planted hot blocks)",
        "config": {"workload": args.workload, "sel_fmt": args.sel_fmt, "sample": sample},
        "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "cpu": cpu_model(), "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_reference_tok(args, world, rank):
    """Reference arm for the token-selector workloads: each step times the
    fp64 oracle's decode step of one sequence (all heads) on the host cores."""
    if rank != 0:
        return None
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = workloads.make_tok(args.workload, seed=0, device=dev)
    times = []
    sp = wl.spec
    sh, pr, a = tok_oracle_inputs(wl, args.sel_fmt)
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        oracle.tok_decode_step(sh, pr, seqs=[i % wl.batch], **a)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    per_layer = float(np.mean(times)) * wl.batch
    value = wl.batch / (per_layer * sp.layers_sparse)
    sample = f"one sequence (all heads) per step; x{wl.batch} sequences x{sp.layers_sparse} layers"
    return {
        "impl": "reference",
        "metric": "decode tokens/s at L=128K (whole model = per-layer step x sparse layers)",
        "value": round(value, 6), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_layer * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 with planted hot 16-token blocks)",
        "config": {"workload": args.workload, "sel_fmt": args.sel_fmt, "sample": sample},
        "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s",
                         "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_reference_prefill(args, world, rank):
    """Reference arm for the sparse-prefill workloads: the fp64 oracle's
    prefill on the host cores, one tile (all KV heads) per step at tiles
    spread evenly over the chunk (at most 8 timed tiles, so the run stays
    bounded); the layer time is the mean tile time x the layer's tiles."""
    if rank != 0:
        return None
    import oracle
    wl = workloads.make_prefill(args.workload, seed=0, device="cpu")
    fmt = args.sel_fmt
    sp = wl.spec
    lens, ql = wl.seq_lens.numpy(), wl.q_lens.numpy()
    nt = len(oracle.prefill_tiles(lens, ql))
    sh = oracle.make_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, 128, 64, 64, fmt,
                           wl.num_pages, wl.max_blocks)
    pr = oracle.make_params(sink_blocks=sp.sink_blocks, recency_blocks=sp.recency_blocks,
                            kmin_blocks=sp.kmin_blocks)
    bits = workloads.bits(wl.sel_keys)
    sd, ss = (bits, None) if fmt == "bf16" else oracle.quantize_selector(fmt, bits)
    a = dict(q_sel=workloads.bits(wl.q_sel), w=None, sel_data=sd, sel_scales=ss,
             q=workloads.bits(wl.q), k_pool=workloads.bits(wl.k_pool),
             v_pool=workloads.bits(wl.v_pool), page_table=wl.page_table.numpy(), seq_lens=lens,
             q_lens=ql, top_p=wl.top_p.numpy(), sm_scale=wl.sm_scale)
    n = min(args.steps, 8)
    strata = [int((k + 0.5) * nt / n) for k in range(n)]
    for _ in range(args.warmup):                  # warm-up on the chunk's first (cheapest) tile
        oracle.prefill_step(sh, pr, tiles=[0], **a)
    times = []
    for t in strata:
        t0 = time.perf_counter()
        oracle.prefill_step(sh, pr, tiles=[t], **a)
        times.append(time.perf_counter() - t0)
    layer_s = float(np.mean(times)) * nt
    tokens = int(ql.sum())
    layers_model = sp_layers(args)
    value = tokens / (layer_s * layers_model)
    sample = (f"{n} tiles spread over the chunk's {nt} (all KV heads), one per step; "
              f"mean tile time x {nt} tiles x{layers_model} layers")
    return {
        "impl": "reference",
        "metric": "prefill tokens/s at L=32K (whole model = per-layer time x layers)",
        "value": round(value, 6), "unit": "tokens/s", "n_gpus": world, "steps": n,
        "warmup": args.warmup, "ms_per_step": round(layer_s * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 with planted hot blocks)",
        "config": {"workload": args.workload, "sel_fmt": fmt, "sample": sample},
        "cpu_baseline": {"value": round(value, 6), "unit": "tokens/s",
                         "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="spot", choices=["spot", "reference"])
    ap.add_argument("--workload", default="qwen3_32b_128k")
    ap.add_argument("--sel-fmt", default=None)
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per GPU (default: the workload's own); a smaller batch "
                         "keeps an ncu capture within a few GB of device memory")
    args = ap.parse_args()
    tok = args.workload in workloads.TOK_SPECS
    pf = args.workload in workloads.PREFILL_SPECS
    if args.sel_fmt is None:
        args.sel_fmt = "bf16" if (tok or pf) else workloads.SPECS[args.workload].sel_fmt
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            if world > 1:
                torch.distributed.barrier()
            res = (run_reference_tok if tok else
                   run_reference_prefill if pf else run_reference)(args, world, rank)
            if res is not None:
                print(json.dumps(res), flush=True)
            return
        if pf:
            res, layers = run_spot_prefill(args, world, rank, local)
        elif tok:
            res, layers = run_spot_tok(args, world, rank, local)
        else:
            res, layers = run_spot(args, world, rank, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                if pf:
                    res["cpu_baseline"] = cpu_baseline_prefill(layers[0][0], layers[1], layers[2],
                                                               sp_layers(args), args.sel_fmt)
                else:
                    res["cpu_baseline"] = (cpu_baseline_tok(layers[0][0], args.sel_fmt) if tok else
                                           cpu_baseline(layers[0][0], args.sel_fmt))
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
