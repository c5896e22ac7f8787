"""Seeded synthetic decode workloads for the SpotAttention hot path.

Shared by the tests, the smoke check and the benchmark: it produces INPUTS
only (query / key / value tensors, selector queries and bf16 selector keys,
paged-cache page tables, sequence lengths, per-sequence top-p) and holds none
of the method's arithmetic -- no scoring, softmax, selection, quantisation or
attention.  Quantised selector caches are produced by each side's own append
step (the CUDA library's ``append_selector_keys`` and the oracle's quantiser).

Shapes follow the decode workloads the SpotAttention paper measures (Qwen3 /
Qwen3.5 full-attention layers, contexts up to 128K; §4.2 Tab. 1, §5.3):

==================  =====  =======  =======  ==================  ========
name                batch  q / kv   context  selector keys       top-p
==================  =====  =======  =======  ==================  ========
tiny_4k             1      8 / 2    4096     bf16                0.9
qwen3_4b_32k        8      32 / 8   32768    bf16                0.95
qwen3_32b_128k      4      64 / 8   131072   bf16                0.95
quant_128k          16     32 / 8   131072   int4 or mxfp4       0.95
ragged_hybrid       32     32 / 8   U[8K,128K] ragged  mxfp4    {.9,.95,.99}
==================  =====  =======  =======  ==================  ========

head_dim 128, block (= page) 64 tokens, selector dim 64 everywhere.  Values
are N(0,1) rounded to bf16; per (sequence, KV head) some "hot" blocks get
their backbone keys and selector key shifted along the group's mean query
direction so the estimated attention is peaked (see ``_plant_hot``).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

HEAD_DIM = 128
BLOCK = 64
SEL_DIM = 64


@dataclasses.dataclass
class Spec:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seq_len: Optional[int]              # None -> ragged draw
    sel_fmt: str = "bf16"
    top_p: float = 0.95
    top_p_choices: Optional[tuple] = None
    sink_blocks: int = 1
    recency_blocks: int = 4
    kmin_blocks: int = 8
    hot: str = "logit"                  # "unit3" (fixed +3 u) or "logit" (U[2,4] logit offset)
    hot_count: int = 16
    hot_geometric_mean: Optional[float] = None
    page_order: str = "permuted"        # "contiguous" | "permuted"
    ragged_range: tuple = (8192, 131072)
    layers_total: int = 1               # layers of the model this layer stands for
    layers_sparse: int = 1              # of which use sparse selection


SPECS = {
    "tiny_4k": Spec("tiny_4k", 1, 8, 2, 4096, top_p=0.9, recency_blocks=2, hot="unit3",
                    hot_count=4, page_order="contiguous"),
    "qwen3_4b_32k": Spec("qwen3_4b_32k", 8, 32, 8, 32768, top_p=0.95, layers_total=36,
                         layers_sparse=36),
    "qwen3_32b_128k": Spec("qwen3_32b_128k", 4, 64, 8, 131072, top_p=0.95,
                           hot_geometric_mean=24.0, layers_total=64, layers_sparse=64),
    "quant_128k": Spec("quant_128k", 16, 32, 8, 131072, sel_fmt="int4", top_p=0.95,
                       layers_total=36, layers_sparse=36),
    "ragged_hybrid": Spec("ragged_hybrid", 32, 32, 8, None, sel_fmt="mxfp4",
                          top_p_choices=(0.9, 0.95, 0.99), layers_total=32, layers_sparse=8),
}


@dataclasses.dataclass
class Workload:
    spec: Spec
    seed: int
    seq_lens: torch.Tensor              # int32 [B]
    page_table: torch.Tensor            # int32 [B, max_blocks], -1 past each sequence
    num_pages: int
    q: torch.Tensor                     # bf16 [B, Hq, D]
    q_sel: torch.Tensor                 # bf16 [B, Hq, ds]
    w: Optional[torch.Tensor]           # fp32 [B, Hq] or None (uniform 1/G)
    sel_keys: torch.Tensor              # bf16 [num_pages, Hkv, ds]
    k_pool: torch.Tensor                # bf16 [num_pages, Hkv, BLOCK, D]
    v_pool: torch.Tensor                # bf16 [num_pages, Hkv, BLOCK, D]
    top_p: torch.Tensor                 # fp32 [B]
    hot_blocks: list                    # per (b, g): logical ids of planted blocks

    @property
    def batch(self):
        return self.spec.batch

    @property
    def num_q_heads(self):
        return self.spec.num_q_heads

    @property
    def num_kv_heads(self):
        return self.spec.num_kv_heads

    @property
    def max_blocks(self):
        return int(self.page_table.shape[1])

    @property
    def sm_scale(self):
        return 1.0 / math.sqrt(HEAD_DIM)


def _normal_bf16(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def _int_bf16(shape, gen, device, lo=-3, hi=3):
    return torch.randint(lo, hi + 1, shape, generator=gen, device=device).to(torch.bfloat16)


def make(name: str, seed: int = 0, device="cpu", *, seq_len=None, batch=None, sel_fmt=None,
         integer: bool = False, top_p=None, max_blocks=None, structure_from=None,
         **spec_overrides) -> Workload:
    """Build a seeded workload.  Overrides shrink a spec for oracle-sized
    runs (seq_len, batch) or switch its selector format; integer=True draws
    selector queries and keys from {-3..3} (exact scores in any precision).
    structure_from=<Workload> reuses that workload's sequence lengths, page
    table and top-p (another layer of the same model) and draws new data."""
    spec = dataclasses.replace(SPECS[name], **spec_overrides)
    if seq_len is not None:
        spec = dataclasses.replace(spec, seq_len=seq_len)
    if batch is not None:
        spec = dataclasses.replace(spec, batch=batch)
    if sel_fmt is not None:
        spec = dataclasses.replace(spec, sel_fmt=sel_fmt)
    if top_p is not None:
        spec = dataclasses.replace(spec, top_p=top_p, top_p_choices=None)
    device = torch.device(device)
    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    B, Hq, Hkv = spec.batch, spec.num_q_heads, spec.num_kv_heads
    if structure_from is not None:
        lens = structure_from.seq_lens.cpu().numpy().astype(np.int64)
    elif spec.seq_len is None:
        lo, hi = spec.ragged_range
        lens = rng.integers(lo // BLOCK, hi // BLOCK + 1, size=B) * BLOCK
    else:
        lens = np.full(B, spec.seq_len, np.int64)
    nbs = (lens + BLOCK - 1) // BLOCK
    mb = int(max(nbs.max() if B else 0, 1)) if max_blocks is None else int(max_blocks)
    num_pages = int(max(nbs.sum(), 1))
    pages = np.arange(num_pages) if spec.page_order == "contiguous" else rng.permutation(num_pages)
    pt = np.full((B, mb), -1, np.int32)
    off = 0
    for b in range(B):
        pt[b, :nbs[b]] = pages[off:off + nbs[b]]
        off += nbs[b]
    if structure_from is not None:
        pt = structure_from.page_table.cpu().numpy()
        num_pages = structure_from.num_pages

    if structure_from is not None:
        p = structure_from.top_p.cpu().numpy()
    elif spec.top_p_choices:
        p = rng.choice(np.asarray(spec.top_p_choices, np.float32), size=B)
    else:
        p = np.full(B, spec.top_p, np.float32)

    q = _normal_bf16((B, Hq, HEAD_DIM), gen, device)
    if integer:
        q_sel = _int_bf16((B, Hq, SEL_DIM), gen, device)
        sel_keys = _int_bf16((num_pages, Hkv, SEL_DIM), gen, device)
    else:
        q_sel = _normal_bf16((B, Hq, SEL_DIM), gen, device)
        sel_keys = _normal_bf16((num_pages, Hkv, SEL_DIM), gen, device)
    k_pool = _normal_bf16((num_pages, Hkv, BLOCK, HEAD_DIM), gen, device)
    v_pool = _normal_bf16((num_pages, Hkv, BLOCK, HEAD_DIM), gen, device)

    wl = Workload(spec, seed, torch.as_tensor(lens, dtype=torch.int32, device=device),
                  torch.as_tensor(pt, device=device), num_pages, q, q_sel, None, sel_keys,
                  k_pool, v_pool, torch.as_tensor(p, device=device), [])
    _plant_hot(wl, rng, integer)
    return wl


def _plant_hot(wl: Workload, rng, integer: bool):
    """Shift the keys of some blocks along the GQA group's mean query
    direction u (unit vector of the sum of the group's queries).

    "unit3": selector key and every backbone key of the block get +3.0 u.
    "logit": an offset o ~ U[2, 4] per block; the selector key gets c u with
    c = o * G / |sum_h q_sel_h| (so the mean over the group of q_h . key rises
    by o), the backbone keys get c' u with c' = o * G * sqrt(D) / |sum_h q_h|
    (the mean scaled logit rises by o).  Integer workloads instead set the
    selector key to 3 * sign(sum_h q_sel_h), keeping it integer.
    Hot blocks avoid the sink and recency blocks."""
    spec = wl.spec
    B, Hkv = spec.batch, spec.num_kv_heads
    G = spec.num_q_heads // Hkv
    qs = wl.q_sel.float().view(B, Hkv, G, SEL_DIM).sum(2)
    qk = wl.q.float().view(B, Hkv, G, HEAD_DIM).sum(2)
    pt = wl.page_table.cpu().numpy()
    lens = wl.seq_lens.cpu().numpy()
    for b in range(B):
        nb = int((lens[b] + BLOCK - 1) // BLOCK)
        lo, hi = spec.sink_blocks, nb - spec.recency_blocks
        cand = np.arange(max(lo, 0), max(hi, 0))
        for g in range(Hkv):
            if spec.hot_geometric_mean:
                n_hot = int(rng.geometric(1.0 / spec.hot_geometric_mean))
            else:
                n_hot = spec.hot_count
            n_hot = min(n_hot, cand.size)
            hot = np.sort(rng.choice(cand, size=n_hot, replace=False)) if n_hot else cand[:0]
            wl.hot_blocks.append(hot.tolist())
            if n_hot == 0:
                continue
            if spec.hot == "unit3":
                o = np.full(n_hot, 3.0)
            else:
                o = rng.uniform(2.0, 4.0, size=n_hot)
            pages = torch.as_tensor(pt[b, hot].astype(np.int64), device=wl.q.device)
            nsel, nkv = qs[b, g].norm(), qk[b, g].norm()
            u_sel, u_kv = qs[b, g] / nsel, qk[b, g] / nkv
            o_t = torch.as_tensor(o, dtype=torch.float32, device=wl.q.device)
            if integer:
                new_sel = (3.0 * torch.sign(qs[b, g])).expand(n_hot, SEL_DIM)
            elif spec.hot == "unit3":
                new_sel = wl.sel_keys[pages, g].float() + 3.0 * u_sel
            else:
                c = o_t * G / nsel
                new_sel = wl.sel_keys[pages, g].float() + c[:, None] * u_sel
            wl.sel_keys[pages, g] = new_sel.to(torch.bfloat16)
            if spec.hot == "unit3":
                ck = torch.full_like(o_t, 3.0)
            else:
                ck = o_t * G * math.sqrt(HEAD_DIM) / nkv
            new_k = wl.k_pool[pages, g].float() + ck[:, None, None] * u_kv
            wl.k_pool[pages, g] = new_k.to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 / fp16 tensor as a host numpy array."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def gather_units(wl: Workload, seqs) -> Workload:
    """A smaller workload holding only the sequences `seqs` and the pool
    pages they reference (pages renumbered densely, order kept).  Used to
    hand a full-size problem's sampled sequences to a CPU checker."""
    seqs = list(seqs)
    pt = wl.page_table[seqs]
    used = pt[pt >= 0].unique(sorted=True)
    remap = torch.full((wl.num_pages,), -1, dtype=torch.int32, device=pt.device)
    remap[used.long()] = torch.arange(used.numel(), dtype=torch.int32, device=pt.device)
    new_pt = torch.where(pt >= 0, remap[pt.clamp(min=0).long()], pt)
    idx = used.long()
    spec = dataclasses.replace(wl.spec, batch=len(seqs))
    return Workload(spec, wl.seed, wl.seq_lens[seqs].clone(), new_pt.contiguous(),
                    int(used.numel()), wl.q[seqs].contiguous(), wl.q_sel[seqs].contiguous(),
                    None if wl.w is None else wl.w[seqs].contiguous(),
                    wl.sel_keys[idx].contiguous(), wl.k_pool[idx].contiguous(),
                    wl.v_pool[idx].contiguous(), wl.top_p[seqs].contiguous(),
                    [wl.hot_blocks[b * wl.num_kv_heads + g] for b in seqs
                     for g in range(wl.num_kv_heads)])


# --------------------------------------------------------------------------
# Token-level, layer-shared selector (SpotAttention §2.1 and App. A Tab. 3 as
# written: H_idx = 4 index heads of width d_idx = 128 with per-token keys,
# blocks of 16 tokens scored by their maximum token score, one selection per
# query shared by every head of the layer).

TOK_PAGE = 64          # tokens per KV / selector page (the paged-cache page)


@dataclasses.dataclass
class TokSpec:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seq_len: Optional[int]              # None -> ragged draw
    idx_heads: int = 4
    idx_dim: int = 128
    sel_block: int = 16
    top_p: float = 0.9
    sink_blocks: int = 8                # 128 tokens (Tab. 3)
    recency_blocks: int = 16            # 256 tokens
    kmin_blocks: int = 32               # 512 tokens
    q_scale: float = 0.3                # selector query scale: ~40% of blocks at p = 0.9, 128K
    hot_count: int = 64                 # hot 16-token blocks per sequence
    page_order: str = "permuted"
    ragged_range: tuple = (8192, 131072)
    layers_total: int = 1
    layers_sparse: int = 1


TOK_SPECS = {
    "tok_tiny_2k": TokSpec("tok_tiny_2k", 1, 8, 2, 2048, hot_count=6, page_order="contiguous"),
    "qwen3_8b_128k_tok": TokSpec("qwen3_8b_128k_tok", 1, 32, 8, 131072, layers_total=36,
                                 layers_sparse=36),
}


@dataclasses.dataclass
class TokWorkload:
    spec: TokSpec
    seed: int
    seq_lens: torch.Tensor              # int32 [B]
    page_table: torch.Tensor            # int32 [B, max_pages], -1 past each sequence
    num_pages: int
    q: torch.Tensor                     # bf16 [B, Hq, D]
    q_idx: torch.Tensor                 # bf16 [B, H_idx, d_idx]
    w_idx: Optional[torch.Tensor]       # fp32 [B, H_idx] or None (uniform 1/H_idx)
    sel_tok: torch.Tensor               # bf16 [num_pages, TOK_PAGE, H_idx, d_idx]
    k_pool: torch.Tensor                # bf16 [num_pages, Hkv, TOK_PAGE, D]
    v_pool: torch.Tensor                # bf16 [num_pages, Hkv, TOK_PAGE, D]
    top_p: torch.Tensor                 # fp32 [B]
    hot_blocks: list                    # per b: logical ids of planted 16-token blocks

    @property
    def batch(self):
        return self.spec.batch

    @property
    def num_q_heads(self):
        return self.spec.num_q_heads

    @property
    def num_kv_heads(self):
        return self.spec.num_kv_heads

    @property
    def max_pages(self):
        return int(self.page_table.shape[1])

    @property
    def max_blocks(self):
        return self.max_pages * (TOK_PAGE // self.spec.sel_block)

    @property
    def sm_scale(self):
        return 1.0 / math.sqrt(HEAD_DIM)


def make_tok(name: str, seed: int = 0, device="cpu", *, seq_len=None, batch=None,
             integer: bool = False, top_p=None, uniform_w: bool = False,
             **spec_overrides) -> TokWorkload:
    """Seeded token-selector workload.  integer=True draws selector queries
    and keys from {-3..3} and uses uniform weights (exact scores in any
    precision)."""
    spec = dataclasses.replace(TOK_SPECS[name], **spec_overrides)
    if seq_len is not None:
        spec = dataclasses.replace(spec, seq_len=seq_len)
    if batch is not None:
        spec = dataclasses.replace(spec, batch=batch)
    if top_p is not None:
        spec = dataclasses.replace(spec, top_p=top_p)
    device = torch.device(device)
    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, Hq, Hkv, Hi, di = spec.batch, spec.num_q_heads, spec.num_kv_heads, spec.idx_heads, spec.idx_dim
    if spec.seq_len is None:
        lo, hi = spec.ragged_range
        lens = rng.integers(lo // spec.sel_block, hi // spec.sel_block + 1, size=B) * spec.sel_block
    else:
        lens = np.full(B, spec.seq_len, np.int64)
    npg = (lens + TOK_PAGE - 1) // TOK_PAGE
    mp = int(max(npg.max() if B else 0, 1))
    num_pages = int(max(npg.sum(), 1))
    pages = np.arange(num_pages) if spec.page_order == "contiguous" else rng.permutation(num_pages)
    pt = np.full((B, mp), -1, np.int32)
    off = 0
    for b in range(B):
        pt[b, :npg[b]] = pages[off:off + npg[b]]
        off += npg[b]
    p = np.full(B, spec.top_p, np.float32)

    q = _normal_bf16((B, Hq, HEAD_DIM), gen, device)
    if integer:
        q_idx = _int_bf16((B, Hi, di), gen, device)
        sel_tok = _int_bf16((num_pages, TOK_PAGE, Hi, di), gen, device)
        w_idx = None
    else:
        q_idx = (torch.randn((B, Hi, di), generator=gen, device=device) * spec.q_scale).to(
            torch.bfloat16)
        sel_tok = _normal_bf16((num_pages, TOK_PAGE, Hi, di), gen, device)
        w_idx = None if uniform_w else torch.as_tensor(
            rng.uniform(0.5, 1.5, size=(B, Hi)) / Hi, dtype=torch.float32, device=device)
    k_pool = _normal_bf16((num_pages, Hkv, TOK_PAGE, HEAD_DIM), gen, device)
    v_pool = _normal_bf16((num_pages, Hkv, TOK_PAGE, HEAD_DIM), gen, device)
    wl = TokWorkload(spec, seed, torch.as_tensor(lens, dtype=torch.int32, device=device),
                     torch.as_tensor(pt, device=device), num_pages, q, q_idx, w_idx, sel_tok,
                     k_pool, v_pool, torch.as_tensor(p, device=device), [])
    _plant_hot_tok(wl, rng, integer)
    return wl


def _plant_hot_tok(wl: TokWorkload, rng, integer: bool):
    """Per sequence, some 16-token blocks (outside the sink / recency blocks)
    get every token's selector key shifted along each index head's query
    direction by o / |q_h| (o ~ U[2, 4]: each head's dot rises by o, so the
    weighted token score rises by about o * sum_h w_h), and their backbone
    keys shifted along each KV group's summed query direction (the group's
    mean scaled logit rises by o).  Integer workloads set the hot tokens'
    selector keys to 3 * sign(q_h) instead."""
    spec = wl.spec
    B, Hkv, sb = spec.batch, spec.num_kv_heads, spec.sel_block
    G = spec.num_q_heads // Hkv
    per_page = TOK_PAGE // sb
    qk = wl.q.float().view(B, Hkv, G, HEAD_DIM).sum(2)
    pt = wl.page_table.cpu().numpy()
    lens = wl.seq_lens.cpu().numpy()
    dev = wl.q.device
    for b in range(B):
        nb = int((lens[b] + sb - 1) // sb)
        cand = np.arange(max(spec.sink_blocks, 0), max(nb - spec.recency_blocks, 0))
        n_hot = min(spec.hot_count, cand.size)
        hot = np.sort(rng.choice(cand, size=n_hot, replace=False)) if n_hot else cand[:0]
        wl.hot_blocks.append(hot.tolist())
        if n_hot == 0:
            continue
        o = torch.as_tensor(rng.uniform(2.0, 4.0, size=n_hot), dtype=torch.float32, device=dev)
        pages = torch.as_tensor(pt[b, hot // per_page].astype(np.int64), device=dev)
        slot0 = torch.as_tensor((hot % per_page) * sb, device=dev)
        slots = slot0[:, None] + torch.arange(sb, device=dev)[None, :]        # [n_hot, sb]
        pg = pages[:, None].expand(-1, sb)
        qi = wl.q_idx[b].float()                                              # [Hi, di]
        if integer:
            new = (3.0 * torch.sign(qi))[None, None].expand(n_hot, sb, -1, -1)
        else:
            u = qi / qi.norm(dim=1, keepdim=True)
            c = o[:, None] / qi.norm(dim=1)[None, :]                          # [n_hot, Hi]
            new = wl.sel_tok[pg, slots].float() + c[:, None, :, None] * u[None, None]
        wl.sel_tok[pg, slots] = new.to(torch.bfloat16)
        for g in range(Hkv):
            nkv = qk[b, g].norm()
            ck = o * G * math.sqrt(HEAD_DIM) / nkv
            kk = wl.k_pool[pg, g, slots].float() + ck[:, None, None] * (qk[b, g] / nkv)
            wl.k_pool[pg, g, slots] = kk.to(torch.bfloat16)


# --------------------------------------------------------------------------
# Sparse prefill: a chunk of new queries per sequence (the last q_len of its
# seq_len cached tokens), selector keys per (block, KV head) as in decode.

@dataclasses.dataclass
class PrefillSpec:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    seq_len: int
    q_len: int
    top_p: float = 0.9
    sink_blocks: int = 1
    recency_blocks: int = 4
    kmin_blocks: int = 8
    hot_count: int = 16
    page_order: str = "permuted"
    q_scale: float = 0.12               # selector query scale: ~45% of a late tile's blocks
                                        # at p = 0.9 (the tile score is a max over 64 queries)


PREFILL_SPECS = {
    "prefill_tiny": PrefillSpec("prefill_tiny", 2, 8, 2, 1000, 300, hot_count=3,
                                page_order="contiguous"),
    "qwen3_8b_prefill_32k": PrefillSpec("qwen3_8b_prefill_32k", 1, 32, 8, 32768, 32768),
}


@dataclasses.dataclass
class PrefillWorkload:
    spec: PrefillSpec
    seed: int
    seq_lens: torch.Tensor              # int32 [B]
    q_lens: torch.Tensor                # int32 [B]
    page_table: torch.Tensor            # int32 [B, max_blocks]
    num_pages: int
    q: torch.Tensor                     # bf16 [rows, Hq, D]   (rows = sum of q_lens)
    q_sel: torch.Tensor                 # bf16 [rows, Hq, ds]
    w: Optional[torch.Tensor]           # fp32 [rows, Hq] or None (1/G)
    sel_keys: torch.Tensor              # bf16 [num_pages, Hkv, ds]
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    top_p: torch.Tensor                 # fp32 [B]

    @property
    def batch(self):
        return self.spec.batch

    @property
    def num_q_heads(self):
        return self.spec.num_q_heads

    @property
    def num_kv_heads(self):
        return self.spec.num_kv_heads

    @property
    def max_blocks(self):
        return int(self.page_table.shape[1])

    @property
    def sm_scale(self):
        return 1.0 / math.sqrt(HEAD_DIM)


def make_prefill(name: str, seed: int = 0, device="cpu", *, seq_lens=None, q_lens=None,
                 batch=None, integer: bool = False, top_p=None, **spec_overrides):
    """Seeded prefill workload.  seq_lens / q_lens (lists) override the
    spec's uniform ones; integer=True draws selector queries and keys from
    {-3..3}."""
    spec = dataclasses.replace(PREFILL_SPECS[name], **spec_overrides)
    if batch is not None:
        spec = dataclasses.replace(spec, batch=batch)
    if top_p is not None:
        spec = dataclasses.replace(spec, top_p=top_p)
    device = torch.device(device)
    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, Hq, Hkv = spec.batch, spec.num_q_heads, spec.num_kv_heads
    lens = np.array(seq_lens if seq_lens is not None else [spec.seq_len] * B, np.int64)
    qls = np.array(q_lens if q_lens is not None else [spec.q_len] * B, np.int64)
    B = len(lens)
    spec = dataclasses.replace(spec, batch=B)
    nbs = (lens + BLOCK - 1) // BLOCK
    mb = int(max(nbs.max() if B else 0, 1))
    num_pages = int(max(nbs.sum(), 1))
    pages = np.arange(num_pages) if spec.page_order == "contiguous" else rng.permutation(num_pages)
    pt = np.full((B, mb), -1, np.int32)
    off = 0
    for b in range(B):
        pt[b, :nbs[b]] = pages[off:off + nbs[b]]
        off += nbs[b]
    rows = int(qls.sum())
    q = _normal_bf16((rows, Hq, HEAD_DIM), gen, device)
    if integer:
        q_sel = _int_bf16((rows, Hq, SEL_DIM), gen, device)
        sel_keys = _int_bf16((num_pages, Hkv, SEL_DIM), gen, device)
    else:
        q_sel = (torch.randn((rows, Hq, SEL_DIM), generator=gen, device=device) *
                 spec.q_scale).to(torch.bfloat16)
        sel_keys = _normal_bf16((num_pages, Hkv, SEL_DIM), gen, device)
    k_pool = _normal_bf16((num_pages, Hkv, BLOCK, HEAD_DIM), gen, device)
    v_pool = _normal_bf16((num_pages, Hkv, BLOCK, HEAD_DIM), gen, device)
    wl = PrefillWorkload(spec, seed, torch.as_tensor(lens, dtype=torch.int32, device=device),
                         torch.as_tensor(qls, dtype=torch.int32, device=device),
                         torch.as_tensor(pt, device=device), num_pages, q, q_sel, None, sel_keys,
                         k_pool, v_pool,
                         torch.full((B,), spec.top_p, dtype=torch.float32, device=device))
    # hot blocks per (sequence, KV head) along the chunk's mean query direction
    G = Hq // Hkv
    row = 0
    for b in range(B):
        nb = int(nbs[b])
        cand = np.arange(spec.sink_blocks, max(nb - spec.recency_blocks, spec.sink_blocks))
        rows_b = slice(row, row + int(qls[b]))
        row += int(qls[b])
        if cand.size == 0 or qls[b] == 0:
            continue
        qs = q_sel[rows_b].float().view(-1, Hkv, G, SEL_DIM).sum((0, 2))
        qk = q[rows_b].float().view(-1, Hkv, G, HEAD_DIM).sum((0, 2))
        for g in range(Hkv):
            n_hot = min(spec.hot_count, cand.size)
            hot = np.sort(rng.choice(cand, size=n_hot, replace=False))
            o = torch.as_tensor(rng.uniform(2.0, 4.0, size=n_hot), dtype=torch.float32,
                                device=device)
            pg = torch.as_tensor(pt[b, hot].astype(np.int64), device=device)
            us, uk = qs[g] / qs[g].norm(), qk[g] / qk[g].norm()
            if integer:
                wl.sel_keys[pg, g] = (3.0 * torch.sign(qs[g])).expand(n_hot, SEL_DIM).to(
                    torch.bfloat16)
            else:
                wl.sel_keys[pg, g] = (wl.sel_keys[pg, g].float() +
                                      (o * 8.0)[:, None] * us).to(torch.bfloat16)
            wl.k_pool[pg, g] = (wl.k_pool[pg, g].float() +
                                (o * math.sqrt(HEAD_DIM) / 4.0)[:, None, None] * uk).to(
                                    torch.bfloat16)
    return wl
