"""GPU parity of the token-level, layer-shared selector path (per-token keys
of 4 index heads x 128, blocks of 16 tokens scored by their maximum token
score, one selection per sequence shared by every head) through the C ABI,
against the fp64 oracle.  Rules and tolerances: tests/harness.py."""
import numpy as np
import pytest
import torch

import block_sparse_long_spot_b200 as spot
import oracle
import workloads
from harness import (check_tok_outputs, check_tok_selection_near_cut, gpu_tok_pool,
                     oracle_tok_scores, run_gpu_tok, run_oracle_tok, safe_top_p_tok,
                     tok_oracle_args, tok_selection)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _same(gpu, ora, wl):
    assert np.array_equal(gpu["sel_cnt"], ora["sel_cnt"]), (gpu["sel_cnt"], ora["sel_cnt"])
    for b in range(wl.batch):
        assert tok_selection(gpu, b) == tok_selection(ora, b), b


@pytest.mark.parametrize("kmin", [32, 0])
def test_tok_tiny_decode_step(kmin):
    wl = workloads.make_tok("tok_tiny_2k", seed=0, device=DEV)
    gpu = run_gpu_tok(wl, kmin=kmin)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl)
    ora = run_oracle_tok(wl, args=args, kmin=kmin)
    scores = oracle_tok_scores(wl, args=args)
    assert check_tok_selection_near_cut(gpu, ora, scores, wl, kmin=kmin) == 0
    _, n = check_tok_outputs(gpu, ora, wl)
    assert n == wl.batch


INTEGER = [
    ("tok_tiny_2k", dict()),
    ("tok_tiny_2k", dict(batch=5, seq_len=None, ragged_range=(16, 4096))),
    ("qwen3_8b_128k_tok", dict(seq_len=16384, batch=3)),
]


@pytest.mark.parametrize("name,kw", INTEGER)
def test_tok_integer_inputs_select_bit_exact(name, kw):
    # Selector queries and keys in {-3..3}, uniform weights: every token and
    # block score is exact in fp32 and fp64, so the selections must match.
    wl = workloads.make_tok(name, seed=5, device=DEV, integer=True, **kw)
    wl.top_p = safe_top_p_tok(wl)
    gpu = run_gpu_tok(wl)
    assert gpu["status"] == 0
    ora = run_oracle_tok(wl)
    _same(gpu, ora, wl)
    check_tok_outputs(gpu, ora, wl)


def test_tok_topk_and_reserved_modes():
    wl = workloads.make_tok("tok_tiny_2k", seed=6, device=DEV, integer=True, batch=3,
                            seq_len=None, ragged_range=(64, 2048))
    for kw in (dict(mode="topk", topk=10), dict(mode="topk", topk=0, sink=0, rec=1),
               dict(kmin=200), dict(sink=300, rec=0)):
        gpu = run_gpu_tok(wl, **kw)
        assert gpu["status"] == 0
        ora = run_oracle_tok(wl, **kw)
        _same(gpu, ora, wl)
        check_tok_outputs(gpu, ora, wl)


def test_tok_ragged_partial_blocks_and_empty_sequences():
    wl = workloads.make_tok("tok_tiny_2k", seed=7, device=DEV, batch=7, seq_len=None,
                            ragged_range=(2048, 2048))
    lens = torch.tensor([0, 1, 15, 16, 17, 16 * 37 + 9, 2048], dtype=torch.int32)
    wl.seq_lens = lens.to(DEV)
    gpu = run_gpu_tok(wl)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl)
    ora = run_oracle_tok(wl, args=args)
    scores = oracle_tok_scores(wl, args=args)
    assert check_tok_selection_near_cut(gpu, ora, scores, wl) <= 1
    check_tok_outputs(gpu, ora, wl)
    assert gpu["sel_cnt"][0] == 0 and np.all(gpu["out"][0] == 0)
    assert np.all(np.isneginf(gpu["lse"][0]))


@pytest.mark.parametrize("dense", [True, False])
def test_tok_runs_of_slices_stop_at_page_blocks(dense):
    """One KV head and a contiguous page table put consecutive pages next to
    each other in the pool, so the 16-token slices of a run could run on into
    the next page: the attention must still match the oracle, with every
    block reserved (runs of four slices) and with the nucleus selection."""
    wl = workloads.make_tok("tok_tiny_2k", seed=9, device=DEV, batch=2, num_q_heads=8,
                            num_kv_heads=1, page_order="contiguous")
    kw = dict(sink=300, rec=0) if dense else {}
    gpu = run_gpu_tok(wl, **kw)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl)
    ora = run_oracle_tok(wl, args=args, **kw)
    if dense:
        _same(gpu, ora, wl)
        n_diff = 0
    else:
        scores = oracle_tok_scores(wl, args=args)
        n_diff = check_tok_selection_near_cut(gpu, ora, scores, wl)
        assert n_diff <= 1
    _, n = check_tok_outputs(gpu, ora, wl)
    assert n >= wl.batch - n_diff


@pytest.mark.parametrize("batch,seq_len", [(1, 131072), (2, None)])
def test_tok_full_size(batch, seq_len):
    """Qwen3-8B layer at 128K (and two ragged sequences): the selection of
    every sequence checked on the oracle's scores, every head's attention
    output against the oracle."""
    kw = dict(batch=batch)
    if seq_len is None:
        kw.update(seq_len=None, ragged_range=(60000, 131072))
    wl = workloads.make_tok("qwen3_8b_128k_tok", seed=1, device=DEV, **kw)
    gpu = run_gpu_tok(wl)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl)
    ora = run_oracle_tok(wl, args=args)
    scores = oracle_tok_scores(wl, args=args)
    n_diff = check_tok_selection_near_cut(gpu, ora, scores, wl)
    assert n_diff <= 1
    frac = gpu["sel_cnt"] / np.maximum(1, (wl.seq_lens.cpu().numpy() + 15) // 16)
    print(f"|S|/nb {frac.tolist()}, near-cut differences {n_diff}")
    _, n = check_tok_outputs(gpu, ora, wl)
    assert n >= wl.batch - n_diff


def test_tok_append_writes_the_pool():
    wl = workloads.make_tok("tok_tiny_2k", seed=8, device=DEV, batch=3, seq_len=None,
                            ragged_range=(100, 2048))
    desc = spot.tok_layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages)
    pool, _ = spot.tok_selector_pool(wl.num_pages, device=DEV)
    lens = wl.seq_lens.cpu().numpy()
    pt = wl.page_table.cpu().numpy()
    seq_ids = np.concatenate([np.full(lens[b], b) for b in range(wl.batch)]).astype(np.int32)
    pos = np.concatenate([np.arange(lens[b]) for b in range(wl.batch)]).astype(np.int32)
    perm = np.random.default_rng(0).permutation(seq_ids.size)
    seq_ids, pos = seq_ids[perm], pos[perm]
    pages = pt[seq_ids, pos // 64]
    keys = wl.sel_tok[torch.as_tensor(pages).long().to(DEV), torch.as_tensor(pos % 64).long().to(DEV)]
    ws = spot.new_tok_workspace(desc, wl.batch, wl.max_blocks, DEV)
    spot.tok_append_selector_keys(desc, pool, None, wl.page_table,
                                  torch.as_tensor(seq_ids).to(DEV),
                                  torch.as_tensor(pos).to(DEV), keys.contiguous(), ws)
    torch.cuda.synchronize()
    assert spot.read_device_status(ws) == 0
    written = torch.zeros(wl.num_pages, 64, dtype=torch.bool)
    written[torch.as_tensor(pages).long(), torch.as_tensor(pos % 64).long()] = True
    a = pool.cpu().view(torch.int16)
    b = wl.sel_tok.cpu().view(torch.int16)
    assert torch.equal(a[written], b[written])
    assert (a[~written] == 0).all()
    # a bad position / sequence is skipped and reported
    bad = torch.tensor([wl.batch, 0], dtype=torch.int32, device=DEV)
    badpos = torch.tensor([0, 64 * wl.max_pages], dtype=torch.int32, device=DEV)
    spot.tok_append_selector_keys(desc, pool, None, wl.page_table, bad, badpos,
                                  keys[:2].contiguous(),
                                  ws)
    torch.cuda.synchronize()
    assert spot.read_device_status(ws) == 5              # SPOT_ERR_DEVICE_BOUNDS
    assert torch.equal(pool.cpu().view(torch.int16)[written], b[written])


def test_tok_bad_selection_is_reported_not_faulted():
    wl = workloads.make_tok("tok_tiny_2k", seed=9, device=DEV)
    desc = spot.tok_layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages)
    ws = spot.new_tok_workspace(desc, 1, wl.max_blocks, DEV)
    sel_idx = torch.tensor([[0, 5, 10_000, 7] + [-1] * (wl.max_blocks - 4)], dtype=torch.int32,
                           device=DEV)
    sel_cnt = torch.tensor([4], dtype=torch.int32, device=DEV)
    out = torch.empty(1, wl.num_q_heads, 128, dtype=torch.float32, device=DEV)
    spot.tok_sparse_decode(desc, wl.q, wl.k_pool, wl.v_pool, wl.page_table, wl.seq_lens,
                           sel_idx, sel_cnt, wl.sm_scale, out, None, ws)
    torch.cuda.synchronize()
    assert spot.read_device_status(ws) == 5
    assert torch.isfinite(out).all()


# ------------------------------------------------ quantised per-token keys

QFMTS = ["int4", "mxfp4", "fp8", "int8"]


@pytest.mark.parametrize("fmt", QFMTS)
def test_tok_append_quantises_like_the_oracle(fmt):
    wl = workloads.make_tok("tok_tiny_2k", seed=12, device=DEV, batch=2, seq_len=None,
                            ragged_range=(700, 2048))
    desc = spot.tok_layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, sel_fmt=fmt)
    data, scales = gpu_tok_pool(wl, fmt, desc)
    ref_d, ref_s = oracle.quantize_selector(fmt, workloads.bits(wl.sel_tok))
    lens = wl.seq_lens.cpu().numpy()
    pt = wl.page_table.cpu().numpy()
    rows = np.zeros(wl.num_pages * 64, bool)          # (page, slot) rows that were appended
    for b, L in enumerate(lens):
        for t in range(int(L)):
            rows[pt[b, t // 64] * 64 + t % 64] = True
    gd = data.cpu().view(torch.uint8).numpy().reshape(wl.num_pages * 64, -1)
    assert np.array_equal(gd[rows], ref_d.view(np.uint8).reshape(wl.num_pages * 64, -1)[rows])
    if ref_s is not None:
        gs = scales.cpu()
        gs = (gs.view(torch.int16).numpy().view(np.uint16) if gs.dtype == torch.float16
              else gs.numpy()).reshape(wl.num_pages * 64, -1)
        assert np.array_equal(gs[rows], ref_s.reshape(wl.num_pages * 64, -1)[rows])


@pytest.mark.parametrize("fmt", QFMTS)
def test_tok_quantised_keys_tiny(fmt):
    wl = workloads.make_tok("tok_tiny_2k", seed=13, device=DEV)
    gpu = run_gpu_tok(wl, fmt=fmt)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl, fmt)
    ora = run_oracle_tok(wl, args=args, fmt=fmt)
    scores = oracle_tok_scores(wl, args=args, fmt=fmt)
    assert check_tok_selection_near_cut(gpu, ora, scores, wl) <= 1
    _, n = check_tok_outputs(gpu, ora, wl)
    assert n >= wl.batch - 1


@pytest.mark.parametrize("fmt", ["mxfp4", "fp8"])
def test_tok_quantised_integer_keys_select_bit_exact(fmt):
    # keys in {-3..3} are stored losslessly by MXFP4 (power-of-two group
    # scales) and E4M3: every score stays exact on both sides
    wl = workloads.make_tok("tok_tiny_2k", seed=14, device=DEV, integer=True, batch=3,
                            seq_len=None, ragged_range=(64, 4096))
    wl.top_p = safe_top_p_tok(wl, fmt=fmt)
    gpu = run_gpu_tok(wl, fmt=fmt)
    assert gpu["status"] == 0
    ora = run_oracle_tok(wl, fmt=fmt)
    _same(gpu, ora, wl)
    check_tok_outputs(gpu, ora, wl)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4"])
def test_tok_quantised_keys_full_size(fmt):
    wl = workloads.make_tok("qwen3_8b_128k_tok", seed=2, device=DEV)
    gpu = run_gpu_tok(wl, fmt=fmt)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl, fmt)
    ora = run_oracle_tok(wl, args=args, fmt=fmt)
    scores = oracle_tok_scores(wl, args=args, fmt=fmt)
    assert check_tok_selection_near_cut(gpu, ora, scores, wl) <= 1
    check_tok_outputs(gpu, ora, wl)


@pytest.mark.parametrize("fmt", ["mxfp4", "fp8"])
def test_tok_every_e2m1_magnitude_bit_exact(fmt):
    # Keys over {0, +-1/4, +-1/2, +-3/4, +-1, +-3/2, +-2, +-3} (the planted +-3
    # kept): each MXFP4 group's codes are exact -- all eight E2M1 magnitudes
    # occur, the zero-exponent 0.5 among them -- and so are the E4M3 codes;
    # with integer queries every score is exact in any precision, so the
    # selections must match the oracle's.
    wl = workloads.make_tok("tok_tiny_2k", seed=16, device=DEV, integer=True, batch=3,
                            seq_len=None, ragged_range=(64, 4096))
    vals = torch.tensor([0.0, 0.25, 0.5, 0.75, 1.0, 1.5, 2.0, 3.0], device=DEV)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(16)
    mag = vals[torch.randint(0, 8, wl.sel_tok.shape, generator=gen, device=DEV)]
    sign = torch.where(torch.rand(wl.sel_tok.shape, generator=gen, device=DEV) < 0.5, -1.0, 1.0)
    keep = wl.sel_tok.float().abs() == 3
    wl.sel_tok = torch.where(keep, wl.sel_tok.float(), mag * sign).to(torch.bfloat16)
    wl.top_p = safe_top_p_tok(wl, fmt=fmt)
    gpu = run_gpu_tok(wl, fmt=fmt)
    assert gpu["status"] == 0
    ora = run_oracle_tok(wl, fmt=fmt)
    _same(gpu, ora, wl)
    check_tok_outputs(gpu, ora, wl)


# ------------------------------------------------ quantised index-head queries

@pytest.mark.parametrize("fmt", ["mxfp4", "fp8"])
def test_tok_quantised_queries_integer_inputs_bit_exact(fmt):
    # queries and keys in {-3..3}: MXFP4 and E4M3 store them losslessly, so the
    # scores are exact on both sides and the selections must match
    wl = workloads.make_tok("tok_tiny_2k", seed=17, device=DEV, integer=True, batch=3,
                            seq_len=None, ragged_range=(64, 4096))
    wl.top_p = safe_top_p_tok(wl, fmt=fmt, quantize_queries=True)
    gpu = run_gpu_tok(wl, fmt=fmt, quantize_queries=True)
    assert gpu["status"] == 0
    ora = run_oracle_tok(wl, fmt=fmt, quantize_queries=True)
    _same(gpu, ora, wl)
    check_tok_outputs(gpu, ora, wl)


@pytest.mark.parametrize("fmt", QFMTS)
def test_tok_quantised_queries_tiny(fmt):
    wl = workloads.make_tok("tok_tiny_2k", seed=18, device=DEV)
    gpu = run_gpu_tok(wl, fmt=fmt, quantize_queries=True)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl, fmt)
    ora = run_oracle_tok(wl, args=args, fmt=fmt, quantize_queries=True)
    scores = oracle_tok_scores(wl, args=args, fmt=fmt, quantize_queries=True)
    assert check_tok_selection_near_cut(gpu, ora, scores, wl) <= 1
    _, n = check_tok_outputs(gpu, ora, wl)
    assert n >= wl.batch - 1


def test_tok_quantised_queries_full_size_int4():
    wl = workloads.make_tok("qwen3_8b_128k_tok", seed=3, device=DEV)
    gpu = run_gpu_tok(wl, fmt="int4", quantize_queries=True)
    assert gpu["status"] == 0
    args = tok_oracle_args(wl, "int4")
    ora = run_oracle_tok(wl, args=args, fmt="int4", quantize_queries=True)
    scores = oracle_tok_scores(wl, args=args, fmt="int4", quantize_queries=True)
    assert check_tok_selection_near_cut(gpu, ora, scores, wl) <= 1
    check_tok_outputs(gpu, ora, wl)
