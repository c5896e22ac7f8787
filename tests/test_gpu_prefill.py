"""GPU parity of the sparse-prefill path (query tiles of one KV block select
like a decode query at the tile's end from block scores maxed over the
tile's queries; causal attention over the selection) through the C ABI,
against the fp64 oracle.  Rules and tolerances: tests/harness.py."""
import numpy as np
import pytest
import torch

import block_sparse_long_spot_b200 as spot
import oracle
import workloads
from harness import (ATOL, RTOL, P_ROUND, check_prefill_outputs,
                     check_prefill_selection_near_cut, oracle_prefill_scores,
                     prefill_weighted_abs_v, prefill_oracle_args, run_gpu_prefill,
                     run_oracle_prefill, safe_top_p_prefill, tile_selection)

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
    assert gpu["num_tiles"] == len(ora["tiles"])
    assert np.array_equal(gpu["sel_cnt"], ora["sel_cnt"]), (gpu["sel_cnt"], ora["sel_cnt"])
    for t in range(gpu["num_tiles"]):
        for g in range(wl.num_kv_heads):
            assert tile_selection(gpu, t, g) == tile_selection(ora, t, g), (t, g)


def test_prefill_tiny():
    wl = workloads.make_prefill("prefill_tiny", seed=0, device=DEV)
    gpu = run_gpu_prefill(wl)
    assert gpu["status"] == 0
    args = prefill_oracle_args(wl)
    ora = run_oracle_prefill(wl, args=args)
    scores = oracle_prefill_scores(wl, args=args)
    assert check_prefill_selection_near_cut(gpu, ora, scores, wl) <= 1
    _, n = check_prefill_outputs(gpu, ora, wl)
    assert n >= gpu["num_tiles"] * wl.num_kv_heads - 1


def test_prefill_worst_rows_within_the_bf16_weight_bound():
    # Whole sequences prefilled from position 0: the first rows attend 1, 2,
    # ... keys, where rounding the softmax weights to bf16 weighs most.
    # Every element must lie within 2e-3 + 1e-2 |ref| + 2^-9 sum_i w_i |v_i|
    # (reading r21), and rows attending at least 256 keys within the plain
    # decode rule 2e-3 + 1e-2 |ref|.
    wl = workloads.make_prefill("prefill_tiny", seed=7, device=DEV, integer=True,
                                seq_lens=[640, 130, 64], q_lens=[640, 130, 64])
    wl.top_p = safe_top_p_prefill(wl)
    gpu = run_gpu_prefill(wl)
    assert gpu["status"] == 0
    ora = run_oracle_prefill(wl)
    _same(gpu, ora, wl)
    info = oracle.prefill_tiles(wl.seq_lens.cpu().numpy(), wl.q_lens.cpu().numpy())
    G = wl.num_q_heads // wl.num_kv_heads
    worst_extra = 0.0
    for t, (b, lo, hi, r0) in enumerate(info):
        rows = slice(r0, r0 + hi - lo + 1)
        for g in range(wl.num_kv_heads):
            hs = slice(g * G, (g + 1) * G)
            o_g, o_r = gpu["out"][rows, hs], ora["out"][rows, hs]
            err = np.abs(o_g - o_r)
            plain = ATOL + RTOL * np.abs(o_r)
            assert (err <= plain + P_ROUND * prefill_weighted_abs_v(wl, ora, t, g)).all(), (t, g)
            sel = ora["sel_idx"][t, g, :ora["sel_cnt"][t, g]]
            keys = np.array([sum(min(64, max(0, pos - 64 * j + 1)) for j in sel)
                             for pos in range(lo, hi + 1)])
            many = keys >= 256
            assert (err[many] <= plain[many]).all(), (t, g)
            worst_extra = max(worst_extra, float((err - plain).max()))
    print(f"largest excess over the decode rule: {worst_extra:.2e}")


@pytest.mark.parametrize("lens,qlens", [
    ([1000, 1000], [300, 300]),
    ([777, 64, 129, 2048, 5], [777, 1, 70, 200, 5]),
])
def test_prefill_integer_inputs_select_bit_exact(lens, qlens):
    wl = workloads.make_prefill("prefill_tiny", seed=3, device=DEV, integer=True, seq_lens=lens,
                                q_lens=qlens)
    wl.top_p = safe_top_p_prefill(wl)
    gpu = run_gpu_prefill(wl)
    assert gpu["status"] == 0
    ora = run_oracle_prefill(wl)
    _same(gpu, ora, wl)
    check_prefill_outputs(gpu, ora, wl)


def test_prefill_keep_all_and_modes():
    wl = workloads.make_prefill("prefill_tiny", seed=4, device=DEV, integer=True,
                                seq_lens=[900, 300], q_lens=[250, 300])
    for kw in (dict(mode="topk", topk=3), dict(kmin=12), dict(sink=100, rec=0),
               dict(mode="topk", topk=0, sink=0, rec=1)):
        gpu = run_gpu_prefill(wl, **kw)
        assert gpu["status"] == 0
        ora = run_oracle_prefill(wl, **kw)
        _same(gpu, ora, wl)
        check_prefill_outputs(gpu, ora, wl)
    wl.top_p = torch.ones_like(wl.top_p)          # p = 1: dense causal attention
    gpu = run_gpu_prefill(wl)
    ora = run_oracle_prefill(wl)
    _same(gpu, ora, wl)
    check_prefill_outputs(gpu, ora, wl)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 2), (12, 4)])
def test_prefill_group_sizes(hq, hkv):
    wl = workloads.make_prefill("prefill_tiny", seed=5, device=DEV, num_q_heads=hq,
                                num_kv_heads=hkv, seq_lens=[600], q_lens=[200])
    gpu = run_gpu_prefill(wl)
    assert gpu["status"] == 0
    args = prefill_oracle_args(wl)
    ora = run_oracle_prefill(wl, args=args)
    scores = oracle_prefill_scores(wl, args=args)
    assert check_prefill_selection_near_cut(gpu, ora, scores, wl) <= 1
    check_prefill_outputs(gpu, ora, wl)


def test_prefill_full_size_sampled_tiles():
    """Qwen3-8B layer, 32K-token prefill in the benchmark's launch
    configuration; selection and outputs of sampled tiles against the oracle."""
    wl = workloads.make_prefill("qwen3_8b_prefill_32k", seed=1, device=DEV)
    gpu = run_gpu_prefill(wl)
    assert gpu["status"] == 0
    nt = gpu["num_tiles"]
    tiles = [0, 3, nt // 2, nt - 2, nt - 1]
    args = prefill_oracle_args(wl)
    ora = run_oracle_prefill(wl, tiles=tiles, args=args)
    scores = oracle_prefill_scores(wl, tiles=tiles, args=args)
    n_diff = check_prefill_selection_near_cut(gpu, ora, scores, wl, tiles=tiles)
    assert n_diff <= 1
    frac = [gpu["sel_cnt"][t].mean() / (t + 1) for t in tiles]
    print("selected fraction of sampled tiles", np.round(frac, 3).tolist())
    _, n = check_prefill_outputs(gpu, ora, wl, tiles=tiles)
    assert n >= len(tiles) * wl.num_kv_heads - n_diff


def test_prefill_bad_page_id_and_small_max_tiles_are_reported():
    wl = workloads.make_prefill("prefill_tiny", seed=6, device=DEV)
    wl.page_table[0, 3] = wl.num_pages + 7
    gpu = run_gpu_prefill(wl)
    assert gpu["status"] == 5
    assert np.isfinite(gpu["out"]).all()
    wl = workloads.make_prefill("prefill_tiny", seed=6, device=DEV)
    gpu = run_gpu_prefill(wl, max_tiles=2)
    assert gpu["status"] == 5


# ------------------------------------------------ quantised selector keys / queries

@pytest.mark.parametrize("fmt,qq", [("mxfp4", False), ("fp8", False), ("mxfp4", True),
                                    ("fp8", True)])
def test_prefill_quantised_keys_integer_inputs_select_bit_exact(fmt, qq):
    # selector queries and keys in {-3..3}: MXFP4 and E4M3 store them
    # losslessly, so every tile score is exact on both sides
    wl = workloads.make_prefill("prefill_tiny", seed=7, device=DEV, integer=True,
                                seq_lens=[1000, 300], q_lens=[300, 300])
    wl.top_p = safe_top_p_prefill(wl, fmt=fmt, quantize_queries=qq)
    gpu = run_gpu_prefill(wl, fmt=fmt, quantize_queries=qq)
    assert gpu["status"] == 0
    ora = run_oracle_prefill(wl, fmt=fmt, quantize_queries=qq)
    _same(gpu, ora, wl)
    check_prefill_outputs(gpu, ora, wl)


@pytest.mark.parametrize("fmt,qq", [("int4", False), ("mxfp4", False), ("fp8", False),
                                    ("int8", False), ("int4", True), ("int8", True)])
def test_prefill_quantised_keys_tiny(fmt, qq):
    wl = workloads.make_prefill("prefill_tiny", seed=8, device=DEV)
    gpu = run_gpu_prefill(wl, fmt=fmt, quantize_queries=qq)
    assert gpu["status"] == 0
    args = prefill_oracle_args(wl, fmt)
    ora = run_oracle_prefill(wl, args=args, fmt=fmt, quantize_queries=qq)
    scores = oracle_prefill_scores(wl, args=args, fmt=fmt, quantize_queries=qq)
    assert check_prefill_selection_near_cut(gpu, ora, scores, wl) <= 1
    _, n = check_prefill_outputs(gpu, ora, wl)
    assert n >= gpu["num_tiles"] * wl.num_kv_heads - 1


def test_prefill_full_size_int4_keys_sampled_tiles():
    """The 32K-token prefill with INT4 selector keys (written by the library's
    quantising append) in the benchmark's launch configuration: selection and
    outputs of sampled tiles against the oracle on the same codes."""
    wl = workloads.make_prefill("qwen3_8b_prefill_32k", seed=4, device=DEV)
    gpu = run_gpu_prefill(wl, fmt="int4")
    assert gpu["status"] == 0
    nt = gpu["num_tiles"]
    tiles = [1, nt // 3, nt - 1]
    args = prefill_oracle_args(wl, "int4")
    ora = run_oracle_prefill(wl, tiles=tiles, args=args, fmt="int4")
    scores = oracle_prefill_scores(wl, tiles=tiles, args=args, fmt="int4")
    n_diff = check_prefill_selection_near_cut(gpu, ora, scores, wl, tiles=tiles)
    assert n_diff <= 1
    _, n = check_prefill_outputs(gpu, ora, wl, tiles=tiles)
    assert n >= len(tiles) * wl.num_kv_heads - n_diff
