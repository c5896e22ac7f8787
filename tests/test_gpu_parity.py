"""GPU parity of the CUDA decode path (through the C ABI) against the fp64
oracle, on the seeded workloads of the SpotAttention decode configurations
and on edge cases.  Rules and tolerances: tests/harness.py."""
import math
import time

import numpy as np
import pytest
import torch

import block_sparse_long_spot_b200 as spot
import oracle
import workloads
from harness import (check_outputs, check_selection_near_cut, gpu_selector_pool, oracle_args,
                     oracle_scores, oracle_selector_pool, run_gpu, run_oracle, safe_top_p,
                     unit_selection)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _assert_same_selection(gpu, ora, wl):
    assert np.array_equal(gpu["sel_cnt"], ora["sel_cnt"]), (gpu["sel_cnt"], ora["sel_cnt"])
    for b in range(wl.batch):
        for g in range(wl.num_kv_heads):
            assert unit_selection(gpu, b, g) == unit_selection(ora, b, g), (b, g)


# ------------------------------------------------------------ small, whole

@pytest.mark.parametrize("kmin", [8, 0])
def test_tiny_decode_step(kmin):
    wl = workloads.make("tiny_4k", seed=0, device=DEV)
    gpu = run_gpu(wl, kmin=kmin)
    assert gpu["status"] == 0
    ora = run_oracle(wl, kmin=kmin)
    n_diff = check_selection_near_cut(gpu, ora, oracle_scores(wl), wl, kmin=kmin)
    assert n_diff == 0
    check_outputs(gpu, ora, wl)


INTEGER_CASES = [
    ("tiny_4k", dict(), "bf16"),
    ("qwen3_4b_32k", dict(seq_len=8192), "bf16"),
    ("qwen3_32b_128k", dict(seq_len=16384, batch=2), "bf16"),
    ("quant_128k", dict(seq_len=8192, batch=4), "mxfp4"),
    ("quant_128k", dict(seq_len=8192, batch=4), "fp8"),
    ("ragged_hybrid", dict(batch=8, ragged_range=(512, 8192)), "bf16"),
]


@pytest.mark.parametrize("name,kw,fmt", INTEGER_CASES)
def test_integer_inputs_select_bit_exact(name, kw, fmt):
    # Selector queries and keys in {-3..3}: every score is exact in fp32 and
    # fp64 (MXFP4 and FP8 E4M3 store these values losslessly), so the selected sets must
    # be identical; p is placed away from every cumulative mass.
    wl = workloads.make(name, seed=11, device=DEV, integer=True, **kw)
    wl.top_p = safe_top_p(wl, fmt)
    gpu = run_gpu(wl, fmt)
    assert gpu["status"] == 0
    ora = run_oracle(wl, fmt)
    _assert_same_selection(gpu, ora, wl)
    check_outputs(gpu, ora, wl)


@pytest.mark.parametrize("fmt", ["mxfp4", "fp8"])
def test_integer_inputs_quantised_queries_select_bit_exact(fmt):
    # Queries in {-3..3} are stored losslessly by MXFP4 (power-of-two group
    # scales) and E4M3, so quantising them keeps every score exact on both
    # sides and the selections must be identical.
    wl = workloads.make("quant_128k", seed=12, device=DEV, integer=True, seq_len=8192, batch=4)
    wl.top_p = safe_top_p(wl, fmt, quantize_queries=True)
    gpu = run_gpu(wl, fmt, quantize_queries=True)
    assert gpu["status"] == 0
    ora = run_oracle(wl, fmt, quantize_queries=True)
    _assert_same_selection(gpu, ora, wl)
    check_outputs(gpu, ora, wl)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "fp8", "int8"])
def test_quantised_queries_small(fmt):
    # 4 sequences x 8 KV heads = 32 units of real-valued scores: units may
    # differ only by blocks next to the cut (the near-cut rule checks each),
    # and every unit whose selection agrees has its outputs compared.
    wl = workloads.make("qwen3_4b_32k", seed=3, device=DEV, sel_fmt=fmt, seq_len=4096, batch=4)
    gpu = run_gpu(wl, fmt, quantize_queries=True)
    assert gpu["status"] == 0
    scores = oracle_scores(wl, fmt, quantize_queries=True)
    assert not np.allclose(scores, oracle_scores(wl, fmt), equal_nan=True)
    ora = run_oracle(wl, fmt, quantize_queries=True)
    units = wl.batch * wl.num_kv_heads
    n_diff = check_selection_near_cut(gpu, ora, scores, wl)
    assert n_diff <= 2
    _, _, n = check_outputs(gpu, ora, wl)
    assert n == units - n_diff


def test_integer_inputs_topk_and_kmin_modes():
    wl = workloads.make("qwen3_4b_32k", seed=5, device=DEV, integer=True, seq_len=4096)
    for kw in (dict(mode="topk", topk=17), dict(mode="topk", topk=0), dict(kmin=40),
               dict(kmin=1000), dict(sink=0, rec=0, kmin=0)):
        gpu = run_gpu(wl, **kw)
        ora = run_oracle(wl, **kw)
        _assert_same_selection(gpu, ora, wl)
        check_outputs(gpu, ora, wl)


@pytest.mark.parametrize("fmt", ["bf16", "int4", "mxfp4", "fp8", "int8"])
def test_append_matches_oracle_quantiser(fmt):
    wl = workloads.make("qwen3_4b_32k", seed=3, device=DEV, seq_len=4096 + 64 * 7)
    data, scales = gpu_selector_pool(wl, fmt, DEV)
    o_data, o_scales = oracle_selector_pool(wl, fmt)
    g_data = data.cpu().view(torch.int16).numpy().view(np.uint16) if fmt == "bf16" \
        else data.cpu().numpy()
    assert np.array_equal(g_data, o_data)
    if o_scales is not None:
        g_scales = scales.cpu().view(torch.int16).numpy().view(np.uint16) \
            if fmt in ("int4", "int8") else scales.cpu().numpy()
        assert np.array_equal(g_scales, o_scales)
    else:
        assert scales is None


def test_append_extreme_values_match_oracle():
    # Zeros, subnormal-range, huge and mixed-sign groups from a seeded draw,
    # plus rows that hold +-inf and NaN explicitly: both quantisers follow
    # the same rule for them (a NaN scale and zero codes for the group, the
    # E4M3 NaN for an FP8 element), so the pools must be bit-identical.
    rows = 72
    gen = torch.Generator().manual_seed(20)
    x = torch.randn(rows, 1, 64, generator=gen) * torch.logspace(-40, 37, rows)[:, None, None]
    x[0] = 0.0
    x[1, 0, :32] = 0.0
    x[2, 0, 5] = 3.0e38
    x[3] = -x[3].abs()
    x[64, 0, 7] = float("inf")                       # group 0 only
    x[65, 0, 40] = float("-inf")                     # group 1 only
    x[66, 0, 0] = float("nan")
    x[67, 0, 33] = float("nan")
    x[67, 0, 2] = float("inf")                       # both groups
    x[68] = 3.3895313892515355e38                    # the bf16 maximum everywhere
    x[68, 0, 1::2] *= -1
    x[69] = 2.0 ** -130                              # bf16 subnormals only
    x[70, 0, :] = torch.linspace(-1e-38, 1e-38, 64)
    x[71, 0, ::3] = float("nan")
    keys = x.to(torch.bfloat16).to(DEV)
    pt = torch.arange(rows, dtype=torch.int32, device=DEV).view(1, rows)
    for fmt in ("int4", "mxfp4", "fp8", "int8"):
        desc = spot.layer_desc(1, 1, rows, fmt)
        data, scales = spot.selector_pool(fmt, rows, 1, device=DEV)
        spot.append_selector_keys(desc, data, scales, pt,
                                  torch.zeros(rows, dtype=torch.int32, device=DEV),
                                  torch.arange(rows, dtype=torch.int32, device=DEV), keys)
        o_data, o_scales = oracle.quantize_selector(fmt, workloads.bits(keys))
        assert np.array_equal(data.cpu().numpy(), o_data), fmt
        if o_scales is not None:
            sc = scales.cpu()
            sc = sc.view(torch.int16).numpy().view(np.uint16) if fmt in ("int4", "int8") \
                else sc.numpy()
            assert np.array_equal(sc, o_scales), fmt


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "fp8", "int8"])
@pytest.mark.parametrize("qq", [False, True])
def test_nonfinite_selector_inputs_select_like_oracle(fmt, qq):
    # Selector keys holding +-inf / NaN are stored with a NaN scale (or the
    # E4M3 NaN), and a query head holding NaN gives NaN dot products: the
    # score's ReLU turns each undefined dot product into 0 on both sides, so
    # with integer-valued inputs the selections must still be identical.
    wl = workloads.make("qwen3_4b_32k", seed=21, device=DEV, integer=True, seq_len=4096, batch=2)
    pt = wl.page_table.cpu().numpy()
    poison = [(0, 3, 0, 5, float("inf")), (0, 10, 1, 40, float("-inf")),
              (1, 7, 2, 0, float("nan")), (1, 20, 3, 33, float("nan")),
              (1, 21, 3, 2, float("inf"))]
    for b, j, g, d, v in poison:
        wl.sel_keys[int(pt[b, j]), g, d] = v
    wl.q_sel[1, 5, 17] = float("nan")                # one index head of KV head 1
    wl.top_p = safe_top_p(wl, fmt, quantize_queries=qq)
    scores = oracle_scores(wl, fmt, quantize_queries=qq)
    for b, j, g, _, _ in poison:
        assert scores[b, g, j] == 0.0
    gpu = run_gpu(wl, fmt, quantize_queries=qq)
    assert gpu["status"] == 0
    ora = run_oracle(wl, fmt, quantize_queries=qq)
    _assert_same_selection(gpu, ora, wl)
    check_outputs(gpu, ora, wl)


def test_sparse_decode_on_oracle_selection():
    # The attention kernels alone, fed the oracle's selection.
    wl = workloads.make("qwen3_4b_32k", seed=2, device=DEV)
    a = oracle_args(wl)
    ora = run_oracle(wl, args=a)
    desc = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages)
    ws = spot.new_workspace(desc, wl.batch, wl.max_blocks, DEV)
    sel_idx = torch.as_tensor(ora["sel_idx"], device=DEV)
    sel_cnt = torch.as_tensor(ora["sel_cnt"], device=DEV)
    out = torch.empty(wl.batch, wl.num_q_heads, 128, device=DEV)
    lse = torch.empty(wl.batch, wl.num_q_heads, device=DEV)
    spot.sparse_decode(desc, wl.q, wl.k_pool, wl.v_pool, wl.page_table, wl.seq_lens, sel_idx,
                       sel_cnt, wl.sm_scale, out, lse, ws)
    torch.cuda.synchronize()
    assert spot.read_device_status(ws) == 0
    gpu = {"sel_idx": ora["sel_idx"], "sel_cnt": ora["sel_cnt"],
           "out": out.cpu().double().numpy(), "lse": lse.cpu().double().numpy()}
    _, _, n = check_outputs(gpu, ora, wl)
    assert n == wl.batch * wl.num_kv_heads


# ------------------------------------------------------------ full size

FULL = [
    ("qwen3_4b_32k", "bf16", None, False),
    ("qwen3_32b_128k", "bf16", [0, 3], False),
    ("quant_128k", "int4", [1, 14], False),
    ("quant_128k", "mxfp4", [0, 9], False),
    ("quant_128k", "fp8", [3, 12], False),
    ("quant_128k", "int8", [2, 11], False),
    ("quant_128k", "int4", [4], True),
    ("quant_128k", "mxfp4", [6], True),
    ("quant_128k", "fp8", [8], True),
    ("quant_128k", "int8", [10], True),
    ("ragged_hybrid", "mxfp4", [0, 7, 31], False),
]


@pytest.mark.parametrize("name,fmt,sample,qq", FULL)
def test_full_size_config(name, fmt, sample, qq):
    """Full-size workload in the benchmark's launch configuration: selection
    of every (sequence, KV head) checked against the oracle's scores; the
    attention output of the sampled sequences against the oracle.  qq: the
    selector queries are quantised like the keys."""
    wl = workloads.make(name, seed=1, device=DEV, sel_fmt=fmt)
    gpu = run_gpu(wl, fmt, quantize_queries=qq)
    assert gpu["status"] == 0
    pool = gpu.pop("pool")
    del pool
    # selection, every unit (scores and selection need only the selector pool)
    sh, pr = oracle.make_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, 128, 64, 64, fmt,
                               wl.num_pages, wl.max_blocks), None
    o_data, o_scales = oracle_selector_pool(wl, fmt)
    pr = oracle.make_params(sink_blocks=wl.spec.sink_blocks, recency_blocks=wl.spec.recency_blocks,
                            kmin_blocks=wl.spec.kmin_blocks, quantize_queries=qq)
    scores = oracle.block_scores(sh, pr, workloads.bits(wl.q_sel), None, o_data, o_scales,
                                 wl.page_table.cpu().numpy(), wl.seq_lens.cpu().numpy())
    lens = wl.seq_lens.cpu().numpy()
    top_p = wl.top_p.cpu().numpy()
    sel = {"sel_idx": np.full_like(gpu["sel_idx"], -1), "sel_cnt": np.zeros_like(gpu["sel_cnt"])}
    for b in range(wl.batch):
        nb = (int(lens[b]) + 63) // 64
        for g in range(wl.num_kv_heads):
            s, _ = oracle.select_from_scores(scores[b, g, :nb], nb=nb, n_full=int(lens[b]) // 64,
                                             params=pr, p=float(top_p[b]))
            sel["sel_idx"][b, g, :s.size] = s
            sel["sel_cnt"][b, g] = s.size
    n_diff = check_selection_near_cut(gpu, sel, scores, wl)
    assert n_diff <= max(1, wl.batch * wl.num_kv_heads // 50)
    frac = gpu["sel_cnt"] / np.maximum(1, (lens[:, None] + 63) // 64)
    print(f"{name}/{fmt}: |S|/nb mean {frac.mean():.3f} min {frac.min():.3f} "
          f"max {frac.max():.3f}; near-cut differences {n_diff}")
    # attention, sampled sequences
    seqs = list(range(wl.batch)) if sample is None else sample
    sub = workloads.gather_units(wl, seqs)
    ora = run_oracle(sub, fmt, quantize_queries=qq)
    g_sub = {k: gpu[k][seqs] for k in ("sel_idx", "sel_cnt", "out", "lse")}
    _assert_same_selection_or_near(g_sub, ora, sub)
    _, _, n = check_outputs(g_sub, ora, sub)
    assert n >= len(seqs) * wl.num_kv_heads - n_diff


def _assert_same_selection_or_near(gpu, ora, wl):
    diff = sum(unit_selection(gpu, b, g) != unit_selection(ora, b, g)
               for b in range(wl.batch) for g in range(wl.num_kv_heads))
    assert diff <= 1


@pytest.mark.parametrize("batch", [2, 8])
def test_scoring_split_over_ctas_bit_exact_and_repeatable(batch):
    # Contexts of 300K - 512K tokens (up to 8192 blocks per (sequence, KV
    # head)) over only 16 or 64 units: each unit's scoring is spread over a
    # cluster of 8 or 2 CTAs, which store their scores into the first CTA's
    # shared memory, and that CTA selects.  Integer selector inputs make
    # every score exact, so every selection must equal the oracle's, and a
    # second call on the same workspace must repeat it.
    wl = workloads.make("ragged_hybrid", seed=13, device=DEV, integer=True, batch=batch,
                        sel_fmt="bf16", ragged_range=(300000, 524288))
    data, scales = oracle_selector_pool(wl, "bf16")
    a = dict(q_sel=workloads.bits(wl.q_sel), w=None, sel_data=data, sel_scales=scales,
             page_table=wl.page_table.cpu().numpy(), seq_lens=wl.seq_lens.cpu().numpy())
    wl.top_p = safe_top_p(wl, "bf16", args=a)
    scores = oracle_scores(wl, "bf16", args=a)
    sp = wl.spec
    pr = oracle.make_params(sink_blocks=sp.sink_blocks, recency_blocks=sp.recency_blocks,
                            kmin_blocks=sp.kmin_blocks)
    lens, top_p = a["seq_lens"], wl.top_p.cpu().numpy()
    want = {}
    for b in range(wl.batch):
        nb = (int(lens[b]) + 63) // 64
        for g in range(wl.num_kv_heads):
            sel, _ = oracle.select_from_scores(scores[b, g, :nb], nb=nb, n_full=int(lens[b]) // 64,
                                               params=pr, p=float(top_p[b]))
            want[b, g] = sel.tolist()
    desc = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, "bf16")
    prm = spot.select_params("topp", sp.sink_blocks, sp.recency_blocks, sp.kmin_blocks)
    ws = spot.new_workspace(desc, wl.batch, wl.max_blocks, DEV)
    for call in range(2):
        sel_idx = torch.full((wl.batch, wl.num_kv_heads, wl.max_blocks), -1, dtype=torch.int32,
                             device=DEV)
        sel_cnt = torch.full((wl.batch, wl.num_kv_heads), -1, dtype=torch.int32, device=DEV)
        spot.select(desc, prm, wl.q_sel, None, wl.sel_keys, None, wl.page_table, wl.seq_lens,
                    wl.top_p, sel_idx, sel_cnt, ws)
        torch.cuda.synchronize()
        assert spot.read_device_status(ws) == 0
        got = {"sel_idx": sel_idx.cpu().numpy(), "sel_cnt": sel_cnt.cpu().numpy()}
        for (b, g), sel in want.items():
            assert unit_selection(got, b, g) == sel, (call, b, g)


# ------------------------------------------------------------ edge cases

def test_ragged_partial_blocks_and_empty_sequences():
    wl = workloads.make("ragged_hybrid", seed=4, device=DEV, batch=6, sel_fmt="bf16",
                        ragged_range=(2048, 2048))
    lens = torch.tensor([0, 1, 63, 65, 64 * 9 + 17, 2048], dtype=torch.int32)
    nb = (lens + 63) // 64
    pt = torch.full((6, int(nb.max())), -1, dtype=torch.int32)
    perm = torch.randperm(int(nb.sum()), generator=torch.Generator().manual_seed(0))
    off = 0
    for b in range(6):
        pt[b, :nb[b]] = perm[off:off + nb[b]].int()
        off += int(nb[b])
    wl.seq_lens = lens.to(DEV)
    wl.page_table = pt.to(DEV)
    for kw in (dict(), dict(rec=0, sink=0, kmin=0), dict(kmin=3)):
        gpu = run_gpu(wl, **kw)
        assert gpu["status"] == 0
        ora = run_oracle(wl, **kw)
        _assert_same_selection(gpu, ora, wl)
        check_outputs(gpu, ora, wl)
        assert (gpu["out"][0] == 0).all() and np.isneginf(gpu["lse"][0]).all()
        assert gpu["sel_cnt"][0].tolist() == [0] * wl.num_kv_heads


def test_p_one_is_dense_attention_and_p_zero_keeps_reserved():
    wl = workloads.make("qwen3_4b_32k", seed=6, device=DEV, seq_len=4096, batch=2)
    wl.top_p = torch.ones(2, device=DEV)
    gpu = run_gpu(wl, kmin=0)
    assert (gpu["sel_cnt"] == 64).all()
    ora = run_oracle(wl, kmin=0)
    check_outputs(gpu, ora, wl)
    # dense reference from torch's own attention on the gathered cache
    k = wl.k_pool[wl.page_table.long()].float()       # [B, nb, Hkv, 64, D]
    v = wl.v_pool[wl.page_table.long()].float()
    B, nbk, Hkv = k.shape[:3]
    k = k.permute(0, 2, 1, 3, 4).reshape(B, Hkv, nbk * 64, 128)
    v = v.permute(0, 2, 1, 3, 4).reshape(B, Hkv, nbk * 64, 128)
    G = wl.num_q_heads // Hkv
    q = wl.q.float().view(B, Hkv, G, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=wl.sm_scale)
    ref = ref.reshape(B, wl.num_q_heads, 128).double().cpu().numpy()
    assert np.allclose(gpu["out"], ref, atol=2e-3, rtol=1e-2)
    wl.top_p = torch.zeros(2, device=DEV)
    gpu = run_gpu(wl, kmin=0)
    assert (gpu["sel_cnt"] == 1 + 4).all()


def test_heavy_ties_in_the_cut():
    # All scores equal (q_sel = 0): one tie group of 507 residual blocks; the
    # cut takes the lowest block indices.  Then four score levels from one
    # selector-query dimension: tie groups of ~70-300 blocks at the cut.
    wl = workloads.make("qwen3_4b_32k", seed=9, device=DEV, integer=True, batch=2)
    wl.q_sel.zero_()
    for p in (0.3, 0.5, 0.77):
        wl.top_p = torch.full((2,), p, device=DEV)
        gpu = run_gpu(wl, kmin=0)
        ora = run_oracle(wl, kmin=0)
        _assert_same_selection(gpu, ora, wl)
    wl.q_sel[:, :, 0] = 1.0
    wl.top_p = safe_top_p(wl)
    for kw in (dict(kmin=0), dict(kmin=300), dict(mode="topk", topk=200)):
        gpu = run_gpu(wl, **kw)
        ora = run_oracle(wl, **kw)
        _assert_same_selection(gpu, ora, wl)
        check_outputs(gpu, ora, wl)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (12, 4), (16, 2), (8, 8)])
def test_group_sizes(hq, hkv):
    wl = workloads.make("qwen3_4b_32k", seed=7, device=DEV, seq_len=2048 + 64 * 3, batch=3,
                        num_q_heads=hq, num_kv_heads=hkv, integer=True)
    wl.top_p = safe_top_p(wl)
    gpu = run_gpu(wl)
    ora = run_oracle(wl)
    _assert_same_selection(gpu, ora, wl)
    check_outputs(gpu, ora, wl)


def test_weights_temperature_and_padding():
    wl = workloads.make("qwen3_4b_32k", seed=8, device=DEV, seq_len=3000, batch=2, integer=True)
    g = torch.Generator(device="cpu").manual_seed(1)
    wl.w = (torch.rand(2, wl.num_q_heads, generator=g) * 2).float().to(DEV)
    wl.w = (wl.w * 8).round() / 8                       # exact in fp32 and fp64
    for temp in (1.0, 2.0, 0.5):
        wl.top_p = safe_top_p(wl, temperature=temp)
        # an odd max_blocks (47 + 38 = 85) also checks the alignment of the
        # kernels' shared-memory layouts
        gpu = run_gpu(wl, temperature=temp, max_blocks=wl.max_blocks + 38)
        ora = run_oracle(wl, temperature=temp, max_blocks=wl.max_blocks + 38)
        _assert_same_selection(gpu, ora, wl)
        check_outputs(gpu, ora, wl)


def test_bad_page_id_is_reported_not_faulted():
    wl = workloads.make("tiny_4k", seed=0, device=DEV)
    # Build the selector pool from the valid table first; only the kernels
    # under test ever see the out-of-range page id.
    pool = gpu_selector_pool(wl, "bf16", DEV)
    wl.page_table[0, 5] = wl.num_pages + 100
    gpu = run_gpu(wl, pool=pool)
    assert gpu["status"] == 5                          # SPOT_ERR_DEVICE_BOUNDS
    assert np.isfinite(gpu["out"]).all()
    # the context is still usable
    wl2 = workloads.make("tiny_4k", seed=0, device=DEV)
    assert run_gpu(wl2)["status"] == 0


def test_bounded_wait_reports_timeout_and_context_survives():
    # A wait that nothing satisfies gives up after about a second, records
    # SPOT_ERR_DEVICE_TIMEOUT (6) and the context keeps working.
    ws = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    t0 = time.time()
    spot.check_wait_timeout(ws)
    assert spot.read_device_status(ws) == 6
    assert 0.5 < time.time() - t0 < 30
    assert spot.read_device_status(ws) == 0          # read clears it
    wl = workloads.make("tiny_4k", seed=0, device=DEV)
    assert run_gpu(wl)["status"] == 0


def test_workspace_too_small_and_bad_arguments():
    wl = workloads.make("tiny_4k", seed=0, device=DEV)
    desc = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages)
    prm = spot.select_params()
    n = spot.workspace_size(desc, 1, wl.max_blocks)
    ws = torch.zeros(n - 256, dtype=torch.uint8, device=DEV)
    sel_idx = torch.zeros(1, wl.num_kv_heads, wl.max_blocks, dtype=torch.int32, device=DEV)
    sel_cnt = torch.zeros(1, wl.num_kv_heads, dtype=torch.int32, device=DEV)
    with pytest.raises(spot.SpotError) as e:
        spot.select(desc, prm, wl.q_sel, None, wl.sel_keys, None, wl.page_table, wl.seq_lens,
                    wl.top_p, sel_idx, sel_cnt, ws)
    assert e.value.code == 3
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    with pytest.raises(spot.SpotError) as e:       # TOPP without top_p
        spot.select(desc, prm, wl.q_sel, None, wl.sel_keys, None, wl.page_table, wl.seq_lens,
                    None, sel_idx, sel_cnt, ws)
    assert e.value.code == 1
    bad = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, "int4")
    with pytest.raises(spot.SpotError) as e:       # INT4 without scales
        spot.select(bad, prm, wl.q_sel, None, wl.sel_keys, None, wl.page_table, wl.seq_lens,
                    wl.top_p, sel_idx, sel_cnt, ws)
    assert e.value.code == 1


def test_decode_step_captured_in_a_cuda_graph():
    """spot_decode_step is capture-safe: one capture, replayed on new
    queries copied into the captured buffers, matches the oracle."""
    wl = workloads.make("tiny_4k", seed=21, device=DEV)
    desc = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, "bf16")
    prm = spot.select_params("topp", wl.spec.sink_blocks, wl.spec.recency_blocks,
                             wl.spec.kmin_blocks)
    B, Hq, Hkv, mb = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.max_blocks
    ws = spot.new_workspace(desc, B, mb, DEV)
    q, q_sel = wl.q.clone(), wl.q_sel.clone()
    sel_idx = torch.full((B, Hkv, mb), -1, dtype=torch.int32, device=DEV)
    sel_cnt = torch.zeros((B, Hkv), dtype=torch.int32, device=DEV)
    out = torch.zeros((B, Hq, 128), dtype=torch.float32, device=DEV)
    lse = torch.zeros((B, Hq), dtype=torch.float32, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        spot.decode_step(desc, prm, q_sel, wl.w, wl.sel_keys, None, q, wl.k_pool, wl.v_pool,
                         wl.page_table, wl.seq_lens, wl.top_p, wl.sm_scale, sel_idx, sel_cnt,
                         out, lse, ws, s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        spot.decode_step(desc, prm, q_sel, wl.w, wl.sel_keys, None, q, wl.k_pool, wl.v_pool,
                         wl.page_table, wl.seq_lens, wl.top_p, wl.sm_scale, sel_idx, sel_cnt,
                         out, lse, ws, s)
    for seed in (22, 23):
        other = workloads.make("tiny_4k", seed=seed, device=DEV)
        wl2 = workloads.make("tiny_4k", seed=21, device=DEV)
        wl2.q, wl2.q_sel = other.q, other.q_sel
        q.copy_(other.q)
        q_sel.copy_(other.q_sel)
        graph.replay()
        torch.cuda.synchronize()
        assert spot.read_device_status(ws) == 0
        gpu = {"sel_idx": sel_idx.cpu().numpy(), "sel_cnt": sel_cnt.cpu().numpy(),
               "out": out.cpu().double().numpy(), "lse": lse.cpu().double().numpy()}
        ora = run_oracle(wl2)
        assert check_selection_near_cut(gpu, ora, oracle_scores(wl2), wl2) == 0
        _, _, n = check_outputs(gpu, ora, wl2)
        assert n == B * Hkv
    del graph
