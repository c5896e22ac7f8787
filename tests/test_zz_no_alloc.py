"""spot_sparse_decode_noalloc: the sparse-attention entry point for callers
that cannot allocate device memory (a serving engine that keeps all free HBM
for its KV pool and forbids further cudaMalloc calls, or a plugin host that
passes tensors but no allocator).  Its scratch is a fixed 8 MiB array inside
the library.  Checked through the C ABI against spot_sparse_decode (which
takes a caller-allocated workspace) on two calls in a row, the second on a
different shape so stale scratch from the first call would show.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import block_sparse_long_spot_b200 as spot
import workloads

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()


def _selection(wl, desc, ws):
    B, Hkv, mb = wl.batch, wl.num_kv_heads, wl.max_blocks
    prm = spot.select_params(sink_blocks=wl.spec.sink_blocks,
                             recency_blocks=wl.spec.recency_blocks,
                             kmin_blocks=wl.spec.kmin_blocks)
    sel_idx = torch.full((B, Hkv, mb), -1, dtype=torch.int32, device="cuda")
    sel_cnt = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    spot.select(desc, prm, wl.q_sel, None, wl.sel_keys, None, wl.page_table, wl.seq_lens,
                wl.top_p, sel_idx, sel_cnt, ws)
    return sel_idx, sel_cnt


def _both(wl):
    desc = spot.layer_desc(wl.num_q_heads, wl.num_kv_heads, wl.num_pages, "bf16")
    ws = spot.new_workspace(desc, wl.batch, wl.max_blocks)
    sel_idx, sel_cnt = _selection(wl, desc, ws)
    shape = (wl.batch, wl.num_q_heads)
    out_ws = torch.empty(*shape, 128, device="cuda")
    lse_ws = torch.empty(*shape, device="cuda")
    spot.sparse_decode(desc, wl.q, wl.k_pool, wl.v_pool, wl.page_table, wl.seq_lens, sel_idx,
                       sel_cnt, wl.sm_scale, out_ws, lse_ws, ws)
    out_na = torch.full((*shape, 128), float("nan"), device="cuda")
    lse_na = torch.full(shape, float("nan"), device="cuda")
    spot.sparse_decode_noalloc(desc, wl.q, wl.k_pool, wl.v_pool, wl.page_table, wl.seq_lens,
                               sel_idx, sel_cnt, wl.sm_scale, out_na, lse_na)
    torch.cuda.synchronize()
    assert spot.read_device_status(ws) == 0
    return (out_ws.cpu().double().numpy(), lse_ws.cpu().double().numpy(),
            out_na.cpu().double().numpy(), lse_na.cpu().double().numpy())


def _close(a, b):
    fin = np.isfinite(a)
    assert np.array_equal(fin, np.isfinite(b))
    assert (np.abs(a[fin] - b[fin]) <= ATOL + RTOL * np.abs(a[fin])).all()


def test_noalloc_matches_workspace_call_twice_in_a_row():
    # Both calls launch the same kernel with the same grid and merge the
    # split partials in the same fixed order, so beyond the shared tolerance
    # the results must be bit-identical: a stale or misplaced scratch entry
    # from the first call would show on the second.
    first = workloads.make("qwen3_4b_32k", seed=21, device="cuda", seq_len=8192)
    second = workloads.make("ragged_hybrid", seed=22, device="cuda", batch=12, sel_fmt="bf16",
                            ragged_range=(128, 16384))
    for wl in (first, second):
        out_ws, lse_ws, out_na, lse_na = _both(wl)
        _close(out_ws, out_na)
        _close(lse_ws, lse_na)
        assert np.array_equal(out_ws, out_na)
        assert np.array_equal(lse_ws, lse_na)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 512 sequences x 8 KV heads x 8 query heads per KV head need far more
    # than 8 MiB of partials: refused on the host before any launch.
    B, Hq, Hkv = 512, 64, 8
    desc = spot.layer_desc(Hq, Hkv, 16, "bf16")
    q = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(16, Hkv, 64, 128, dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros(B, 1, dtype=torch.int32, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    sel_idx = torch.zeros(B, Hkv, 1, dtype=torch.int32, device="cuda")
    sel_cnt = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    out = torch.zeros(B, Hq, 128, device="cuda")
    with pytest.raises(spot.SpotError) as e:
        spot.sparse_decode_noalloc(desc, q, pool, pool, pt, lens, sel_idx, sel_cnt, 0.1, out,
                                   None)
    assert e.value.code == 3
