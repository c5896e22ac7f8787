"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to something the SpotAttention paper or
the mathematics fixes: hand-worked examples of Eq. 7-8 (tests/golden),
brute-force subset enumeration, closed forms, hand-computed selector scores
(§2.1), the published MX / binary16 formats, and the special cases in which
sparse attention reduces to a library softmax attention (all blocks kept).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_bits(values):
    t = torch.as_tensor(np.asarray(values, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- selection

def test_topp_worked_example():
    ex = _golden("topp_worked_example.json")
    for case in ex["cases"]:
        pr = oracle.make_params(sink_blocks=ex["sink_blocks"], recency_blocks=ex["recency_blocks"],
                                kmin_blocks=case["kmin"])
        sel, mass = oracle.select_from_scores(ex["scores"], params=pr, p=case["p"])
        assert sel.tolist() == case["selected"], case
        # The nucleus mass is the cumulative residual-softmax mass of the
        # chosen residual blocks.
        n_res = len(case["selected"]) - 2
        expect = ex["cumulative_mass"][n_res - 1] if n_res > 0 else 0.0
        assert abs(mass - expect) < 2e-6, (case, mass)
    t = ex["tie_case"]
    pr = oracle.make_params(sink_blocks=1, recency_blocks=1, kmin_blocks=t["kmin"])
    sel, mass = oracle.select_from_scores(t["scores"], params=pr, p=t["p"])
    assert sel.tolist() == t["selected"]
    assert mass == 0.5


def _brute_force_nucleus(scores, res, p):
    """Smallest subsets of the residual blocks whose softmax mass reaches p,
    found by enumerating every subset (no sorting, no prefix sums)."""
    s = np.asarray([scores[j] for j in res], np.float64)
    e = np.exp(s - s.max())
    prob = e / e.sum()
    if p <= 0:
        return 0, [()]
    for k in range(0, len(res) + 1):
        hits = [c for c in itertools.combinations(range(len(res)), k)
                if prob[list(c)].sum() >= p - 1e-12]
        if hits:
            return k, [tuple(res[i] for i in c) for c in hits]
    return len(res), [tuple(res)]


@pytest.mark.parametrize("seed", range(40))
def test_select_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(1, 15))
    sink = int(rng.integers(0, 3))
    rec = int(rng.integers(0, 3))
    kmin = int(rng.integers(0, 8))
    if seed % 2:
        scores = rng.integers(-2, 3, size=nb).astype(np.float64)      # many ties
    else:
        scores = rng.normal(size=nb) * 2.0
    p = float(rng.choice([0.3, 0.5, 0.7, 0.9, 0.95, 0.99, 1.0, 0.0]))
    pr = oracle.make_params(sink_blocks=sink, recency_blocks=rec, kmin_blocks=kmin)
    sel, _ = oracle.select_from_scores(scores, params=pr, p=p)
    reserved = {j for j in range(nb) if j < sink or j >= nb - rec}
    res = [j for j in range(nb) if j not in reserved]
    sel_set = set(sel.tolist())
    # Sorted, unique, reserved blocks always present.
    assert sel.tolist() == sorted(sel_set)
    assert reserved <= sel_set
    nuc = sel_set - reserved
    if res:
        k_min_card, minimal = _brute_force_nucleus(scores, res, p)
        expect_card = min(max(k_min_card, kmin - len(reserved)), len(res))
        assert len(nuc) == expect_card
        if expect_card == k_min_card:
            assert tuple(sorted(nuc)) in [tuple(sorted(c)) for c in minimal]
        # Ranked-prefix closure: nothing outside beats something inside,
        # ties broken toward the lower block index.
        for a in nuc:
            for b in set(res) - nuc:
                assert (scores[a] > scores[b]) or (scores[a] == scores[b] and a < b)
    else:
        assert nuc == set()
    if nb:
        assert len(sel) >= min(kmin, nb)


def test_select_incomplete_last_block_is_reserved():
    # 5 blocks, only 4 complete: block 4 has no score and must be kept.
    pr = oracle.make_params(sink_blocks=0, recency_blocks=0, kmin_blocks=0)
    sel, _ = oracle.select_from_scores([5.0, 0.0, 0.0, 0.0, float("nan")], nb=5, n_full=4,
                                       params=pr, p=0.5)
    assert sel.tolist() == [0, 4]


def test_select_degenerate_sizes():
    pr = oracle.make_params(sink_blocks=2, recency_blocks=4, kmin_blocks=8)
    sel, _ = oracle.select_from_scores([1.0, 2.0, 3.0], params=pr, p=0.9)
    assert sel.tolist() == [0, 1, 2]                       # reserved covers everything
    sel, _ = oracle.select_from_scores(np.zeros(0), nb=0, params=pr, p=0.9)
    assert sel.size == 0
    pr = oracle.make_params(sink_blocks=0, recency_blocks=0, kmin_blocks=100)
    sel, _ = oracle.select_from_scores(np.arange(10.0), params=pr, p=0.1)
    assert sel.tolist() == list(range(10))                 # K_min clamps to nb


def test_static_topk_mode():
    pr = oracle.make_params(mode="topk", sink_blocks=0, recency_blocks=0, topk_blocks=3)
    sel, _ = oracle.select_from_scores([0.5, 4.0, 1.0, 4.0, 3.0, -1.0], params=pr)
    assert sel.tolist() == [1, 3, 4]
    pr = oracle.make_params(mode="topk", sink_blocks=1, recency_blocks=1, topk_blocks=2)
    sel, _ = oracle.select_from_scores([0.5, 2.0, 2.0, 2.0, 3.0, -1.0], params=pr)
    assert sel.tolist() == [0, 1, 4, 5]


# ---------------------------------------------------------------- scoring

def _one_seq_shape(Hq, Hkv, num_pages, max_blocks, fmt="bf16"):
    return oracle.make_shape(1, Hq, Hkv, 128, 64, 64, fmt, num_pages, max_blocks)


def test_scores_hand_computed():
    # Two query heads share one KV head (G = 2).  Selector dim 64.
    q = np.zeros((1, 2, 64), np.float32)
    q[0, 0, 0], q[0, 0, 1] = 1.0, 2.0          # head 0: e0 + 2 e1
    q[0, 1, 0] = -1.0                           # head 1: -e0
    keys = np.zeros((2, 1, 64), np.float32)     # two pages
    keys[1, 0, 0], keys[1, 0, 1], keys[1, 0, 2] = 3.0, -1.0, 5.0   # page 1: dots 1, -3
    keys[0, 0, 0], keys[0, 0, 1] = -1.0, 4.0                        # page 0: dots 7, 1
    pt = np.array([[1, 0]], np.int32)           # logical block 0 -> page 1, block 1 -> page 0
    lens = np.array([128], np.int32)
    sh = _one_seq_shape(2, 1, 2, 2)
    w = np.array([[0.25, 0.75]], np.float32)
    s = oracle.block_scores(sh, oracle.make_params(), _bf16_bits(q), w, _bf16_bits(keys), None,
                            pt, lens)
    assert s[0, 0].tolist() == [0.25 * 1 + 0.75 * 0, 0.25 * 7 + 0.75 * 1]
    s = oracle.block_scores(sh, oracle.make_params(), _bf16_bits(q), None, _bf16_bits(keys), None,
                            pt, lens)
    assert s[0, 0].tolist() == [0.5, 4.0]                   # w = 1/G
    s = oracle.block_scores(sh, oracle.make_params(temperature=2.0), _bf16_bits(q), None,
                            _bf16_bits(keys), None, pt, lens)
    assert s[0, 0].tolist() == [0.25, 2.0]


def test_scores_gqa_grouping_and_partial_block():
    # Hq = 4, Hkv = 2: heads 2, 3 read KV head 1 only.
    q = np.zeros((1, 4, 64), np.float32)
    q[0, :, 0] = [1.0, 1.0, 2.0, 3.0]
    keys = np.zeros((1, 2, 64), np.float32)
    keys[0, 0, 0], keys[0, 1, 0] = 10.0, -1.0
    sh = _one_seq_shape(4, 2, 1, 2)
    s = oracle.block_scores(sh, oracle.make_params(), _bf16_bits(q), None, _bf16_bits(keys), None,
                            np.array([[0, -1]], np.int32), np.array([100], np.int32))
    assert s[0, 0, 0] == 10.0            # (1*10 + 1*10) / 2
    assert s[0, 1, 0] == 0.0             # both dots negative: ReLU
    assert np.isnan(s[0, 0, 1])          # block 1 is incomplete: no score


# ---------------------------------------------------------------- key formats

def test_decode_known_codes():
    g = _golden("selector_codes.json")
    for c in g["decode"]:
        data = np.zeros(32, np.uint8)
        data[0] = c["byte"]
        if c["fmt"] == "int4":
            scales = np.array([c["scale_bits"], 0x3C00], np.uint16)
        else:
            scales = np.array([c["scale"], 127], np.uint8)
        vals = oracle.dequant_selector(c["fmt"], data, scales, 64)[0]
        assert vals[:2].tolist() == c["values"], c["note"]


def test_encode_known_codes():
    g = _golden("selector_codes.json")
    mx = g["encode_mxfp4"]
    data, scales = oracle.quantize_selector("mxfp4", _bf16_bits(mx["inputs"] * 2)[None])
    codes = [int(data[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(64)]
    assert codes[:32] == mx["codes"] and codes[32:] == mx["codes"]
    assert scales[0].tolist() == [mx["scale"], mx["scale"]]
    i4 = g["encode_int4"]
    data, scales = oracle.quantize_selector("int4", _bf16_bits(i4["inputs"] * 2)[None])
    codes = [int(data[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(64)]
    codes = [c - 16 if c >= 8 else c for c in codes]
    assert codes[:32] == i4["codes"] and codes[32:] == i4["codes"]
    assert scales[0].tolist() == [i4["scale_bits"], i4["scale_bits"]]


def _codes_of(fmt, data):
    """Element codes of one 64-element key row (signed for int4 / int8)."""
    if fmt in ("int4", "mxfp4"):
        c = [int(data[i // 2] >> (4 * (i % 2))) & 0xF for i in range(64)]
        return [x - 16 if (fmt == "int4" and x >= 8) else x for x in c]
    if fmt == "int8":
        return data.view(np.int8).astype(int).tolist()
    return data.astype(int).tolist()


def test_nonfinite_and_extreme_groups():
    # Hand-worked rows (tests/golden/selector_codes.json): a group holding NaN
    # or an infinity gets the NaN scale and zero codes (OCP MX's rule, read
    # for every scaled format), FP8 stores such an element as its NaN, and the
    # bf16 maximum / subnormal range land where the format definitions say.
    for case in _golden("selector_codes.json")["nonfinite_and_extremes"]["cases"]:
        fmt = case["fmt"]
        bits = np.zeros(64, np.uint16)
        for i, b in case["set"]:
            bits[i] = b
        data, scales = oracle.quantize_selector(fmt, bits[None])
        want = [0] * 64
        for i, c in case["codes"]:
            want[i] = c
        assert _codes_of(fmt, data[0]) == want, case["note"]
        if case["scales"] is None:
            assert scales is None
        else:
            assert scales[0].tolist() == case["scales"], case["note"]
        # a poisoned group reads back as NaN, every other element as finite
        back = oracle.dequant_selector(fmt, data, scales, 64)[0]
        nonfinite = np.zeros(64, bool)
        for i, b in case["set"]:
            if (b & 0x7F80) == 0x7F80:
                nonfinite[i] = True
        if fmt == "fp8":
            poisoned = nonfinite
        elif fmt == "int8":
            poisoned = np.full(64, nonfinite.any())
        else:
            poisoned = np.repeat(nonfinite.reshape(2, 32).any(1), 32)
        assert np.isnan(back[poisoned]).all() and np.isfinite(back[~poisoned]).all(), case["note"]


def test_int4_scale_is_binary16_rne():
    # The scale is amax/7 rounded to the nearest binary16 (numpy's IEEE
    # conversion is the independent reference), saturating at 65504.
    rng = np.random.default_rng(0)
    amax = np.concatenate([np.exp(rng.uniform(-20, 12, size=400)), [1.0, 7.0, 0.1, 3e5, 1e-9]])
    x = np.zeros((amax.size, 64), np.float32)
    x[:, 3] = amax
    x[:, 40] = -amax
    bits = _bf16_bits(x)
    _, scales = oracle.quantize_selector("int4", bits)
    amax_bf16 = torch.as_tensor(amax.astype(np.float32)).to(torch.bfloat16).double().numpy()
    ref = np.minimum(amax_bf16 / 7.0, 65504.0).astype(np.float16).view(np.uint16)
    assert (scales[:, 0] == ref).all() and (scales[:, 1] == ref).all()


@pytest.mark.parametrize("fmt", ["int4", "mxfp4"])
def test_on_grid_values_round_trip_exactly(fmt):
    rng = np.random.default_rng(1)
    rows = 64
    if fmt == "int4":
        codes = rng.integers(-7, 8, size=(rows, 64)).astype(np.float64)
        codes[:, 0], codes[:, 32] = 7, -7                 # amax = 7 * scale
        scale = np.exp2(rng.integers(-6, 6, size=(rows, 1)))
        x = codes * scale
    else:
        grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
        x = grid[rng.integers(0, 8, size=(rows, 64))] * rng.choice([-1, 1], size=(rows, 64))
        x[:, 0], x[:, 32] = 6.0, -4.0                     # amax = 6 -> X = 0 before scaling
        x = x * np.exp2(rng.integers(-10, 10, size=(rows, 1)))
    bits = _bf16_bits(x)
    data, scales = oracle.quantize_selector(fmt, bits)
    back = oracle.dequant_selector(fmt, data, scales, 64)
    assert np.array_equal(back, x)


def test_quantisation_error_bounds():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(256, 64)).astype(np.float32)
    bits = _bf16_bits(x)
    xb = torch.as_tensor(x).to(torch.bfloat16).double().numpy()
    for fmt in ("int4", "mxfp4"):
        data, scales = oracle.quantize_selector(fmt, bits)
        back = oracle.dequant_selector(fmt, data, scales, 64).reshape(256, 2, 32)
        xg = xb.reshape(256, 2, 32)
        amax = np.abs(xg).max(-1, keepdims=True)
        if fmt == "int4":
            s = amax / 7.0
            assert (np.abs(back - xg) <= 0.5 * s * (1 + 1e-3) + 1e-12).all()
        else:
            # Scale 2^X with X = floor(log2 amax) - 2 puts |x|/2^X below 8.
            # Rounding on the E2M1 grid (steps 0.5 / 1 / 2) or saturation at 6
            # moves an element by less than 2 * 2^X; below 2 * 2^X the grid
            # step is 0.5, so the error there is at most 2^X / 4.
            X = np.floor(np.log2(amax)) - 2
            err = np.abs(back - xg)
            assert (err < 2 * np.exp2(X)).all()
            small = np.abs(xg) < 2 * np.exp2(X)
            assert (err[small] <= (np.exp2(X) / 4 + 0 * xg)[small]).all()


def test_footprint_closed_form():
    # Selector K-cache bits per element: bf16 16, INT4 4 + 16/32, MXFP4
    # 4 + 8/32, FP8 8, INT8 8 + 16/64.  The paper's GiB figures for BF16,
    # INT4 and FP4 (§5.3) follow; FP8 is its 0.500x (App. G Tab. 9), INT8
    # carries a per-key scale on top.
    fp = _golden("selector_codes.json")["footprint"]
    n = fp["layers"] * fp["tokens"] * fp["elements_per_token"]
    for fmt, bits_per in fp["bits"].items():
        x = np.zeros((1, 64), np.float32)
        data, scales = oracle.quantize_selector(fmt, _bf16_bits(x))
        stored = data.nbytes + (0 if scales is None else scales.nbytes)
        assert stored * 8 / 64 == bits_per
        assert round(n * bits_per / 8 / 2**30, 2) == fp["gib"][fmt]
    assert fp["bits"]["fp8"] / fp["bits"]["bf16"] == 0.5


def test_fp8_known_codes():
    g = _golden("selector_codes.json")
    enc = g["encode_fp8"]
    data, scales = oracle.quantize_selector("fp8", _bf16_bits(enc["inputs"] * 4)[None])
    assert scales is None
    assert data[0].tolist() == enc["codes"] * 4
    dec = g["decode_fp8"]
    vals = oracle.dequant_selector("fp8", np.array(dec["codes"] + [0] * 57, np.uint8), None, 64)[0]
    for v, e in zip(vals, dec["values"]):
        assert (np.isnan(v) if e == "nan" else v == e)


def test_fp8_rounding_matches_torch_float8():
    # torch's float8_e4m3fn cast (round to nearest even) is an independent
    # implementation of the same format for magnitudes up to 448.
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.normal(size=4000) * 10.0 ** rng.uniform(-3, 2.6, size=4000),
                        np.linspace(-448, 448, 1793)])
    x = torch.as_tensor(x.astype(np.float32)).to(torch.bfloat16).float().numpy()
    x = x[np.abs(x) <= 448][: 64 * 80]
    bits = _bf16_bits(x.reshape(-1, 64))
    data, _ = oracle.quantize_selector("fp8", bits)
    ref = torch.as_tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = data.reshape(-1)
    zero = x == 0
    assert np.array_equal(ours[~zero], ref[~zero])
    assert (ours[zero] == 0).all()
    back = oracle.dequant_selector("fp8", data, None, 64).reshape(-1)
    ref_back = torch.as_tensor(x).to(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(back, ref_back)


def test_int8_known_codes_and_scale():
    g = _golden("selector_codes.json")["encode_int8"]
    row = g["inputs"] + [0.0] * (64 - len(g["inputs"]))
    data, scales = oracle.quantize_selector("int8", _bf16_bits(row)[None])
    assert data[0, :len(g["codes"])].tolist() == g["codes"]
    assert scales[0].tolist() == [g["scale_bits"]]
    rng = np.random.default_rng(5)
    x = (rng.normal(size=(300, 64)) * 10.0 ** rng.uniform(-4, 4, size=(300, 1))).astype(np.float32)
    bits = _bf16_bits(x)
    data, scales = oracle.quantize_selector("int8", bits)
    xb = torch.as_tensor(x).to(torch.bfloat16).double().numpy()
    amax = np.abs(xb).max(1)
    ref = np.minimum(amax / 127.0, 65504.0).astype(np.float16).view(np.uint16)
    assert (scales[:, 0] == ref).all()
    back = oracle.dequant_selector("int8", data, scales, 64)
    s = scales[:, 0].view(np.float16).astype(np.float64)[:, None]
    assert (np.abs(back - xb) <= 0.5 * s * (1 + 1e-9) + 1e-300).all()
    e = np.exp2(rng.integers(-8, 8, size=(8, 1)))
    on_grid = rng.integers(-127, 128, size=(8, 64)) * e
    on_grid[:, 0] = 127 * e[:, 0]                      # amax = 127 * scale
    d2, s2 = oracle.quantize_selector("int8", _bf16_bits(on_grid))
    assert np.array_equal(oracle.dequant_selector("int8", d2, s2, 64), on_grid)


# ------------------------------------------------ quantised selector queries
# SpotAttention §5.3 / App. G Tab. 9 quantise the selector's queries along
# with its key cache; a query row goes through the key format's quantiser.

# One hand-worked case per format: (query elements {index: value}, key row
# as codes + scales, score with quantised queries, score with bf16 queries).
_QQ_CASES = {
    # E4M3 at [1, 2) has step 1/8: 1.0625 is a tie -> 1.0 (even mantissa);
    # at [2, 4) step 1/4: 3.375 is a tie -> 3.5.  Key = (1, 2).
    "fp8": ({0: 1.0625, 1: 3.375},
            (np.array([0x38, 0x40] + [0] * 62, np.uint8), None), 8.0, 7.8125),
    # group 0 amax 7 -> scale 1: codes 7, 4 (3.5 ties to even), -1;
    # group 1 amax 14 -> scale 2: code 7.  Key = 1 at dims 0, 1, 2, 32.
    "int4": ({0: 7.0, 1: 3.5, 2: -1.2, 32: 14.0},
             (np.array([0x11, 0x01] + [0] * 14 + [0x01] + [0] * 15, np.uint8),
              np.array([0x3C00, 0x3C00], np.uint16)), 24.0, 7 + 3.5 - 1.203125 + 14),
    # amax 127 -> scale 1: codes 127, 2 (2.5 ties to even), -4 (-3.5 ties to
    # even), 0.  Key = 1 at dims 0-3.
    "int8": ({0: 127.0, 1: 2.5, 2: -3.5, 3: 0.4},
             (np.array([1, 1, 1, 1] + [0] * 60, np.int8), np.array([0x3C00], np.uint16)),
             125.0, 127 + 2.5 - 3.5 + 0.400390625),
    # group 0 amax 6 -> X = 2 - 2 = 0: 6 -> 6, 2.5 -> 2 (tie between codes 4
    # and 5, even code), 0.2 -> 0.  Key = 1.0 (code 2, E8M0 127) at dims 0-2.
    "mxfp4": ({0: 6.0, 1: 2.5, 2: 0.2},
              (np.array([0x22, 0x02] + [0] * 30, np.uint8), np.array([127, 127], np.uint8)),
              8.0, 6 + 2.5 + 0.2001953125),
}


@pytest.mark.parametrize("fmt", sorted(_QQ_CASES))
def test_quantised_query_scores_hand_worked(fmt):
    qvals, (data, scales), want_q, want_plain = _QQ_CASES[fmt]
    q = np.zeros((1, 1, 64), np.float32)
    for i, v in qvals.items():
        q[0, 0, i] = v
    sh = _one_seq_shape(1, 1, 1, 1, fmt)
    args = (_bf16_bits(q), None, data, scales, np.array([[0]], np.int32),
            np.array([64], np.int32))
    s_q = oracle.block_scores(sh, oracle.make_params(quantize_queries=True), *args)
    s_p = oracle.block_scores(sh, oracle.make_params(), *args)
    assert s_q[0, 0, 0] == want_q
    assert s_p[0, 0, 0] == want_plain


def test_quantised_queries_have_no_effect_on_bf16_keys():
    rng = np.random.default_rng(7)
    sh = oracle.make_shape(2, 8, 2, 128, 64, 64, "bf16", 6, 3)
    q = _bf16_bits(rng.normal(size=(2, 8, 64)))
    keys = _bf16_bits(rng.normal(size=(6, 2, 64)))
    pt = np.array([[0, 1, 2], [3, 4, 5]], np.int32)
    lens = np.array([192, 150], np.int32)
    a = oracle.block_scores(sh, oracle.make_params(quantize_queries=True), q, None, keys, None,
                            pt, lens)
    b = oracle.block_scores(sh, oracle.make_params(), q, None, keys, None, pt, lens)
    assert np.array_equal(a, b, equal_nan=True)


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "fp8", "int8"])
def test_quantised_queries_follow_the_key_quantiser(fmt):
    # Every query head's row is quantised on its own, with the pinned key
    # quantiser, and read back exactly; the score is then the plain weighted
    # ReLU sum (numpy matmul here).
    rng = np.random.default_rng(11)
    B, Hq, Hkv, P, MB = 2, 8, 2, 8, 4
    q = _bf16_bits(rng.normal(size=(B, Hq, 64)) * 10.0 ** rng.uniform(-2, 2, size=(B, Hq, 1)))
    kb = _bf16_bits(rng.normal(size=(P, Hkv, 64)))
    kdata, kscales = oracle.quantize_selector(fmt, kb)
    w = rng.uniform(0.1, 1.0, size=(B, Hq)).astype(np.float32)
    pt = rng.permutation(P).astype(np.int32).reshape(B, MB)
    lens = np.array([256, 200], np.int32)
    sh = oracle.make_shape(B, Hq, Hkv, 128, 64, 64, fmt, P, MB)
    got = oracle.block_scores(sh, oracle.make_params(quantize_queries=True), q, w, kdata, kscales,
                              pt, lens)
    qd_, qs_ = oracle.quantize_selector(fmt, q)
    qd = oracle.dequant_selector(fmt, qd_, qs_, 64).reshape(B, Hq, 64)
    kd = oracle.dequant_selector(fmt, kdata, kscales, 64).reshape(P, Hkv, 64)
    G = Hq // Hkv
    for b in range(B):
        for g in range(Hkv):
            for j in range(lens[b] // 64):
                dots = qd[b, g * G:(g + 1) * G] @ kd[pt[b, j], g]
                want = float((w[b, g * G:(g + 1) * G] * np.maximum(dots, 0.0)).sum())
                assert abs(got[b, g, j] - want) <= 1e-12 * max(1.0, abs(want)), (b, g, j)
    plain = oracle.block_scores(sh, oracle.make_params(), q, w, kdata, kscales, pt, lens)
    assert not np.allclose(got, plain, equal_nan=True)       # the queries really changed


# ---------------------------------------------------------------- attention

def _rand_kv(rng, num_pages, Hkv, Hq, B=1):
    q = rng.normal(size=(B, Hq, 128)).astype(np.float32)
    k = rng.normal(size=(num_pages, Hkv, 64, 128)).astype(np.float32)
    v = rng.normal(size=(num_pages, Hkv, 64, 128)).astype(np.float32)
    to64 = lambda a: torch.as_tensor(a).to(torch.bfloat16).double()
    return (q, k, v), (to64(q), to64(k), to64(v))


def _sdpa(q64, k64, v64, scale):
    # torch's own scaled-dot-product attention in float64 (library routine).
    o = torch.nn.functional.scaled_dot_product_attention(
        q64[None, None, None], k64[None, None], v64[None, None], scale=scale)
    return o[0, 0, 0]


@pytest.mark.parametrize("L", [1, 64, 200, 256])
def test_all_blocks_equals_dense_attention(L):
    rng = np.random.default_rng(L)
    Hq, Hkv, nb = 4, 2, (L + 63) // 64
    (q, k, v), (q64, k64, v64) = _rand_kv(rng, nb + 1, Hkv, Hq)
    pt = np.array([rng.permutation(nb + 1)[:nb]], np.int32)
    sh = oracle.make_shape(1, Hq, Hkv, 128, 64, 64, "bf16", nb + 1, nb)
    sel = np.tile(np.arange(nb, dtype=np.int32), (1, Hkv, 1))
    cnt = np.full((1, Hkv), nb, np.int32)
    scale = 1 / math.sqrt(128)
    out, lse = oracle.sparse_attention(sh, _bf16_bits(q), _bf16_bits(k), _bf16_bits(v), pt,
                                       np.array([L], np.int32), sel, cnt, scale)
    for h in range(Hq):
        g = h // 2
        kk = k64[pt[0], g].reshape(-1, 128)[:L]
        vv = v64[pt[0], g].reshape(-1, 128)[:L]
        ref = _sdpa(q64[0, h], kk, vv, scale)
        assert np.allclose(out[0, h], ref.numpy(), atol=1e-12, rtol=1e-10)
        ref_lse = torch.logsumexp(scale * (kk @ q64[0, h]), 0).item()
        assert abs(lse[0, h] - ref_lse) < 1e-10


def test_subset_equals_attention_over_gathered_tokens():
    rng = np.random.default_rng(7)
    Hq, Hkv, nb = 8, 2, 6
    (q, k, v), (q64, k64, v64) = _rand_kv(rng, nb, Hkv, Hq)
    pt = np.array([rng.permutation(nb)], np.int32)
    sh = oracle.make_shape(1, Hq, Hkv, 128, 64, 64, "bf16", nb, nb)
    sel = np.full((1, Hkv, nb), -1, np.int32)
    sel[0, 0, :3] = [0, 2, 5]
    sel[0, 1, :2] = [1, 4]
    cnt = np.array([[3, 2]], np.int32)
    scale = 0.1
    out, _ = oracle.sparse_attention(sh, _bf16_bits(q), _bf16_bits(k), _bf16_bits(v), pt,
                                     np.array([nb * 64 - 10], np.int32), sel, cnt, scale)
    for h in range(Hq):
        g = h // 4
        blocks = sel[0, g, :cnt[0, g]]
        kk = torch.cat([k64[pt[0, j], g] for j in blocks])
        vv = torch.cat([v64[pt[0, j], g] for j in blocks])
        if blocks[-1] == nb - 1:
            kk, vv = kk[:-10], vv[:-10]           # last block holds 54 valid tokens
        ref = _sdpa(q64[0, h], kk, vv, scale)
        assert np.allclose(out[0, h], ref.numpy(), atol=1e-12, rtol=1e-10)


def test_single_token_and_empty_sequence():
    rng = np.random.default_rng(3)
    (q, k, v), (q64, k64, v64) = _rand_kv(rng, 1, 1, 1)
    sh = oracle.make_shape(1, 1, 1, 128, 64, 64, "bf16", 1, 1)
    out, lse = oracle.sparse_attention(sh, _bf16_bits(q), _bf16_bits(k), _bf16_bits(v),
                                       np.array([[0]], np.int32), np.array([1], np.int32),
                                       np.array([[[0]]], np.int32), np.array([[1]], np.int32), 0.3)
    assert np.array_equal(out[0, 0], v64[0, 0, 0].numpy())            # o = v
    assert lse[0, 0] == pytest.approx(0.3 * float(q64[0, 0] @ k64[0, 0, 0]), abs=1e-12)
    out, lse = oracle.sparse_attention(sh, _bf16_bits(q), _bf16_bits(k), _bf16_bits(v),
                                       np.array([[0]], np.int32), np.array([0], np.int32),
                                       np.array([[[0]]], np.int32), np.array([[0]], np.int32), 0.3)
    assert (out == 0).all() and lse[0, 0] == -np.inf


def test_decode_step_composes_and_is_page_order_invariant():
    import workloads
    wl = workloads.make("tiny_4k", seed=3, seq_len=1024 + 64 * 3)
    sh = oracle.make_shape(wl.batch, wl.num_q_heads, wl.num_kv_heads, 128, 64, 64, "bf16",
                           wl.num_pages, wl.max_blocks)
    pr = oracle.make_params(sink_blocks=1, recency_blocks=2, kmin_blocks=8)
    args = dict(q_sel=workloads.bits(wl.q_sel), w=None, sel_data=workloads.bits(wl.sel_keys),
                sel_scales=None, q=workloads.bits(wl.q), k_pool=workloads.bits(wl.k_pool),
                v_pool=workloads.bits(wl.v_pool), page_table=wl.page_table.numpy(),
                seq_lens=wl.seq_lens.numpy(), top_p=wl.top_p.numpy(), sm_scale=wl.sm_scale)
    r = oracle.decode_step(sh, pr, **args)
    s = oracle.block_scores(sh, pr, args["q_sel"], None, args["sel_data"], None,
                            args["page_table"], args["seq_lens"])
    for g in range(wl.num_kv_heads):
        nb = (int(wl.seq_lens[0]) + 63) // 64
        sel, _ = oracle.select_from_scores(s[0, g, :nb], params=pr, p=float(wl.top_p[0]))
        assert sel.tolist() == r["sel_idx"][0, g, :r["sel_cnt"][0, g]].tolist()
    out, lse = oracle.sparse_attention(sh, args["q"], args["k_pool"], args["v_pool"],
                                       args["page_table"], args["seq_lens"], r["sel_idx"],
                                       r["sel_cnt"], wl.sm_scale)
    assert np.array_equal(out, r["out"]) and np.array_equal(lse, r["lse"])
    # Planted hot blocks are selected.
    for g in range(wl.num_kv_heads):
        chosen = set(r["sel_idx"][0, g, :r["sel_cnt"][0, g]].tolist())
        assert set(wl.hot_blocks[g]) <= chosen
    # Moving the pages around (and the page table with them) changes nothing.
    perm = np.random.default_rng(0).permutation(wl.num_pages)
    inv = np.argsort(perm)
    pt2 = np.where(args["page_table"] >= 0, inv[np.maximum(args["page_table"], 0)], -1)
    args2 = dict(args, page_table=pt2.astype(np.int32), sel_data=args["sel_data"][perm],
                 k_pool=args["k_pool"][perm], v_pool=args["v_pool"][perm])
    r2 = oracle.decode_step(sh, pr, **args2)
    assert np.array_equal(r2["sel_cnt"], r["sel_cnt"])
    assert np.allclose(r2["out"], r["out"], atol=1e-13, rtol=0)


# ------------------------------------------- token-level, layer-shared selector
# §2.1 / §2.3 / App. A Tab. 3 as written: per-token keys for each index head,
# a block's score is the maximum of its tokens' scores, one selection per
# sequence shared by every head, blocks of 16 tokens inside 64-token pages.

def _tok_shape(B, Hq, Hkv, num_pages, max_pages, idx_heads=2):
    return oracle.make_tok_shape(B, Hq, Hkv, num_pages, max_pages, idx_heads=idx_heads)


def test_tok_scores_hand_computed():
    q = np.zeros((1, 2, 128), np.float32)
    q[0, 0, 0] = 1.0                         # head 0: e0
    q[0, 1, 1] = 2.0                         # head 1: 2 e1
    keys = np.zeros((1, 64, 2, 128), np.float32)
    keys[0, 3, 0, 0], keys[0, 3, 1, 1] = 5.0, -1.0     # token 3: dots 5, -2
    keys[0, 7, 0, 0], keys[0, 7, 1, 1] = 1.0, 1.5      # token 7: dots 1, 3
    keys[0, 20, 0, 0], keys[0, 20, 1, 1] = -3.0, 2.0   # token 20: dots -3, 4
    sh = _tok_shape(1, 4, 2, 1, 1)
    args = (_bf16_bits(q), None, _bf16_bits(keys), np.array([[0]], np.int32),
            np.array([40], np.int32))
    w = np.array([[0.5, 0.25]], np.float32)
    s = oracle.tok_block_scores(sh, oracle.make_params(), args[0], w, *args[2:])
    # block 0: max(0.5*5, 0.5*1 + 0.25*3) = 2.5 (the max, not the sum 3.75);
    # block 1: 0.25*4 = 1; block 2 (tokens 32..39) is incomplete: no score
    assert s[0, :2].tolist() == [2.5, 1.0]
    assert np.isnan(s[0, 2:]).all()
    s = oracle.tok_block_scores(sh, oracle.make_params(), *args)           # w = 1/H_idx
    assert s[0, :2].tolist() == [2.5, 2.0]
    s = oracle.tok_block_scores(sh, oracle.make_params(temperature=2.0), *args)
    assert s[0, :2].tolist() == [1.25, 1.0]


def test_tok_page_indirection_and_invariance():
    rng = np.random.default_rng(3)
    q = _bf16_bits(rng.normal(size=(1, 2, 128)))
    keys = rng.normal(size=(3, 64, 2, 128)).astype(np.float32) * 0.1
    keys[2, 17, 0] = 10.0 * np.asarray(q[0, 0].view(np.uint16).astype(np.uint32) << 16,
                                       np.uint32).view(np.float32)    # a hot token
    sh = _tok_shape(1, 4, 2, 3, 3)
    pt = np.array([[1, 2, 0]], np.int32)     # logical page 1 -> physical page 2
    lens = np.array([192], np.int32)
    s = oracle.tok_block_scores(sh, oracle.make_params(), q, None, _bf16_bits(keys), pt, lens)
    assert int(np.argmax(s[0, :12])) == 4 + 17 // 16          # logical block 5
    perm = np.array([2, 0, 1])               # physical page i moves to perm[i]
    moved = np.empty_like(keys)
    moved[perm] = keys
    s2 = oracle.tok_block_scores(sh, oracle.make_params(), q, None, _bf16_bits(moved),
                                 perm[pt].astype(np.int32), lens)
    assert np.array_equal(s, s2, equal_nan=True)


def _tok_problem(rng, B=1, Hq=4, Hkv=2, L=160, idx_heads=2):
    npg = (L + 63) // 64
    q_idx = _bf16_bits(rng.normal(size=(B, idx_heads, 128)) * 0.3)
    sel_tok = _bf16_bits(rng.normal(size=(B * npg, 64, idx_heads, 128)))
    (q, k, v), (q64, k64, v64) = _rand_kv(rng, B * npg, Hkv, Hq, B)
    pt = rng.permutation(B * npg).astype(np.int32).reshape(B, npg)
    sh = _tok_shape(B, Hq, Hkv, B * npg, npg, idx_heads)
    return sh, q_idx, sel_tok, (q, k, v), (q64, k64, v64), pt


def _tok_tokens(k64, v64, pt, b, g, positions):
    rows_k = torch.stack([k64[pt[b, t // 64], g, t % 64] for t in positions])
    rows_v = torch.stack([v64[pt[b, t // 64], g, t % 64] for t in positions])
    return rows_k, rows_v


def test_tok_all_blocks_is_dense_attention_for_every_head():
    rng = np.random.default_rng(8)
    L = 150
    sh, q_idx, sel_tok, (q, k, v), (q64, k64, v64), pt = _tok_problem(rng, L=L)
    pr = oracle.make_params(sink_blocks=1, recency_blocks=1, kmin_blocks=0)
    r = oracle.tok_decode_step(sh, pr, q_idx, None, sel_tok, _bf16_bits(q), _bf16_bits(k),
                               _bf16_bits(v), pt, np.array([L], np.int32),
                               np.array([1.0], np.float32), 1 / math.sqrt(128))
    nb = (L + 15) // 16
    assert r["sel_idx"][0, :r["sel_cnt"][0]].tolist() == list(range(nb))
    G = 2
    for h in range(4):
        kk, vv = _tok_tokens(k64, v64, pt, 0, h // G, range(L))
        ref = _sdpa(q64[0, h], kk, vv, 1 / math.sqrt(128))
        assert np.allclose(r["out"][0, h], ref.numpy(), atol=1e-12, rtol=1e-10)


def test_tok_topk_selection_feeds_attention_of_every_head():
    # Static top-K with no reserved blocks keeps exactly the planted blocks;
    # every head then attends exactly their tokens (16-token granularity
    # inside 64-token pages).
    rng = np.random.default_rng(9)
    L = 256
    sh, q_idx, sel_tok, (q, k, v), (q64, k64, v64), pt = _tok_problem(rng, L=L)
    tok = sel_tok.copy()
    hot = [2, 5, 13]
    qv = torch.as_tensor(q_idx.view(np.int16)).view(torch.bfloat16).double().numpy()[0]
    keys = torch.as_tensor(tok.view(np.int16)).view(torch.bfloat16).float().numpy()
    for j in hot:
        for t in range(16 * j, 16 * j + 16):
            keys[pt[0, t // 64], t % 64] += 20.0 * qv / np.linalg.norm(qv, axis=1, keepdims=True)
    tok = _bf16_bits(keys)
    pr = oracle.make_params(mode="topk", sink_blocks=0, recency_blocks=0, topk_blocks=3)
    r = oracle.tok_decode_step(sh, pr, q_idx, None, tok, _bf16_bits(q), _bf16_bits(k),
                               _bf16_bits(v), pt, np.array([L], np.int32),
                               np.array([0.9], np.float32), 0.1)
    assert r["sel_idx"][0, :r["sel_cnt"][0]].tolist() == hot
    pos = [t for j in hot for t in range(16 * j, 16 * j + 16)]
    for h in range(4):
        kk, vv = _tok_tokens(k64, v64, pt, 0, h // 2, pos)
        ref = _sdpa(q64[0, h], kk, vv, 0.1)
        assert np.allclose(r["out"][0, h], ref.numpy(), atol=1e-12, rtol=1e-10)


def test_tok_reserved_blocks_and_incomplete_last_block():
    rng = np.random.default_rng(10)
    L = 16 * 10 + 5                           # 11 blocks, the last one incomplete
    sh, q_idx, sel_tok, (q, k, v), _, pt = _tok_problem(rng, L=L)
    pr = oracle.make_params(sink_blocks=2, recency_blocks=2, kmin_blocks=0)
    r = oracle.tok_decode_step(sh, pr, q_idx, None, sel_tok, _bf16_bits(q), _bf16_bits(k),
                               _bf16_bits(v), pt, np.array([L], np.int32),
                               np.array([0.0], np.float32), 0.1)
    # p = 0: empty nucleus; the incomplete block 10 joins the recency blocks
    assert r["sel_idx"][0, :r["sel_cnt"][0]].tolist() == [0, 1, 9, 10]
    pr = oracle.make_params(sink_blocks=2, recency_blocks=2, kmin_blocks=6)
    r2 = oracle.tok_decode_step(sh, pr, q_idx, None, sel_tok, _bf16_bits(q), _bf16_bits(k),
                                _bf16_bits(v), pt, np.array([L], np.int32),
                                np.array([0.0], np.float32), 0.1)
    s = oracle.tok_block_scores(sh, pr, q_idx, None, sel_tok, pt, np.array([L], np.int32))[0]
    best = sorted(range(2, 9), key=lambda j: (-s[j], j))[:2]           # K_min floor of 6
    assert r2["sel_idx"][0, :r2["sel_cnt"][0]].tolist() == sorted([0, 1, 9, 10] + best)


# ------------------------------------------------------------ sparse prefill
# A chunk's queries are grouped into tiles (queries whose positions share a
# KV block); each tile selects like a decode query at the tile's last
# position, from block scores maxed over its queries, and every query
# attends causally over its tile's selection.

def _prefill_problem(rng, lens, qlens, Hq=4, Hkv=2, fmt="bf16"):
    B = len(lens)
    nbs = [(L + 63) // 64 for L in lens]
    mb = max(nbs)
    P = sum(nbs)
    rows = sum(qlens)
    q_sel = rng.normal(size=(rows, Hq, 64)).astype(np.float32)
    keys = rng.normal(size=(P, Hkv, 64)).astype(np.float32)
    (q, k, v), (q64, k64, v64) = _rand_kv(rng, P, Hkv, Hq, rows)
    perm = rng.permutation(P).astype(np.int32)
    pt = np.full((B, mb), -1, np.int32)
    off = 0
    for b, n in enumerate(nbs):
        pt[b, :n] = perm[off:off + n]
        off += n
    sh = oracle.make_shape(B, Hq, Hkv, 128, 64, 64, fmt, P, mb)
    return sh, q_sel, keys, (q, k, v), (q64, k64, v64), pt


def _prefill(sh, pr, q_sel, keys, qkv, pt, lens, qlens, p, scale=0.1):
    q, k, v = qkv
    return oracle.prefill_step(sh, pr, _bf16_bits(q_sel), None, _bf16_bits(keys), None,
                               _bf16_bits(q), _bf16_bits(k), _bf16_bits(v), pt,
                               np.array(lens, np.int32), np.array(qlens, np.int32),
                               np.full(len(lens), p, np.float32), scale)


def test_prefill_single_query_chunk_equals_decode():
    rng = np.random.default_rng(20)
    lens, qlens = [300, 64, 1000], [1, 1, 1]
    sh, q_sel, keys, qkv, _, pt = _prefill_problem(rng, lens, qlens)
    pr = oracle.make_params(sink_blocks=1, recency_blocks=2, kmin_blocks=4)
    pf = _prefill(sh, pr, q_sel, keys, qkv, pt, lens, qlens, 0.8)
    q, k, v = qkv
    dec = oracle.decode_step(sh, pr, _bf16_bits(q_sel), None, _bf16_bits(keys), None,
                             _bf16_bits(q), _bf16_bits(k), _bf16_bits(v), pt,
                             np.array(lens, np.int32), np.full(3, 0.8, np.float32), 0.1)
    assert len(pf["tiles"]) == 3
    for t in range(3):
        for g in range(2):
            a = pf["sel_idx"][t, g, :pf["sel_cnt"][t, g]].tolist()
            assert a == dec["sel_idx"][t, g, :dec["sel_cnt"][t, g]].tolist()
    assert np.array_equal(pf["out"], dec["out"])
    assert np.array_equal(pf["lse"], dec["lse"])


def test_prefill_keep_all_is_causal_dense_attention():
    rng = np.random.default_rng(21)
    lens, qlens = [200, 130], [150, 67]       # chunks start mid-block
    sh, q_sel, keys, qkv, (q64, k64, v64), pt = _prefill_problem(rng, lens, qlens)
    pr = oracle.make_params(sink_blocks=1, recency_blocks=1, kmin_blocks=0)
    pf = _prefill(sh, pr, q_sel, keys, qkv, pt, lens, qlens, 1.0)
    row = 0
    for b, (L, T) in enumerate(zip(lens, qlens)):
        for i in range(T):
            pos = L - T + i
            for h in range(4):
                kk = torch.stack([k64[pt[b, t // 64], h // 2, t % 64] for t in range(pos + 1)])
                vv = torch.stack([v64[pt[b, t // 64], h // 2, t % 64] for t in range(pos + 1)])
                ref = _sdpa(q64[row, h], kk, vv, 0.1)
                assert np.allclose(pf["out"][row, h], ref.numpy(), atol=1e-12, rtol=1e-10), (b, i, h)
            row += 1


def test_prefill_tile_score_is_the_max_over_its_queries():
    rng = np.random.default_rng(22)
    lens, qlens = [260], [100]               # tiles: [160, 191], [192, 255], [256, 259]
    sh, q_sel, keys, qkv, _, pt = _prefill_problem(rng, lens, qlens)
    pr = oracle.make_params()
    sc = oracle.prefill_scores(sh, pr, _bf16_bits(q_sel), None, _bf16_bits(keys), None, pt,
                               np.array(lens, np.int32), np.array(qlens, np.int32))
    tiles = oracle.prefill_tiles(lens, qlens)
    assert [(lo, hi) for _, lo, hi, _ in tiles] == [(160, 191), (192, 255), (256, 259)]
    # each query scored alone (as a decode query) against its tile's blocks:
    # the complete blocks below the tile's last position + 1
    rows = 100
    dsh = oracle.make_shape(rows, 4, 2, 128, 64, 64, "bf16", sh.num_pages, sh.max_blocks)
    tile_end = np.concatenate([np.full(hi - lo + 1, hi + 1) for _, lo, hi, _ in tiles])
    per_q = oracle.block_scores(dsh, pr, _bf16_bits(q_sel), None, _bf16_bits(keys), None,
                                np.repeat(pt, rows, axis=0), tile_end.astype(np.int32))
    for t, (_, lo, hi, r0) in enumerate(tiles):
        nf = (hi + 1) // 64
        want = np.max(per_q[r0:r0 + hi - lo + 1, :, :nf], axis=0)
        assert np.array_equal(sc[t, :, :nf], want), t
        assert np.isnan(sc[t, :, nf:]).all()


def test_prefill_causal_mask_and_tile_recency():
    rng = np.random.default_rng(23)
    lens, qlens = [512], [130]
    sh, q_sel, keys, (q, k, v), _, pt = _prefill_problem(rng, lens, qlens)
    pr = oracle.make_params(sink_blocks=1, recency_blocks=2, kmin_blocks=0)
    base = _prefill(sh, pr, q_sel, keys, (q, k, v), pt, lens, qlens, 0.5)
    # tiles [382, 383], [384, 447], [448, 511]: each keeps block 0 and its last two blocks
    for t, (_, lo, hi, _) in enumerate(base["tiles"]):
        nb = (hi + 1 + 63) // 64
        s = set(base["sel_idx"][t, 0, :base["sel_cnt"][t, 0]].tolist())
        assert {0, nb - 2, nb - 1} <= s and max(s) == nb - 1
    # keys / values after position 400 change: rows of queries at <= 400 do not
    k2, v2 = k.copy(), v.copy()
    for t in range(401, 512):
        k2[pt[0, t // 64], :, t % 64] += 5.0
        v2[pt[0, t // 64], :, t % 64] -= 7.0
    pert = _prefill(sh, pr, q_sel, keys, (q, k2, v2), pt, lens, qlens, 0.5)
    r400 = 400 - 382
    assert np.array_equal(base["out"][:r400 + 1], pert["out"][:r400 + 1])
    assert not np.allclose(base["out"][r400 + 1:], pert["out"][r400 + 1:])


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "fp8", "int8"])
def test_tok_quantised_keys_follow_the_key_quantiser(fmt):
    # Each (token, head) key row of 128 elements is stored like a selector
    # key row of that format (pinned quantiser above); the scores are the
    # plain token scores of the read-back rows, maxed over 16-token blocks.
    rng = np.random.default_rng(30)
    P, Hi, L = 3, 2, 150
    keys = _bf16_bits(rng.normal(size=(P, 64, Hi, 128)))
    data, scales = oracle.quantize_selector(fmt, keys)
    q = _bf16_bits(rng.normal(size=(1, Hi, 128)) * 0.3)
    w = np.array([[0.7, 0.4]], np.float32)
    pt = np.array([[2, 0, 1]], np.int32)
    sh = oracle.make_tok_shape(1, 4, 2, P, 3, idx_heads=Hi, sel_fmt=fmt)
    got = oracle.tok_block_scores(sh, oracle.make_params(), q, w, data, pt,
                                  np.array([L], np.int32), sel_scales=scales)
    kd = oracle.dequant_selector(fmt, data.reshape(-1, data.shape[-1]),
                                 None if scales is None else scales.reshape(-1, scales.shape[-1]),
                                 128).reshape(P, 64, Hi, 128)
    qd = torch.as_tensor(q.view(np.int16)).view(torch.bfloat16).double().numpy()[0]
    for j in range(L // 16):
        tok = []
        for t in range(16 * j, 16 * j + 16):
            dots = np.einsum("hd,hd->h", qd, kd[pt[0, t // 64], t % 64])
            tok.append(float((w[0] * np.maximum(dots, 0.0)).sum()))
        assert abs(got[0, j] - max(tok)) <= 1e-12 * max(1.0, abs(max(tok))), j
    assert np.isnan(got[0, L // 16:]).all()


@pytest.mark.parametrize("fmt", ["int4", "mxfp4", "fp8", "int8"])
def test_tok_quantised_queries_follow_the_key_quantiser(fmt):
    # With quantize_queries each index head's 128-element query row goes
    # through the key format's quantiser (pinned above) and is read back
    # exactly; the scores are the plain token scores of the read-back query
    # and key rows.
    rng = np.random.default_rng(31)
    P, Hi, L = 2, 2, 100
    keys = _bf16_bits(rng.normal(size=(P, 64, Hi, 128)))
    data, scales = oracle.quantize_selector(fmt, keys)
    q = _bf16_bits(rng.normal(size=(1, Hi, 128)) * 0.3)
    w = np.array([[0.6, 0.5]], np.float32)
    pt = np.array([[1, 0]], np.int32)
    sh = oracle.make_tok_shape(1, 4, 2, P, 2, idx_heads=Hi, sel_fmt=fmt)
    got = oracle.tok_block_scores(sh, oracle.make_params(quantize_queries=True), q, w, data, pt,
                                  np.array([L], np.int32), sel_scales=scales)
    kd = oracle.dequant_selector(fmt, data.reshape(-1, data.shape[-1]),
                                 None if scales is None else scales.reshape(-1, scales.shape[-1]),
                                 128).reshape(P, 64, Hi, 128)
    qc, qs = oracle.quantize_selector(fmt, q[0])
    qd = oracle.dequant_selector(fmt, qc, qs, 128)
    plain = oracle.tok_block_scores(sh, oracle.make_params(), q, w, data, pt,
                                    np.array([L], np.int32), sel_scales=scales)
    differs = False
    for j in range(L // 16):
        tok = []
        for t in range(16 * j, 16 * j + 16):
            dots = np.einsum("hd,hd->h", qd, kd[pt[0, t // 64], t % 64])
            tok.append(float((w[0] * np.maximum(dots, 0.0)).sum()))
        assert abs(got[0, j] - max(tok)) <= 1e-12 * max(1.0, abs(max(tok))), j
        differs |= got[0, j] != plain[0, j]
    assert differs                      # the queries really were quantised


@pytest.mark.parametrize("fmt", ["mxfp4", "fp8"])
def test_tok_quantised_queries_lossless_on_small_integers(fmt):
    # Queries in {-3..3} are stored exactly by MXFP4 (power-of-two group
    # scales) and E4M3, so quantising them changes no score; bf16 keys ignore
    # the switch altogether.
    rng = np.random.default_rng(32)
    P, Hi, L = 2, 4, 128
    keys = _bf16_bits(rng.integers(-3, 4, size=(P, 64, Hi, 128)).astype(np.float64))
    data, scales = oracle.quantize_selector(fmt, keys)
    q = _bf16_bits(rng.integers(-3, 4, size=(1, Hi, 128)).astype(np.float64))
    pt = np.array([[0, 1]], np.int32)
    sh = oracle.make_tok_shape(1, 4, 2, P, 2, idx_heads=Hi, sel_fmt=fmt)
    a = oracle.tok_block_scores(sh, oracle.make_params(quantize_queries=True), q, None, data, pt,
                                np.array([L], np.int32), sel_scales=scales)
    b = oracle.tok_block_scores(sh, oracle.make_params(), q, None, data, pt,
                                np.array([L], np.int32), sel_scales=scales)
    assert np.array_equal(a, b)
    shb = oracle.make_tok_shape(1, 4, 2, P, 2, idx_heads=Hi)
    c = oracle.tok_block_scores(shb, oracle.make_params(quantize_queries=True), q, None, keys, pt,
                                np.array([L], np.int32))
    d = oracle.tok_block_scores(shb, oracle.make_params(), q, None, keys, pt,
                                np.array([L], np.int32))
    assert np.array_equal(c, d)
