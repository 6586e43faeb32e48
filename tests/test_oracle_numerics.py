"""Pins for the oracle's routing, bf16 rounding, SwiGLU FFN, combine and the whole
layer (CPU only). Each is checked against a library routine, exact rational
arithmetic, or a direct per-token definition that does not use the schedule."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from combine_top_route_counting_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers
def exact_round_bf16(v: float) -> int:
    """Round-to-nearest-even of a finite double to bf16, in exact rational arithmetic."""
    if v == 0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    fr = Fraction(v)
    sign = 1 if fr < 0 else 0
    a = abs(fr)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (e - 7)          # 8 significant bits
    m = a / q
    lo = math.floor(m)
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    val = float(lo * q)
    bits = int(np.array([val], np.float32).view(np.uint32)[0] >> 16)
    return bits | (sign << 15)


def bits_round_bf16(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float64 values to bf16 via integer bit arithmetic on
    the float64 encoding (keep 7 of 52 explicit mantissa bits)."""
    u = np.ascontiguousarray(x, np.float64).view(np.uint64)
    keep_lsb = (u >> np.uint64(45)) & np.uint64(1)
    u2 = (u + np.uint64((1 << 44) - 1) + keep_lsb) & ~np.uint64((1 << 45) - 1)
    f32 = u2.view(np.float64).astype(np.float32)   # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def exact_fmaf(a: float, b: float, c: float) -> float:
    """fp32 fused multiply-add in exact arithmetic, one round-to-nearest-even to fp32."""
    s = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    if s == 0:
        return 0.0 if not (math.copysign(1, a * b) < 0 and math.copysign(1, c) < 0) else -0.0
    sign = -1 if s < 0 else 1
    m = abs(s)
    e = math.floor(math.log2(m))
    while Fraction(2) ** e > m:
        e -= 1
    while Fraction(2) ** (e + 1) <= m:
        e += 1
    q = Fraction(2) ** (max(e, -126) - 23)
    t = m / q
    lo = math.floor(t)
    rem = t - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * float(lo * q)


# ---------------------------------------------------------------- bf16 rounding
def test_round_bf16_exact_rational():
    rng = np.random.default_rng(1)
    vals = list(rng.normal(size=300) * 10.0 ** rng.integers(-6, 6, size=300))
    # exact ties and near-ties of bf16
    for m in (1.0, 1.5, 3.0, 100.0):
        ulp = 2.0 ** (math.floor(math.log2(m)) - 7)
        vals += [m + ulp / 2, m + 1.5 * ulp, m + ulp / 2 + 1e-13, m + ulp / 2 - 1e-13, -(m + ulp / 2)]
    for v in vals:
        assert oracle.round_bf16(v) == exact_round_bf16(v), v


def test_round_bf16_matches_torch_on_fp32_values():
    x = torch.randn(10000, generator=torch.Generator().manual_seed(3)) * 7
    ours = np.array([oracle.round_bf16(float(v)) for v in x.tolist()], np.uint16)
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (ours == ref).all()


# ---------------------------------------------------------------- routing
def test_topk_matches_torch():
    lg = torch.randn(2000, 64, generator=torch.Generator().manual_seed(5))
    for k in (1, 2, 4, 8, 64):
        ids, g32, g64 = oracle.route_topk(lg, k)
        v, i = torch.topk(lg.double(), k, dim=1)
        assert (ids == i.numpy()).all()
        ref = torch.softmax(v, dim=1).numpy()
        np.testing.assert_allclose(g64, ref, rtol=1e-14, atol=0)
        assert (g32 == g64.astype(np.float32)).all()
        np.testing.assert_allclose(g64.sum(1), 1.0, rtol=1e-14)


def test_topk_ties_and_neg_inf_golden():
    w = json.load(open(os.path.join(GOLD, "worked_numbers.json")))["topk_ties"]
    lg = np.array([[float(v) for v in w["logits"]]], np.float32)
    ids, g32, g64 = oracle.route_topk(lg, w["k"])
    assert ids[0].tolist() == w["ids"]
    d = 2 + math.exp(-2.0)
    np.testing.assert_allclose(g64[0], [1 / d, 1 / d, math.exp(-2.0) / d], rtol=1e-15)


def test_topk_never_picks_forced_empty_experts():
    w = inputs.Workload("z", 4, P=1, N=256, E=64, k=8, H=0, I=0, logits="zipf", n_empty=8)
    lg = inputs.make_logits(w)
    empties = inputs.empty_experts(w)
    ids, _, g64 = oracle.route_topk(lg, 8)
    assert not np.isin(ids, empties).any()
    assert np.isfinite(g64).all()


# ---------------------------------------------------------------- FFN
def _weights(E, H, I, seed):
    g = torch.Generator().manual_seed(seed)
    W1 = (torch.randn(E, H, I, generator=g) * 0.05).to(torch.bfloat16)
    W3 = (torch.randn(E, H, I, generator=g) * 0.05).to(torch.bfloat16)
    W2 = (torch.randn(E, I, H, generator=g) * 0.05).to(torch.bfloat16)
    return W1, W3, W2


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _wdicts(W1, W3, W2):
    return tuple({e: _bits(W[e]) for e in range(W.shape[0])} for W in (W1, W3, W2))


def dense_swiglu(x, W1, W3, W2):
    """Dense SwiGLU MLP with torch fp64 matmuls; h rounded to bf16 by bit arithmetic."""
    a = x.double() @ W1.double()
    b = x.double() @ W3.double()
    s = (a * torch.sigmoid(a) * b).numpy()
    hb = bits_round_bf16(s)
    h = torch.from_numpy(bf16_bits_to_f64(hb))
    return hb, (h @ W2.double()).numpy()


def near_bf16_midpoint(v, rel=1e-12):
    """True where v lies within fp64 summation noise of the midpoint between two
    neighbouring bf16 values (the only place two correct fp64 evaluations of
    the same real number may round to different bf16 values)."""
    v = np.asarray(v, np.float64)
    lo = bf16_bits_to_f64(bits_round_bf16(v))
    ulp = np.abs(lo) * 2.0 ** -7
    mid_up, mid_dn = lo + ulp / 2, lo - ulp / 2
    return np.minimum(np.abs(v - mid_up), np.abs(v - mid_dn)) <= rel * np.abs(v)


def _assert_h_and_y_match_dense(h, y, x, W1, W3, W2):
    """h = bf16_rne of the exact silu(a)*b, equal to the dense fp64 path's except
    where the exact value sits on a rounding midpoint; y = h.W2 through the
    same h, within fp64 summation noise."""
    hb, _ = dense_swiglu(x, W1, W3, W2)
    a = x.double() @ W1.double()
    s = (a * torch.sigmoid(a) * (x.double() @ W3.double())).numpy()
    diff = h != hb
    assert diff.sum() <= 2 and near_bf16_midpoint(s[diff]).all(), int(diff.sum())
    y_dense = (torch.from_numpy(bf16_bits_to_f64(h)) @ W2.double()).numpy()
    np.testing.assert_allclose(y, y_dense, rtol=1e-11, atol=1e-13)
    rows_same = ~diff.any(axis=1)
    y_via_hb = (torch.from_numpy(bf16_bits_to_f64(hb)) @ W2.double()).numpy()
    np.testing.assert_allclose(y[rows_same], y_via_hb[rows_same], rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("H,I", [(64, 32), (128, 96)])
def test_ffn_single_expert_is_dense_swiglu(H, I):
    W1, W3, W2 = _weights(1, H, I, seed=H + I)
    x = torch.randn(40, H, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    h, y = oracle.ffn_rows(_bits(x), np.zeros(40, np.int32), *_wdicts(W1, W3, W2), H=H, I=I)
    _assert_h_and_y_match_dense(h, y, x, W1[0], W3[0], W2[0])


def test_ffn_h_is_rounded_once_from_the_exact_value():
    """Pairs (a, b) whose silu(a)*b lies between a bf16 rounding midpoint and the
    fp32 value next to it: rounding the exact value once and rounding it via
    fp32 give different bf16 values there. One token x = 1 and H = 1 make a, b
    the weights themselves; the oracle must follow the plain definition."""
    g = np.random.default_rng(17)
    a = bf16_bits_to_f64(bits_round_bf16(g.uniform(-4, 4, 4_000_000)))
    b = bf16_bits_to_f64(bits_round_bf16(g.uniform(-4, 4, 4_000_000)))
    s = a / (1.0 + np.exp(-a)) * b
    once = bits_round_bf16(s)
    twice = bits_round_bf16(s.astype(np.float32).astype(np.float64))
    pick = np.nonzero((once != twice) & ~near_bf16_midpoint(s, 1e-12))[0][:64]
    assert len(pick) >= 4, "the search finds double-rounding cases"
    n = len(pick)
    x = torch.ones((1, 1), dtype=torch.bfloat16)
    W1 = torch.from_numpy(a[pick]).reshape(1, 1, n).to(torch.bfloat16)
    W3 = torch.from_numpy(b[pick]).reshape(1, 1, n).to(torch.bfloat16)
    W2 = torch.zeros((1, n, 1), dtype=torch.bfloat16)
    h, _ = oracle.ffn_rows(_bits(x), np.zeros(1, np.int32), *_wdicts(W1, W3, W2), H=1, I=n)
    assert (h[0] == once[pick]).all()
    assert (h[0] != twice[pick]).all()


def test_ffn_expert_selection_and_zero_rows():
    E, H, I = 3, 64, 32
    W1, W3, W2 = _weights(E, H, I, seed=11)
    x = torch.randn(30, H, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    x[5] = 0
    ex = np.array([i % E for i in range(30)], np.int32)
    h, y = oracle.ffn_rows(_bits(x), ex, *_wdicts(W1, W3, W2), H=H, I=I)
    assert (h[5] == 0).all() and (y[5] == 0).all(), "silu(0)*0 = 0: padding rows stay zero"
    for e in range(E):
        m = ex == e
        _assert_h_and_y_match_dense(h[m], y[m], x[torch.from_numpy(m)], W1[e], W3[e], W2[e])


# ---------------------------------------------------------------- combine
def test_combine_f64_is_weighted_sum():
    rng = np.random.default_rng(4)
    y = rng.normal(size=(20, 48))
    sel = rng.integers(0, 20, size=(9, 3))
    g = rng.random(size=(9, 3))
    out64, outb = oracle.combine_f64(y, sel, g, 3)
    ref = np.einsum("aj,ajc->ac", g, y[sel])
    np.testing.assert_allclose(out64, ref, rtol=1e-14, atol=1e-15)
    assert (outb == bits_round_bf16(out64)).all()


def test_combine_f32_fixed_order_fma():
    rng = np.random.default_rng(6)
    y = rng.normal(size=(12, 16)).astype(np.float32)
    sel = rng.integers(0, 12, size=(5, 4))
    g = rng.random(size=(5, 4)).astype(np.float32)
    outb = oracle.combine_f32(y, sel, g, 4)
    for a in range(5):
        for c in range(16):
            acc = 0.0
            for j in range(4):
                acc = exact_fmaf(g[a, j], y[sel[a, j], c], acc)
            assert outb[a, c] == exact_round_bf16(acc)
    # k = 1 with gate 1 is a plain bf16 rounding of y
    o1 = oracle.combine_f32(y, np.arange(12).reshape(12, 1), np.ones((12, 1), np.float32), 1)
    assert (o1 == bits_round_bf16(y.astype(np.float64))).all()


# ---------------------------------------------------------------- whole layer
def test_layer_equals_direct_per_token_definition():
    """Oracle route -> schedule -> dispatch -> FFN -> combine equals
    out[t] = sum_j g[t,j] * FFN_{id[t,j]}(x[t]) computed per token, with no
    schedule, gather or route_row involved."""
    w = inputs.WORKLOADS["tiny"]
    lg = inputs.make_logits(w)
    x = inputs.make_x(w)
    W1, W3, W2 = inputs.make_weights(w)
    toks = list(range(w.n_tokens))
    res = oracle.layer_tokens(lg, _bits(x), _wdicts(W1, W3, W2), w.P, w.N, w.k, w.E, w.H, w.I,
                              toks)
    v, idx = torch.topk(lg.double(), w.k, dim=1)
    g = torch.softmax(v, dim=1)
    assert (res["ids"] == idx.numpy()).all()
    direct = np.zeros((w.n_tokens, w.H))
    for e in range(w.E):
        m = (idx == e)
        rows = m.any(1).nonzero().flatten()
        if len(rows) == 0:
            continue
        _, ye = dense_swiglu(x[rows], W1[e], W3[e], W2[e])
        ge = (g * m).sum(1)[rows].numpy()
        direct[rows.numpy()] += ge[:, None] * ye
    scale = np.sqrt((direct ** 2).mean())
    err = np.abs(res["out64"] - direct) / np.maximum(np.abs(direct), scale)
    assert err.max() < 1e-9
    # every padded row of the tiny workload is accounted for
    s = res["sched"]
    assert s["offsets"][-1] == sum(-(-int(c.sum()) // 256) * 256 for c in s["counts"])
    # weights handed over a few experts at a time give the very same result
    W = _wdicts(W1, W3, W2)
    calls = []

    def by_group(ex):
        calls.append(list(ex))
        return tuple({e: d[e] for e in ex} for d in W)

    res2 = oracle.layer_tokens(lg, _bits(x), by_group, w.P, w.N, w.k, w.E, w.H, w.I, toks,
                               experts_per_group=3)
    assert len(calls) == 3 and sorted(sum(calls, [])) == list(range(w.E))
    assert (res2["out64"] == res["out64"]).all() and (res2["h"] == res["h"]).all()


def test_oracle_results_do_not_depend_on_its_thread_count():
    """The oracle splits rows and routes over OpenMP threads but every output
    element is computed by one thread in a fixed order: one thread and all
    threads give bitwise-identical schedules, FFN rows and gradients (the
    baseline is timed both ways)."""
    w = inputs.WORKLOADS["tiny_bwd"]
    lg, x, dout = inputs.make_logits(w), inputs.make_x(w), inputs.make_dout(w)
    W = inputs.make_weights(w)
    Wd = _wdicts(*W)
    ids, _, g64 = oracle.route_topk(lg, w.k)
    n_all = oracle.num_threads()

    def run():
        s = oracle.schedule(ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, w.pad)
        rows = np.nonzero(s["phi"][:, 0] >= 0)[0]
        xg = oracle.dispatch_rows(_bits(x), w.N, s["phi"], rows)
        ex = oracle.expert_of_rows(s["offsets"], rows)
        h, y = oracle.ffn_rows(xg, ex, *Wd, H=w.H, I=w.I)
        dys = oracle.dispatch_rows(_bits(dout), w.N, s["phi"], rows)
        bwd = oracle.ffn_bwd_rows(xg, dys, np.ones(len(rows)), ex, *Wd, H=w.H, I=w.I)
        return [s["phi"], s["offsets"], s["route_row"], h, y] + [np.asarray(v) for v in bwd.values()]

    try:
        oracle.set_num_threads(1)
        one = run()
    finally:
        oracle.set_num_threads(n_all)
    many = run()
    for a, b in zip(one, many):
        assert np.array_equal(a, b)
