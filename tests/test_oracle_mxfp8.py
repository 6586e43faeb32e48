"""Pins for the oracle's MXFP8 quantisation and MXFP8 layer (CPU only).

E4M3 decoding and rounding are checked against torch's float8_e4m3fn
conversions (a library routine); the saturation rule, the shared-scale rule
and the block axis against their definitions on constructed inputs; the MXFP8
layer against the bf16 layer of the oracle (close, not equal).
"""
import numpy as np
import torch

import oracle
from combine_top_route_counting_b200 import inputs
from tests.helpers import bits


def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_value(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all() and nan.sum() == 2  # 0x7F, 0xFF
    assert (ours[~nan] == ref[~nan]).all()
    assert np.nanmax(ours) == 448.0


def test_e4m3_encode_matches_torch_below_saturation():
    finite = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    grid = np.unique(finite[np.isfinite(finite)])
    mids = (grid[1:] + grid[:-1]) / 2                     # ties: to even
    rng = np.random.default_rng(1)
    rand = rng.standard_normal(20000) * np.exp2(rng.uniform(-12, 8, 20000))
    vals = np.concatenate([grid, mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf), rand,
                           [464.0, -464.0, 2.0 ** -10, -(2.0 ** -10), 1.5 * 2.0 ** -9]])
    vals = vals[np.abs(vals) <= 464.0]
    ours = oracle.e4m3_encode(vals)
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    exact32 = vals.astype(np.float32).astype(np.float64) == vals   # torch sees fp32 inputs
    assert (ours[exact32] == ref[exact32]).all()


def test_e4m3_encode_saturates_above_448():
    big = np.array([464.0001, 470.0, 480.0, 1e6, 3.0e38])
    assert (oracle.e4m3_encode(big) == 0x7E).all()
    assert (oracle.e4m3_encode(-big) == 0xFE).all()


def test_mx_scale_rule_and_error_bound():
    rng = np.random.default_rng(2)
    rows = []
    for mag in (1e-30, 1e-6, 0.02, 1.0, 3.7, 1e4, 1e30):
        rows.append(rng.standard_normal(256) * mag)
    z = np.zeros(256)
    z[40] = 0.5                                  # a block with one value, the rest zero
    rows += [np.zeros(256), z]
    v = np.stack(rows)
    q, s = oracle.mx_quantize(v)
    deq = oracle.mx_dequantize(q, s)
    X = np.exp2(s.astype(np.float64) - 127).repeat(32, axis=1)
    blocks = v.reshape(v.shape[0], -1, 32)
    amax = np.abs(blocks).max(2)
    # all-zero blocks: scale code 0 (2^-127) and zero codes
    zero = amax == 0
    assert (s[zero] == 0).all()
    assert (q.reshape(blocks.shape)[zero] == 0).all()
    # otherwise amax / X in [256, 512) unless the exponent was clamped
    r = amax[~zero] / np.exp2(s[~zero].astype(np.float64) - 127)
    clamped = (s[~zero] == 0) | (s[~zero] == 254)
    assert ((r >= 256) & (r < 512) | clamped).all()
    # element error: half an E4M3 step of v / X, or the clamp to 448
    w = v / X
    step_half = np.maximum(np.abs(w) * 2.0 ** -4, 2.0 ** -10)
    sat = np.abs(w) > 464
    err = np.abs(w - deq / X)
    assert (err[~sat] <= step_half[~sat]).all()
    assert (np.abs(deq[sat] / X[sat]) == 448).all()


def test_mx_round_blocks_run_along_the_reduction_axis():
    """A large entry changes the scale of its own 32-element block along the
    chosen axis only: the block axis is the axis passed (the GEMM's K)."""
    rng = np.random.default_rng(3)
    W = rng.standard_normal((128, 64)) * 0.02
    base = oracle.mx_round(W, axis=0)
    W2 = W.copy()
    W2[37, 5] = 50.0                      # row 37 lies in K-block 1 (rows 32..63)
    changed = oracle.mx_round(W2, axis=0) != base
    changed[37, 5] = False
    rows, cols = np.nonzero(changed)
    assert len(rows) > 0
    assert (cols == 5).all() and rows.min() >= 32 and rows.max() < 64


def test_mxfp8_layer_close_to_bf16_layer():
    w = inputs.Workload("mx_tiny", 10, P=1, N=24, E=4, k=2, H=128, I=64)
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W = [{e: bits(t[e]) for e in range(w.E)} for t in inputs.make_weights(w)]
    toks = range(w.n_tokens)
    mx = oracle.layer_tokens_mxfp8(lg, bits(x), W, w.k, w.H, w.I, toks)
    bf = oracle.layer_tokens(lg, bits(x), W, w.P, w.N, w.k, w.E, w.H, w.I, toks)
    rel = np.sqrt(np.mean((mx["out64"] - bf["out64"]) ** 2) / np.mean(bf["out64"] ** 2))
    assert 1e-3 < rel < 0.1, rel           # quantisation error, neither zero nor gross
    assert (mx["ids"] == bf["ids"]).all()
