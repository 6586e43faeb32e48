"""Pins for the oracle's MXFP8 expert FFN over gathered rows and for the tiled
scale layout the block-scaled tensor cores read (CPU only).

The layout helper is checked from the other side of its definition, the
shared-memory-to-TMEM copy (32 rows x 128 bits, replicated into the four lane
quarters): TMEM lane i, column c, byte j of an atom's copy holds the scale of
row 32c + i, block j. The FFN is pinned on a special case that reduces it to
a library routine (unit-vector rows, MX-exact weights, a permutation as the
down projection: y = mx(silu(W1[e][j]) * W3[e][j]) with silu from scipy's
expit), and against the bf16 FFN of the oracle (close, not equal).
"""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from combine_top_route_counting_b200 import inputs
from tests.helpers import bf16_to_f64, bits, mx_tiled_offsets, to_tiled


def test_tiled_offsets_are_the_tmem_copy_layout():
    R, K = 384, 512
    off = mx_tiled_offsets(R, K)
    KB = K // 32
    # a bijection onto the table's R*K/32 bytes
    assert np.array_equal(np.sort(off.reshape(-1)), np.arange(R * KB))
    row_of = np.empty(R * KB, np.int64)
    blk_of = np.empty(R * KB, np.int64)
    row_of[off.reshape(-1)] = np.repeat(np.arange(R), KB)
    blk_of[off.reshape(-1)] = np.tile(np.arange(KB), R)
    atoms_per_rowblock = K // 128
    for atom in range(R * KB // 512):
        rb, kb4 = divmod(atom, atoms_per_rowblock)
        for i in range(32):              # TMEM lane (in every quarter)
            for c in range(4):           # TMEM column
                for j in range(4):       # byte of the 32-bit cell = scale id
                    byte = atom * 512 + 16 * i + 4 * c + j
                    assert row_of[byte] == rb * 128 + 32 * c + i
                    assert blk_of[byte] == kb4 * 4 + j


def test_to_tiled_round_trip():
    rng = np.random.default_rng(5)
    s = rng.integers(0, 255, (256, 8), dtype=np.uint8)
    t = to_tiled(s)
    assert t.shape == (256 * 8,)
    assert np.array_equal(t[mx_tiled_offsets(256, 256)], s)
    with pytest.raises(ValueError):
        mx_tiled_offsets(100, 256)


def _mx_exact_bf16(W: np.ndarray, axis: int) -> np.ndarray:
    """W rounded to MXFP8 along `axis` (values exactly representable in bf16)."""
    r = oracle.mx_round(W, axis=axis)
    b = torch.from_numpy(r).to(torch.bfloat16)
    assert np.array_equal(b.to(torch.float64).numpy(), r)  # E4M3 x 2^e fits bf16
    return bits(b)


def test_ffn_rows_mxfp8_unit_rows_reduce_to_swiglu():
    H = I = 128
    rng = np.random.default_rng(11)
    W1, W3, W2 = {}, {}, {}
    perm = {0: rng.permutation(I), 1: rng.permutation(I)}
    for e in (0, 1):
        W1[e] = _mx_exact_bf16(rng.standard_normal((H, I)) * 0.7, axis=0)
        W3[e] = _mx_exact_bf16(rng.standard_normal((H, I)) * 1.3, axis=0)
        P = np.zeros((I, H))
        P[np.arange(I), perm[e]] = 1.0   # h @ P moves column i to column perm[i]
        W2[e] = bits(torch.from_numpy(P).to(torch.bfloat16))
    js = [3, 77, 3, 127, 0, 64]
    ex = [0, 1, 1, 0, 1, 0]
    x = np.zeros((len(js), H))
    x[np.arange(len(js)), js] = 1.0
    xg = bits(torch.from_numpy(x).to(torch.bfloat16))
    hq, hs, y = oracle.ffn_rows_mxfp8(xg, ex, W1, W3, W2, H, I)
    for r, (j, e) in enumerate(zip(js, ex)):
        a = bf16_to_f64(W1[e][j])
        b = bf16_to_f64(W3[e][j])
        h = a * expit(a) * b               # silu(a) * b through the library's logistic
        h = h.astype(np.float32).astype(np.float64)  # quantised from fp32, as the kernel holds h
        q, s = oracle.mx_quantize(h)
        assert np.array_equal(hq[r], q) and np.array_equal(hs[r], s), r
        dq = oracle.mx_dequantize(q, s)
        expect_y = np.zeros(H)
        expect_y[perm[e]] = dq
        assert np.array_equal(y[r], expect_y), r


def test_ffn_rows_mxfp8_quantises_weights_along_the_reduction_axis():
    """A planted weight of 2^20 sets the shared scale of its own 32-block along
    the reduction dimension to 2^12, where E4M3 (smallest step 2^-9) flushes
    the block's other entries, of magnitude <= 1, to exactly zero; blocks
    along the other axis are untouched. Unit-vector rows and an identity down
    projection read the flushed entries directly."""
    H = I = 128
    rng = np.random.default_rng(17)
    W1 = rng.uniform(0.5, 1.0, (H, I)) * rng.choice([-1.0, 1.0], (H, I))
    W3 = rng.uniform(0.5, 1.0, (H, I))
    k0, i0 = 37, 5                        # W1: K-block 1 (rows 32..63) of column 5
    W1[k0, i0] = 2.0 ** 20
    W2 = np.eye(I)
    i1, c1 = 70, 66                       # W2: I-block 2 (rows 64..95) of column 66
    W2[i1, c1] = 2.0 ** 20
    to_bits = lambda a: {0: bits(torch.from_numpy(a).to(torch.bfloat16))}
    js = [40, 90, k0]                     # same K-block as k0, another block, k0 itself
    x = np.zeros((len(js), H))
    x[np.arange(len(js)), js] = 1.0
    xg = bits(torch.from_numpy(x).to(torch.bfloat16))
    hq, hs, y = oracle.ffn_rows_mxfp8(xg, [0] * len(js), to_bits(W1), to_bits(W3), to_bits(W2),
                                      H, I)
    h = oracle.mx_dequantize(hq, hs)
    assert h[0, i0] == 0.0                # W1[40, 5] flushed: a = 0, silu(0) * b = 0
    assert h[0, i0 + 1] != 0.0 and h[1, i0] != 0.0  # other column, other K-block: kept
    assert h[2, i0] > 2.0 ** 18           # the planted weight itself: silu(2^20) * b
    for r in range(len(js)):
        # column 66 of W2: its diagonal 1 (row 66, same I-block as row 70) is
        # flushed and only the planted 2^20 remains; column 70 keeps its 1
        assert y[r, c1] == h[r, i1] * 2.0 ** 20, r
        assert y[r, i1] == h[r, i1], r


def test_ffn_rows_mxfp8_close_to_bf16_ffn():
    w = inputs.Workload("mx_ffn", 12, P=1, N=40, E=3, k=1, H=128, I=64)
    W = [{e: bits(t[e]) for e in range(w.E)} for t in inputs.make_weights(w)]
    xg = bits(inputs.make_x(w))
    ex = np.arange(w.n_tokens) % w.E
    hq, hs, y = oracle.ffn_rows_mxfp8(xg, ex, *W, w.H, w.I)
    hb, yb = oracle.ffn_rows(xg, ex, *W, w.H, w.I)
    rel_y = np.sqrt(np.mean((y - yb) ** 2) / np.mean(yb ** 2))
    assert 1e-3 < rel_y < 0.1, rel_y
    h_mx = oracle.mx_dequantize(hq, hs)
    h_bf = bf16_to_f64(hb)
    rel_h = np.sqrt(np.mean((h_mx - h_bf) ** 2) / np.mean(h_bf ** 2))
    assert 1e-3 < rel_h < 0.1, rel_h
    assert hs.shape == (w.n_tokens, w.I // 32)


def _shared_case():
    w = inputs.Workload("mx_shared", 14, P=1, N=16, E=4, k=2, H=128, I=64)
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W = inputs.make_weights(w)
    g = torch.Generator().manual_seed(77)
    Ws = [(torch.randn(shape, generator=g) * 0.02).to(torch.bfloat16)
          for shape in ((w.H, w.I), (w.H, w.I), (w.I, w.H))]
    return w, lg, x, W, Ws


def test_layer_mxfp8_shared_expert_alone_is_a_dense_swiglu():
    """With every routed W2 zero the routed experts add exact zeros, and the
    layer is the shared expert alone: a dense bf16 SwiGLU (torch fp64 matmuls
    on the bf16 weights, h rounded to bf16 as the FFN's operand)."""
    w, lg, x, W, Ws = _shared_case()
    Wr = [{e: bits(t[e]) for e in range(w.E)} for t in (W[0], W[1], torch.zeros_like(W[2]))]
    toks = range(w.n_tokens)
    res = oracle.layer_tokens_mxfp8(lg, bits(x), Wr, w.k, w.H, w.I, toks,
                                    shared=tuple(bits(t) for t in Ws))
    x64, w1, w3, w2 = (t.to(torch.float64) for t in (x, *Ws))
    a, b = x64 @ w1, x64 @ w3
    h = (torch.nn.functional.silu(a) * b).to(torch.bfloat16).to(torch.float64)
    ref = (h @ w2).numpy()
    assert np.allclose(res["out64"], ref, rtol=1e-12, atol=1e-15)


def test_layer_mxfp8_shared_expert_adds_once_per_token_with_gate_one():
    w, lg, x, W, Ws = _shared_case()
    Wr = [{e: bits(t[e]) for e in range(w.E)} for t in W]
    toks = range(w.n_tokens)
    sb = lambda s2: (bits(Ws[0]), bits(Ws[1]), bits(s2))
    base = oracle.layer_tokens_mxfp8(lg, bits(x), Wr, w.k, w.H, w.I, toks)["out64"]
    zero = oracle.layer_tokens_mxfp8(lg, bits(x), Wr, w.k, w.H, w.I, toks,
                                     shared=sb(torch.zeros_like(Ws[2])))["out64"]
    one = oracle.layer_tokens_mxfp8(lg, bits(x), Wr, w.k, w.H, w.I, toks, shared=sb(Ws[2]))["out64"]
    two = oracle.layer_tokens_mxfp8(lg, bits(x), Wr, w.k, w.H, w.I, toks,
                                    shared=sb((Ws[2].float() * 2).to(torch.bfloat16)))["out64"]
    assert np.array_equal(zero, base)                      # a zero shared expert adds nothing
    d1, d2 = one - base, two - base
    assert np.abs(d1).max() > 0
    assert np.allclose(d2, 2 * d1, rtol=1e-12, atol=1e-15)  # linear in Ws2, weight 1, not gated
