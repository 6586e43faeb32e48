"""Pins for the oracle's backward (CPU only).

The oracle's exact mode (no bf16 rounding) is checked against torch.autograd
in fp64 on a dense formulation of the layer that uses no schedule, no rows
and no per-route loop: top-k by torch.topk, gates by torch.softmax, every
token's k experts applied with batched einsums. A dropped term, a wrong sign,
a transposed weight or a misplaced gate fails these. The rounded mode (the
one the GPU parity tests use) is pinned by its distance to the exact mode,
by exact invariants of the definition (linearity in the upstream gradient,
zero-sum router gradients, zero gradient for unused experts) and by the
agreement of the oracle's two independent weight-gradient paths.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import rms_floor_err


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def _bits_to_f64(b) -> torch.Tensor:
    u = np.asarray(b, np.uint16).astype(np.uint32) << 16
    return torch.from_numpy(u.view(np.float32).astype(np.float64))


def _case(T, E, k, H, I, seed, wscale=0.25):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn((T, E), generator=g, dtype=torch.float32)
    x = _bf16_bits(torch.randn((T, H), generator=g))
    dout = _bf16_bits(torch.randn((T, H), generator=g))
    W1 = _bf16_bits(torch.randn((E, H, I), generator=g) * wscale)
    W3 = _bf16_bits(torch.randn((E, H, I), generator=g) * wscale)
    W2 = _bf16_bits(torch.randn((E, I, H), generator=g) * wscale)
    return logits, x, dout, (W1, W3, W2)


def _as_dicts(W):
    return tuple({e: w[e] for e in range(w.shape[0])} for w in W)


def _torch_dense_grads(logits, x, dout, W, k):
    """fp64 autograd of out[t] = sum_j softmax(l[t, top])_j * SwiGLU_e(x[t]), e = top_j."""
    L = torch.from_numpy(logits.numpy().astype(np.float64)).requires_grad_(True)
    X = _bits_to_f64(x).requires_grad_(True)
    Ws = [_bits_to_f64(w).requires_grad_(True) for w in W]
    top = torch.topk(L.detach(), k, dim=1).indices              # [T,k]
    g = torch.softmax(L.gather(1, top), dim=1)                   # [T,k]
    a = torch.einsum("th,tjhi->tji", X, Ws[0][top])
    b = torch.einsum("th,tjhi->tji", X, Ws[1][top])
    h = torch.nn.functional.silu(a) * b
    y = torch.einsum("tji,tjih->tjh", h, Ws[2][top])
    out = (g.unsqueeze(-1) * y).sum(1)
    (out * _bits_to_f64(dout)).sum().backward()
    return dict(dx=X.grad.numpy(), dlogits=L.grad.numpy(), dW1=Ws[0].grad.numpy(),
                dW3=Ws[1].grad.numpy(), dW2=Ws[2].grad.numpy())


def _oracle_grads(logits, x, dout, W, k, exact):
    T = logits.shape[0]
    E, H, I = W[0].shape
    r = oracle.layer_backward_tokens(logits, x, dout, _as_dicts(W), k, E, H, I, range(T),
                                     exact=exact)
    ws = oracle.wgrad_sample(logits, x, dout, _as_dicts(W), k, E, range(E), np.arange(H),
                             np.arange(I), exact=exact)
    dW1 = np.stack([ws[e][0] for e in range(E)])
    dW3 = np.stack([ws[e][1] for e in range(E)])
    dW2 = np.stack([ws[e][2] for e in range(E)])
    return dict(dx=r["dx64"], dlogits=r["dlogits"], dW1=dW1, dW3=dW3, dW2=dW2, dgate=r["dgate"],
                ids=r["ids"])


@pytest.mark.parametrize("T,E,k,H,I,seed", [
    (40, 5, 2, 32, 24, 1),
    (33, 6, 3, 16, 40, 2),
    (17, 1, 1, 24, 16, 3),    # one expert, top-1: a dense SwiGLU MLP, gate 1, no router gradient
    (20, 4, 4, 16, 8, 4),     # k = E: every expert gets every token
])
def test_backward_exact_matches_torch_autograd(T, E, k, H, I, seed):
    logits, x, dout, W = _case(T, E, k, H, I, seed)
    ref = _torch_dense_grads(logits, x, dout, W, k)
    got = _oracle_grads(logits, x, dout, W, k, exact=True)
    for key in ("dx", "dlogits", "dW1", "dW3", "dW2"):
        r, o = ref[key], got[key]
        scale = max(np.abs(r).max(), 1e-300)
        assert np.abs(o - r).max() <= 1e-11 * scale, key
    if E == 1:
        assert (got["dlogits"] == 0).all()


def test_backward_rounded_stays_within_bf16_error_of_exact():
    logits, x, dout, W = _case(64, 6, 2, 48, 32, 7)
    ex = _oracle_grads(logits, x, dout, W, 2, exact=True)
    rd = _oracle_grads(logits, x, dout, W, 2, exact=False)
    for key in ("dx", "dlogits", "dW1", "dW3", "dW2"):
        err = rms_floor_err(rd[key], ex[key])
        # a handful of bf16 roundings (2^-9 relative each) on the way to every value
        assert err < 3e-2, (key, err)
        assert err > 0, key   # the rounding points are really there


def test_backward_linear_in_dout_exactly():
    """Every step is linear in dout and bf16/fp64 rounding commutes with a
    power-of-two scale: 2*dout and -dout give exactly 2x and -1x."""
    logits, x, dout, W = _case(24, 4, 2, 32, 16, 11)
    base = _oracle_grads(logits, x, dout, W, 2, exact=False)
    d2 = _bf16_bits(_bits_to_f64(dout).to(torch.float32) * 2)
    dn = _bf16_bits(-_bits_to_f64(dout).to(torch.float32))
    two = _oracle_grads(logits, x, d2, W, 2, exact=False)
    neg = _oracle_grads(logits, x, dn, W, 2, exact=False)
    for key in ("dx", "dlogits", "dW1", "dW3", "dW2"):
        assert np.array_equal(two[key], 2 * base[key]), key
        assert np.array_equal(neg[key], -base[key]), key


def test_router_bwd_invariants_and_softmax_jacobian():
    rng = np.random.default_rng(3)
    n, k, E = 50, 4, 12
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(n)]).astype(np.int32)
    sel = rng.standard_normal((n, k))
    g = np.exp(sel - sel.max(1, keepdims=True))
    g /= g.sum(1, keepdims=True)
    dgate = rng.standard_normal((n, k))
    dl = oracle.router_bwd(dgate, g, ids, E)
    # zero off the chosen experts, rows sum to zero (softmax is shift invariant)
    mask = np.zeros((n, E), bool)
    np.put_along_axis(mask, ids.astype(np.int64), True, axis=1)
    assert (dl[~mask] == 0).all()
    assert np.abs(dl.sum(1)).max() < 1e-14
    # the Jacobian of torch.softmax
    S = torch.from_numpy(sel).requires_grad_(True)
    (torch.softmax(S, 1) * torch.from_numpy(dgate)).sum().backward()
    got = np.take_along_axis(dl, ids.astype(np.int64), axis=1)
    assert np.abs(got - S.grad.numpy()).max() < 1e-14


def test_wgrad_two_paths_agree():
    """oracle_wgrad_expert (per column) against dW from the per-row path's
    rounded da, db, hg operands: dW1 = xg^T da, dW3 = xg^T db, dW2 = hg^T dout."""
    logits, x, dout, W = _case(48, 3, 2, 32, 24, 13)
    E, H, I = W[0].shape
    ids, _, g64 = oracle.route_topk(logits, 2)
    for e in range(E):
        t, j = np.nonzero(ids == e)
        r = oracle.ffn_bwd_rows(x[t], dout[t], g64[t, j], np.zeros(len(t), np.int32),
                                {0: W[0][e]}, {0: W[1][e]}, {0: W[2][e]}, H, I)
        xg = _bits_to_f64(x[t]).numpy()
        d = _bits_to_f64(dout[t]).numpy()
        da, db, hg = (_bits_to_f64(r[key]).numpy() for key in ("da", "db", "hg"))
        dW1, dW3, dW2 = oracle.wgrad_expert(x[t], dout[t], g64[t, j], W[0][e], W[1][e], W[2][e],
                                            np.arange(H), np.arange(I))
        assert np.allclose(dW1, xg.T @ da, rtol=1e-12, atol=1e-14)
        assert np.allclose(dW3, xg.T @ db, rtol=1e-12, atol=1e-14)
        assert np.allclose(dW2, hg.T @ d, rtol=1e-12, atol=1e-14)


def test_wgrad_of_unused_expert_is_zero():
    logits, x, dout, W = _case(16, 5, 1, 16, 8, 17)
    logits[:, 2] = float("-inf")   # expert 2 is never chosen
    ws = oracle.wgrad_sample(logits, x, dout, _as_dicts(W), 1, 5, [2], np.arange(16), np.arange(8))
    assert all((m == 0).all() for m in ws[2])
