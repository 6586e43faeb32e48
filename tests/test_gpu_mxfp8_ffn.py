"""GPU parity of the MXFP8 routed-expert path (through the C ABI) against the
oracle: the weight quantisation and the tiled-scale dispatch bit-exact; the
block-scaled expert FFN (h codes and scales, fp32 y) and the MXFP8 layer
against the oracle's fp64 arithmetic on the values the codes stand for.

Every GPU input of the FFN test is the oracle's own quantisation of the seeded
bf16 inputs (codes transposed and scales laid out as the header defines); the
expected values come from the oracle alone.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_top_route_counting_b200 import inputs
from tests.helpers import (OUT_TOL, Y_TOL, bf16_to_f64, bits, expert_weights_host,
                           mx_tiled_offsets, rms_floor_err, sha, to_tiled)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _crafted_weights(E=3, K=256, N=256, seed=8):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn((E, K, N), generator=g) * 0.02
    W[0, :32, :] = 0.0                                   # all-zero blocks along K
    W[1, 32:64, 5] = 3.0e38 * torch.sign(W[1, 32:64, 5])  # huge block
    W[2, 64:96, 7] = 2.0 ** -133 * torch.arange(1, 33).float()  # bf16 subnormals
    W[2, 96:128, 9] = 1.99 * 2.0 ** 10                    # saturating block
    return W.to(torch.bfloat16)


def _oracle_weight_operand(W_host: torch.Tensor):
    """Oracle quantisation of W [E, K, N] along K: transposed codes [E, N, K]
    and the tiled scale table of the [E*N, K] code matrix."""
    E, K, N = W_host.shape
    qs, ss = [], []
    for e in range(E):
        q, s = oracle.mx_quantize(bf16_to_f64(bits(W_host[e])).T)
        qs.append(q)
        ss.append(s)
    return np.stack(qs), to_tiled(np.concatenate(ss))


def test_quantize_weights_bit_exact(cuda_lib):
    moe = cuda_lib
    W = _crafted_weights()
    E, K, N = W.shape
    q = torch.full((E, N, K), 0x55, dtype=torch.uint8, device=DEV)
    s = torch.full((E * N * K // 32,), 0x55, dtype=torch.uint8, device=DEV)
    moe.moe_mx_quantize_weights(W.to(DEV), q, s)
    torch.cuda.synchronize()
    oq, os_ = _oracle_weight_operand(W)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(s.cpu().numpy(), os_)


def _route_schedule(moe, w, lg):
    sh = moe.shape(**w.shape())
    o_ids, _, _ = oracle.route_topk(lg, w.k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, w.pad)
    return sh, o_ids, s


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_dispatch_tiled_bit_exact(cuda_lib, name):
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    sh, _, s = _route_schedule(moe, w, lg)
    rm = moe.rows_max(sh)
    phi = torch.from_numpy(np.ascontiguousarray(s["phi"])).to(DEV)
    phi_full = torch.full((rm, 2), -1, dtype=torch.int32, device=DEV)
    phi_full[: phi.shape[0]] = phi
    offsets = torch.from_numpy(s["offsets"]).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    xq = torch.full((rm, w.H), 0x55, dtype=torch.uint8, device=DEV)
    xs = torch.full((rm * w.H // 32,), 0x55, dtype=torch.uint8, device=DEV)
    moe.moe_dispatch_mxfp8_tiled(x.to(DEV), phi_full, offsets, xq, xs, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = int(s["offsets"][-1])
    o_xg = oracle.dispatch_rows(bits(x), w.N, s["phi"], np.arange(rows))
    oq, os_ = oracle.mx_quantize(bf16_to_f64(o_xg))
    assert np.array_equal(xq[:rows].cpu().numpy(), oq)
    idx = mx_tiled_offsets(rm, w.H)[:rows]
    assert np.array_equal(xs.cpu().numpy()[idx], os_)


def _ffn_case(moe, w, sample=None):
    """GPU FFN on the oracle's quantised operands; returns what to compare."""
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = inputs.make_weights(w)
    sh, _, s = _route_schedule(moe, w, lg)
    rm = moe.rows_max(sh)
    rows = int(s["offsets"][-1])
    xg = oracle.dispatch_rows(bits(x), w.N, s["phi"], np.arange(rows))
    xq_o, xs_o = oracle.mx_quantize(bf16_to_f64(xg))
    xq = torch.zeros((rm, w.H), dtype=torch.uint8)
    xq[:rows] = torch.from_numpy(xq_o)
    xs_rows = np.zeros((rm, w.H // 32), np.uint8)
    xs_rows[:rows] = xs_o
    ops = [_oracle_weight_operand(Wt) for Wt in (W1, W3, W2)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    hq = torch.full((rm, w.I), 0x55, dtype=torch.uint8, device=DEV)
    hs = torch.full((rm * w.I // 32,), 0x55, dtype=torch.uint8, device=DEV)
    y = torch.full((rm, w.H), float("nan"), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_expert_ffn_mxfp8(xq.to(DEV), dev(to_tiled(xs_rows)), dev(ops[0][0]), dev(ops[0][1]),
                             dev(ops[1][0]), dev(ops[1][1]), dev(ops[2][0]), dev(ops[2][1]),
                             dev(s["offsets"]), dev(s["counts"]), hq, hs, y, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    real = np.nonzero(s["phi"][:, 0] >= 0)[0]
    if sample is not None:
        real = np.unique(np.random.default_rng(w.wid).choice(real, sample))
    experts = oracle.expert_of_rows(s["offsets"], real)
    Wh = [{e: bits(Wt[e]) for e in np.unique(experts)} for Wt in (W1, W3, W2)]
    o_hq, o_hs, o_y = oracle.ffn_rows_mxfp8(xg[real], experts, *Wh, w.H, w.I)
    g_hs = hs.cpu().numpy()[mx_tiled_offsets(rm, w.I)[real]]
    return dict(hq=hq.cpu().numpy()[real], hs=g_hs, y=y.cpu().numpy()[real].astype(np.float64),
                o_hq=o_hq, o_hs=o_hs, o_y=o_y)


@pytest.mark.parametrize("name,sample", [("tiny", None), ("tiny_bwd", None), ("mid", 300)])
def test_ffn_mxfp8_vs_oracle(cuda_lib, name, sample):
    r = _ffn_case(cuda_lib, inputs.WORKLOADS[name], sample)
    # both sides quantise h from fp32, but the GPU's a and b are fp32 sums in
    # another order: codes may differ where h lands across a rounding point
    assert (r["hq"] == r["o_hq"]).mean() >= 0.99
    assert (r["hs"] == r["o_hs"]).mean() >= 0.99
    err = rms_floor_err(r["y"], r["o_y"])
    print(f"{name}: y rms-floor err {err:.3e}, h codes equal {(r['hq'] == r['o_hq']).mean():.5f}")
    assert err < Y_TOL


def _mx_weights_gpu(moe, W):
    out = []
    for Wt in W:
        E, K, N = Wt.shape
        q = torch.empty((E, N, K), dtype=torch.uint8, device=DEV)
        s = torch.empty((E * N * K // 32,), dtype=torch.uint8, device=DEV)
        moe.moe_mx_quantize_weights(Wt.to(DEV), q, s)
        out += [q, s]
    return out


def _layer_mx(moe, w, lg_d, x_d, Wq):
    sh = moe.shape(**w.shape())
    ws = torch.empty(moe.layer_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_layer_forward_mxfp8(lg_d, x_d, *Wq, out, ws, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out


@pytest.mark.parametrize("name,n_tok", [("tiny", 256), ("mid", 48), ("kimi", 4)])
def test_layer_mxfp8_vs_oracle(cuda_lib, name, n_tok):
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    big = w.H * w.I * w.E > 1e9
    W = inputs.make_weights(w, device=DEV if big else "cpu")
    Wq = _mx_weights_gpu(moe, W)
    out = _layer_mx(moe, w, lg.to(DEV), x.to(DEV), Wq)
    toks = inputs.sample_tokens(w.n_tokens, n_tok, seed=w.wid)
    o_ids, _, _ = oracle.route_topk(lg[toks], w.k)
    Wh = expert_weights_host(*W, np.unique(o_ids))
    res = oracle.layer_tokens_mxfp8(lg, bits(x), Wh, w.k, w.H, w.I, toks)
    got = bf16_to_f64(bits(out[torch.tensor(toks, device=DEV)]))
    err = rms_floor_err(got, res["out64"])
    print(f"{name}: MXFP8 layer rms-floor err {err:.3e}")
    assert err < OUT_TOL


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_layer_mxfp8_bitwise_deterministic(cuda_lib, name):
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    lg, x = inputs.make_logits(w).to(DEV), inputs.make_x(w).to(DEV)
    Wq = _mx_weights_gpu(moe, inputs.make_weights(w))
    a = _layer_mx(moe, w, lg, x, Wq)
    b = _layer_mx(moe, w, lg, x, Wq)
    assert sha(a) == sha(b)


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_layer_mxfp8_equals_its_stage_entries(cuda_lib, name):
    """The MXFP8 layer, whose GEMM1 quantises and lands the dispatch itself,
    gives bit for bit the output of the separate entry points: moe_route_topk,
    moe_schedule, moe_dispatch_mxfp8_tiled, moe_expert_ffn_mxfp8, moe_combine."""
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    lg, x = inputs.make_logits(w).to(DEV), inputs.make_x(w).to(DEV)
    Wq = _mx_weights_gpu(moe, inputs.make_weights(w))
    out = _layer_mx(moe, w, lg, x, Wq)
    sh = moe.shape(**w.shape())
    rm = moe.rows_max(sh)
    ids = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=DEV)
    gates = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg, ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh)
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    xq = torch.empty((rm, w.H), dtype=torch.uint8, device=DEV)
    xs = torch.empty((rm * w.H // 32,), dtype=torch.uint8, device=DEV)
    moe.moe_dispatch_mxfp8_tiled(x, b["phi"], b["offsets"], xq, xs, b["dev_status"], sh)
    hq = torch.empty((rm, w.I), dtype=torch.uint8, device=DEV)
    hs = torch.empty((rm * w.I // 32,), dtype=torch.uint8, device=DEV)
    y = torch.empty((rm, w.H), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn_mxfp8(xq, xs, *Wq, b["offsets"], b["counts"], hq, hs, y, b["dev_status"], sh)
    ref = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(y, b["route_row"], gates, ref, b["dev_status"], sh)
    torch.cuda.synchronize()
    assert int(b["dev_status"].item()) == 0
    assert torch.equal(out, ref)


def test_layer_mxfp8_no_tokens(cuda_lib):
    moe = cuda_lib
    w = inputs.Workload("mx_empty", 13, P=2, N=0, E=8, k=2, H=256, I=256)
    Wq = _mx_weights_gpu(moe, inputs.make_weights(w))
    lg = torch.empty((0, w.E), dtype=torch.float32, device=DEV)
    x = torch.empty((0, w.H), dtype=torch.bfloat16, device=DEV)
    out = _layer_mx(moe, w, lg, x, Wq)
    assert out.numel() == 0


def _shared_weights(w, seed=91):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(shape, generator=g) * 0.02).to(torch.bfloat16)
            for shape in ((w.H, w.I), (w.H, w.I), (w.I, w.H))]


@pytest.mark.parametrize("name,n_tok", [("tiny", 256), ("mid", 48),
                                        ("ragged", 120)])   # P*N % 256 != 0: padded copy of x
def test_layer_mxfp8_shared_expert_vs_oracle(cuda_lib, name, n_tok):
    moe = cuda_lib
    w = (inputs.Workload("mx_ragged", 15, P=2, N=300, E=8, k=2, H=256, I=256)
         if name == "ragged" else inputs.WORKLOADS[name])
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W = inputs.make_weights(w)
    Ws = _shared_weights(w)
    Wq = _mx_weights_gpu(moe, W)
    sh = moe.shape(**w.shape())
    ws = torch.empty(moe.layer_mxfp8_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_layer_forward_mxfp8(lg.to(DEV), x.to(DEV), *Wq, out, ws, st, sh,
                                shared=tuple(t.to(DEV) for t in Ws))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    toks = inputs.sample_tokens(w.n_tokens, n_tok, seed=w.wid)
    o_ids, _, _ = oracle.route_topk(lg[toks], w.k)
    Wh = expert_weights_host(*W, np.unique(o_ids))
    res = oracle.layer_tokens_mxfp8(lg, bits(x), Wh, w.k, w.H, w.I, toks,
                                    shared=tuple(bits(t) for t in Ws))
    got = bf16_to_f64(bits(out[torch.tensor(toks, device=DEV)]))
    err = rms_floor_err(got, res["out64"])
    print(f"{name}: MXFP8 layer + shared expert rms-floor err {err:.3e}")
    assert err < OUT_TOL
