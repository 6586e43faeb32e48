"""GPU parity of the backward pass: the CUDA path (through the C ABI) against
the CPU oracle's backward, plus properties that hold at any size.

Bit-exact: the reverse combine's gathered rows, the fixed-order reverse
dispatch (on seeded stand-in row gradients), zero router gradients off the
chosen experts, zero weight gradients of experts without routes, run-to-run
determinism and exact linearity in the upstream gradient. Within the layer
tolerance (max |d| / max(|ref|, rms(ref)) against the oracle's fp64 values):
dx, the router gradient, the weight gradients and the per-row intermediates.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_top_route_counting_b200 import inputs
from tests.helpers import OUT_TOL, Y_TOL, bf16_to_f64, bits, expert_weights_host, rms_floor_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
_CACHE = {}


@pytest.fixture(scope="module", autouse=True)
def _free_device_memory():
    yield
    _CACHE.clear()
    torch.cuda.empty_cache()


def _inputs(name):
    if name not in _CACHE:
        _CACHE.clear()
        torch.cuda.empty_cache()
        w = inputs.WORKLOADS[name]
        big = w.H * w.I * w.E > 1e9
        lg, x, dout = inputs.make_logits(w), inputs.make_x(w), inputs.make_dout(w)
        W = inputs.make_weights(w, device=DEV if big else "cpu")
        _CACHE[name] = dict(w=w, lg=lg, x=x, dout=dout, W=[t.to(DEV) for t in W])
    return _CACHE[name]


def _train_step(moe, c, dout=None, ws=None):
    """moe_layer_forward_train + moe_layer_backward; returns device tensors."""
    w, Wd = c["w"], c["W"]
    sh = moe.shape(**w.shape())
    if ws is None:
        ws = torch.empty(moe.train_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    T = w.n_tokens
    out = torch.empty((T, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_layer_forward_train(c["lg"].to(DEV), c["x"].to(DEV), *Wd, out, ws, st, sh)
    dx = torch.empty((T, w.H), dtype=torch.bfloat16, device=DEV)
    dl = torch.empty((T, w.E), dtype=torch.float32, device=DEV)
    dW1 = torch.empty((w.E, w.H, w.I), dtype=torch.float32, device=DEV)
    dW3 = torch.empty_like(dW1)
    dW2 = torch.empty((w.E, w.I, w.H), dtype=torch.float32, device=DEV)
    d = (c["dout"] if dout is None else dout).to(DEV)
    moe.moe_layer_backward(d, *Wd, dx, dl, dW1, dW3, dW2, ws, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return dict(out=out, dx=dx, dlogits=dl, dW1=dW1, dW3=dW3, dW2=dW2, ws=ws)


def _check_dx_dlogits(w, c, r, toks, Wd):
    o_ids, _, _ = oracle.route_topk(c["lg"][toks], w.k)
    Wh = expert_weights_host(*Wd, np.unique(o_ids))
    ref = oracle.layer_backward_tokens(c["lg"], bits(c["x"]), bits(c["dout"]), Wh, w.k, w.E, w.H,
                                       w.I, toks)
    ti = torch.tensor(toks, device=DEV)
    dx = bf16_to_f64(bits(r["dx"][ti]))
    err_dx = rms_floor_err(dx, ref["dx64"])
    dl = r["dlogits"][ti].double().cpu().numpy()
    support = ref["dlogits"] != 0
    ids = ref["ids"][toks]
    on = np.zeros_like(support)
    np.put_along_axis(on, ids.astype(np.int64), True, axis=1)
    assert (dl[~on] == 0).all(), "router gradient off the chosen experts must be exactly 0"
    sel = np.take_along_axis(dl, ids.astype(np.int64), axis=1)
    ref_sel = np.take_along_axis(ref["dlogits"], ids.astype(np.int64), axis=1)
    err_dl = rms_floor_err(sel, ref_sel)
    print(f"{w.name}: dx err {err_dx:.3e}, dlogits err {err_dl:.3e}")
    assert err_dx < OUT_TOL
    assert err_dl < OUT_TOL


def _check_wgrad(w, c, r, experts, hs, is_):
    Wh = expert_weights_host(*c["W"], experts)
    ref = oracle.wgrad_sample(c["lg"], bits(c["x"]), bits(c["dout"]), Wh, w.k, w.E, experts, hs, is_)
    hi, ii = torch.tensor(hs, device=DEV), torch.tensor(is_, device=DEV)
    for e in experts:
        g1 = r["dW1"][e][hi][:, ii].double().cpu().numpy()
        g3 = r["dW3"][e][hi][:, ii].double().cpu().numpy()
        g2 = r["dW2"][e][ii][:, hi].double().cpu().numpy()
        o1, o3, o2 = ref[e]
        if not (o1.any() or o3.any() or o2.any()):
            assert not (g1.any() or g3.any() or g2.any()), f"expert {e} without routes: zero dW"
            continue
        errs = [rms_floor_err(g, o) for g, o in ((g1, o1), (g3, o3), (g2, o2))]
        print(f"{w.name}: expert {e} dW1/dW3/dW2 err " + " ".join(f"{x:.2e}" for x in errs))
        assert max(errs) < OUT_TOL


# ---------------------------------------------------------------- stages
def test_tiny_backward_stages_vs_oracle(cuda_lib):
    moe = cuda_lib
    c = _inputs("tiny_bwd")
    w, (W1, W3, W2) = c["w"], c["W"]
    sh = moe.shape(**w.shape())
    T, k, rm = w.n_tokens, w.k, moe.rows_max(sh)
    lg, x, dout = c["lg"].to(DEV), c["x"].to(DEV), c["dout"].to(DEV)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gates = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg, ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh)
    st = b["dev_status"]
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"], st, sh)
    xg = torch.empty((rm, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch(x, b["phi"], b["offsets"], xg, st, sh)
    h = torch.empty((rm, w.I), dtype=torch.bfloat16, device=DEV)
    ab = torch.empty((rm, 2 * w.I), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((rm, w.H), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn_train(xg, W1, W3, W2, b["offsets"], b["counts"], h, ab, y, st, sh)
    h_inf, y_inf = torch.empty_like(h), torch.empty_like(y)
    moe.moe_expert_ffn(xg, W1, W3, W2, b["offsets"], b["counts"], h_inf, y_inf, st, sh)
    dys = torch.empty((rm, w.H), dtype=torch.bfloat16, device=DEV)
    gate_row = torch.empty(rm, dtype=torch.float32, device=DEV)
    moe.moe_reverse_combine(dout, b["phi"], b["offsets"], b["route_row"], gates, dys, gate_row, st, sh)
    dab = torch.empty((rm, 2 * w.I), dtype=torch.bfloat16, device=DEV)
    hg = torch.empty((rm, w.I), dtype=torch.bfloat16, device=DEV)
    part = torch.empty((rm, w.I // 128), dtype=torch.float32, device=DEV)
    dxg = torch.empty((rm, w.H), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn_dgrad(dys, gate_row, ab, h, W1, W3, W2, b["offsets"], b["counts"], dab, hg,
                             part, dxg, st, sh)
    dx = torch.empty((T, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_reverse_dispatch(dxg, b["route_row"], dx, st, sh)
    dl = torch.empty((T, w.E), dtype=torch.float32, device=DEV)
    moe.moe_router_backward(part, b["route_row"], ids, gates, dl, st, sh)
    dW1 = torch.empty((w.E, w.H, w.I), dtype=torch.float32, device=DEV)
    dW3, dW2 = torch.empty_like(dW1), torch.empty((w.E, w.I, w.H), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn_wgrad(xg, dys, dab, hg, b["offsets"], b["counts"], dW1, dW3, dW2, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # the training GEMM1 writes the same h and y as the inference one
    assert torch.equal(h, h_inf) and torch.equal(y, y_inf)

    o_ids, o_g32, o_g64 = oracle.route_topk(c["lg"], k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, k), w.P, w.N, k, w.E, 256)
    assert (b["phi"][: int(s["offsets"][-1])].cpu().numpy() == s["phi"]).all()
    rows = int(s["offsets"][-1])
    # reverse combine: the dispatch gather of dout through the same Phi (bit-exact),
    # and each row's gate (the GPU's gates are within 2 ulp of the oracle's fp32 gates)
    o_dys = oracle.dispatch_rows(bits(c["dout"]), w.N, s["phi"], np.arange(rows))
    assert (bits(dys[:rows]) == o_dys).all()
    o_gate_row = np.zeros(rows, np.float32)
    rr = s["route_row"].reshape(-1, k)
    o_gate_row[rr.reshape(-1)] = o_g32.reshape(-1)
    assert np.allclose(gate_row[:rows].cpu().numpy(), o_gate_row, rtol=3e-7, atol=0)
    assert (gate_row[:rows].cpu().numpy()[s["phi"][:, 0] < 0] == 0).all()
    # per-row intermediates against the oracle's per-row backward
    real = np.nonzero(s["phi"][:, 0] >= 0)[0]
    ex = oracle.expert_of_rows(s["offsets"], real)
    tok = s["phi"][real, 0] * w.N + s["phi"][real, 1]
    g_row = np.zeros(len(real))
    for i, row in enumerate(real):
        j = int(np.nonzero(rr[tok[i]] == row)[0][0])
        g_row[i] = o_g64[tok[i], j]
    Wh = expert_weights_host(W1, W3, W2, range(w.E))
    o = oracle.ffn_bwd_rows(bits(c["x"])[tok], bits(c["dout"])[tok], g_row, ex, *Wh, H=w.H, I=w.I)
    ri = torch.from_numpy(real).to(DEV)
    for key, gpu in (("hg", hg), ("da", dab[:, : w.I]), ("db", dab[:, w.I:])):
        got = bits(gpu[ri])
        match = (got == o[key]).mean()
        err = rms_floor_err(bf16_to_f64(got), bf16_to_f64(o[key]))
        print(f"{key}: bf16 match {match:.4f}, err {err:.2e}")
        assert match > 0.99 and err < Y_TOL
    assert rms_floor_err(dxg[ri].double().cpu().numpy(), o["dxg"]) < Y_TOL
    dgate_rows = part[ri].double().sum(1).cpu().numpy()
    assert rms_floor_err(dgate_rows, o["dgate"]) < Y_TOL
    # the whole backward's outputs
    r = dict(dx=dx, dlogits=dl, dW1=dW1, dW3=dW3, dW2=dW2)
    _check_dx_dlogits(w, c, r, list(range(T)), c["W"])
    _check_wgrad(w, c, r, list(range(w.E)), list(range(w.H)), list(range(w.I)))


def test_reverse_dispatch_fixed_order_bit_exact(cuda_lib):
    """dx = bf16(sum_j dxg[route_row[t,j]]) in ascending j: bit-exact against the
    oracle's fixed-order fp32 sum (unit weights), on seeded stand-in row gradients."""
    moe = cuda_lib
    w = inputs.WORKLOADS["mid"]
    sh = moe.shape(**w.shape())
    o_ids, _, _ = oracle.route_topk(inputs.make_logits(w), w.k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    rows = int(s["offsets"][-1])
    dxg = inputs.make_expert_outputs(w, rows)
    rr = np.ascontiguousarray(s["route_row"].reshape(-1, w.k))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    dx = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_reverse_dispatch(dxg.to(DEV), torch.from_numpy(rr).to(DEV), dx, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    toks = inputs.sample_tokens(w.n_tokens, 400, seed=3)
    used = np.unique(rr[toks])
    exp = oracle.combine_f32(dxg.numpy()[used], np.searchsorted(used, rr[toks]),
                             np.ones((len(toks), w.k), np.float32), w.k)
    assert (bits(dx)[toks] == exp).all()


def test_reverse_combine_flags_inconsistent_schedule(cuda_lib):
    """A Phi row that route_row does not point back to raises MOE_DEV_BAD_SCHEDULE
    and gets gate 0 (all indices stay in range: nothing is read out of bounds)."""
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny_bwd"]
    sh = moe.shape(**w.shape())
    o_ids, o_g32, _ = oracle.route_topk(inputs.make_logits(w), w.k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    rm = moe.rows_max(sh)
    phi = np.full((rm, 2), -1, np.int32)
    phi[: len(s["phi"])] = s["phi"]
    real = np.nonzero(phi[:, 0] >= 0)[0]
    a, b2 = real[0], real[-1]
    if (phi[a] == phi[b2]).all():
        b2 = real[-2]
    phi[[a, b2]] = phi[[b2, a]]  # swap two rows' sources
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    dys = torch.empty((rm, w.H), dtype=torch.bfloat16, device=DEV)
    gr = torch.empty(rm, dtype=torch.float32, device=DEV)
    moe.moe_reverse_combine(inputs.make_dout(w).to(DEV), torch.from_numpy(phi).to(DEV),
                            torch.from_numpy(s["offsets"]).to(DEV),
                            torch.from_numpy(np.ascontiguousarray(s["route_row"])).to(DEV),
                            torch.from_numpy(o_g32.astype(np.float32)).to(DEV), dys, gr, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.DEV_BAD_SCHEDULE
    assert gr[int(a)].item() == 0.0 and gr[int(b2)].item() == 0.0


# ---------------------------------------------------------------- whole backward
@pytest.mark.parametrize("name,n_tok,experts_n", [("tiny_bwd", 512, 8), ("mid", 64, 3),
                                                  ("kimi", 6, 2), ("zipf", 6, 2)])
def test_layer_backward_vs_oracle(cuda_lib, name, n_tok, experts_n):
    moe = cuda_lib
    c = _inputs(name)
    w = c["w"]
    r = _train_step(moe, c)
    toks = inputs.sample_tokens(w.n_tokens, n_tok, seed=w.wid + 11)
    _check_dx_dlogits(w, c, r, toks, c["W"])
    rng = np.random.default_rng(w.wid)
    ids_all, _, _ = oracle.route_topk(c["lg"], w.k)
    counts = np.bincount(ids_all.reshape(-1), minlength=w.E)
    experts = sorted(set(rng.choice(w.E, experts_n, replace=False).tolist()))
    if name == "zipf":  # the hottest expert and one that never gets a route
        experts = sorted(set(experts + [int(counts.argmax()), inputs.empty_experts(w)[0]]))
    if name == "tiny_bwd":
        hs, is_ = list(range(w.H)), list(range(w.I))
    else:
        hs = sorted(set([0, w.H - 1] + rng.choice(w.H, 4, replace=False).tolist()))
        is_ = sorted(set([0, w.I - 1] + rng.choice(w.I, 3, replace=False).tolist()))
    _check_wgrad(w, c, r, experts, hs, is_)
    empty = np.nonzero(counts == 0)[0]
    if len(empty):
        e = int(empty[0])
        assert not r["dW1"][e].any() and not r["dW3"][e].any() and not r["dW2"][e].any()


def _fingerprint(t: torch.Tensor):
    """Bit-level fingerprint of a device tensor, computed on the device in
    chunks (the Kimi-shape gradients are too large to hold twice): the int64
    sums of its 32-bit words (bf16 pairs) and of the words times fixed odd
    weights. Any single changed word changes the weighted sum."""
    v = t.contiguous().view(-1).view(torch.int32 if t.element_size() == 4 else torch.int16)
    n, step = v.numel(), 1 << 26
    w = (torch.arange(step, device=t.device, dtype=torch.int64) * 2654435761 * 2 + 1)
    s0 = torch.zeros((), dtype=torch.int64, device=t.device)
    s1 = torch.zeros((), dtype=torch.int64, device=t.device)
    for i in range(0, n, step):
        c = v[i:i + step].to(torch.int64)
        s0 += c.sum()
        s1 += (c * w[: c.numel()]).sum() * (i // step + 1)
    return int(s0.item()), int(s1.item())


@pytest.mark.parametrize("name", ["tiny_bwd", "mid", "kimi"])
def test_layer_backward_bitwise_deterministic_and_linear(cuda_lib, name):
    """Two runs give identical bits; 2*dout gives exactly twice every gradient
    (every step is linear in dout and rounding commutes with a power-of-two scale)."""
    moe = cuda_lib
    c = _inputs(name)
    keys = ("dx", "dlogits", "dW1", "dW3", "dW2")
    r = _train_step(moe, c)
    ws = r["ws"]
    f0 = {key: _fingerprint(r[key]) for key in keys}
    for key in keys:  # exact: a power-of-two scale of bf16 / fp32 values
        r[key].mul_(2)
    f2 = {key: _fingerprint(r[key]) for key in keys}
    del r
    r = _train_step(moe, c, ws=ws)
    for key in keys:
        assert _fingerprint(r[key]) == f0[key], f"{key} changed between identical runs"
    del r
    r = _train_step(moe, c, dout=c["dout"].float().mul(2).to(torch.bfloat16), ws=ws)
    for key in keys:
        assert _fingerprint(r[key]) == f2[key], f"{key} is not exactly linear in dout"


def test_forward_train_output_equals_forward(cuda_lib):
    moe = cuda_lib
    c = _inputs("mid")
    w = c["w"]
    r = _train_step(moe, c)
    sh = moe.shape(**w.shape())
    ws = torch.empty(moe.layer_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.empty_like(r["out"])
    moe.moe_layer_forward(c["lg"].to(DEV), c["x"].to(DEV), *c["W"], out, ws, st, sh)
    torch.cuda.synchronize()
    assert torch.equal(out, r["out"])


@pytest.mark.parametrize("P,N,E,k,H,I", [
    (3, 131, 5, 5, 512, 256),     # k = E: every expert gets every token
    (2, 700, 1, 1, 256, 512),     # one expert, gate 1: router gradient 0
    (64, 3, 1024, 16, 256, 256),  # most experts empty: their dW must be 0
])
def test_layer_backward_edge_shapes(cuda_lib, P, N, E, k, H, I):
    moe = cuda_lib
    w = inputs.Workload(f"edge{P}x{N}x{E}", 7, P=P, N=N, E=E, k=k, H=H, I=I)
    Wc = inputs.make_weights(w)
    c = dict(w=w, lg=inputs.make_logits(w), x=inputs.make_x(w), dout=inputs.make_dout(w),
             W=[t.to(DEV) for t in Wc])
    r = _train_step(moe, c)
    toks = inputs.sample_tokens(w.n_tokens, 48, seed=5)
    _check_dx_dlogits(w, c, r, toks, c["W"])
    if E == 1:
        assert not r["dlogits"].any()
    ids_all, _, _ = oracle.route_topk(c["lg"], k)
    counts = np.bincount(ids_all.reshape(-1), minlength=E)
    used = np.nonzero(counts)[0]
    experts = sorted(set([int(used[0]), int(used[-1])] + ([int(np.nonzero(counts == 0)[0][0])]
                                                          if (counts == 0).any() else [])))
    _check_wgrad(w, c, r, experts, [0, 7, H - 1], [0, 5, I - 1])
    assert int((r["dW1"].abs().sum((1, 2)) > 0).sum().item()) == len(used)


def test_layer_backward_pad512_skipped_tiles(cuda_lib):
    """Segments padded to 512 rows: tiles holding only padding rows are skipped
    by every GEMM (their rows stay unwritten), and the weight gradients run
    over each expert's real rows only: still within the bound of the oracle."""
    moe = cuda_lib
    w = inputs.Workload("pad512", 9, P=2, N=300, E=6, k=2, H=256, I=256, pad=512)
    c = dict(w=w, lg=inputs.make_logits(w), x=inputs.make_x(w), dout=inputs.make_dout(w),
             W=[t.to(DEV) for t in inputs.make_weights(w)])
    sh = moe.shape(**w.shape())
    ws = torch.full((moe.train_workspace_bytes(sh),), 0xFF, dtype=torch.uint8, device=DEV)  # NaN-filled
    r = _train_step(moe, c, ws=ws)
    ids_all, _, _ = oracle.route_topk(c["lg"], w.k)
    s = oracle.schedule(ids_all.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 512)
    assert (np.diff(s["offsets"]) - np.bincount(ids_all.reshape(-1), minlength=w.E) >= 256).any(), \
        "the case has at least one padding-only tile"
    _check_dx_dlogits(w, c, r, list(range(w.n_tokens)), c["W"])
    _check_wgrad(w, c, r, list(range(w.E)), list(range(w.H)), list(range(w.I)))


def test_backward_stages_without_counts_equal_with_counts(cuda_lib):
    """counts = NULL: the GEMMs take whole segments (padding rows included) and
    give bit-identical activation and weight gradients (padding rows add exact
    zeros to every sum)."""
    moe = cuda_lib
    c = _inputs("tiny_bwd")
    w, (W1, W3, W2) = c["w"], c["W"]
    sh = moe.shape(**w.shape())
    T, k, rm = w.n_tokens, w.k, moe.rows_max(sh)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gates = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(c["lg"].to(DEV), ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh)
    st = b["dev_status"]
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"], st, sh)
    xg = torch.empty((rm, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch(c["x"].to(DEV), b["phi"], b["offsets"], xg, st, sh)
    h = torch.empty((rm, w.I), dtype=torch.bfloat16, device=DEV)
    ab = torch.empty((rm, 2 * w.I), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((rm, w.H), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn_train(xg, W1, W3, W2, b["offsets"], None, h, ab, y, st, sh)
    dys = torch.empty((rm, w.H), dtype=torch.bfloat16, device=DEV)
    gate_row = torch.empty(rm, dtype=torch.float32, device=DEV)
    moe.moe_reverse_combine(c["dout"].to(DEV), b["phi"], b["offsets"], b["route_row"], gates, dys,
                            gate_row, st, sh)
    outs = []
    for counts in (b["counts"], None):
        dab = torch.empty((rm, 2 * w.I), dtype=torch.bfloat16, device=DEV)
        hg = torch.empty((rm, w.I), dtype=torch.bfloat16, device=DEV)
        part = torch.empty((rm, w.I // 128), dtype=torch.float32, device=DEV)
        dxg = torch.empty((rm, w.H), dtype=torch.float32, device=DEV)
        moe.moe_expert_ffn_dgrad(dys, gate_row, ab, h, W1, W3, W2, b["offsets"], counts, dab, hg,
                                 part, dxg, st, sh)
        dW1 = torch.empty((w.E, w.H, w.I), dtype=torch.float32, device=DEV)
        dW3, dW2 = torch.empty_like(dW1), torch.empty((w.E, w.I, w.H), dtype=torch.float32,
                                                      device=DEV)
        moe.moe_expert_ffn_wgrad(xg, dys, dab, hg, b["offsets"], counts, dW1, dW3, dW2, st, sh)
        outs.append((dab, hg, part, dxg, dW1, dW3, dW2))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = int(b["offsets"][-1].item())
    real = torch.from_numpy(np.nonzero(b["phi"][:rows, 0].cpu().numpy() >= 0)[0]).to(DEV)
    for a, b_ in zip(outs[0][:4], outs[1][:4]):
        assert torch.equal(a[real], b_[real])
    for a, b_ in zip(outs[0][4:], outs[1][4:]):
        assert torch.equal(a, b_)


def test_layer_backward_no_tokens(cuda_lib):
    moe = cuda_lib
    w = inputs.Workload("empty", 8, P=2, N=0, E=4, k=2, H=256, I=256)
    sh = moe.shape(**w.shape())
    ws = torch.empty(moe.train_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    W = [t.to(DEV) for t in inputs.make_weights(w)]
    z = torch.empty((0, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_layer_forward_train(torch.empty((0, w.E), device=DEV), z, *W, z, ws, st, sh)
    dW = [torch.full((w.E, w.H, w.I), 7.0, device=DEV), torch.full((w.E, w.H, w.I), 7.0, device=DEV),
          torch.full((w.E, w.I, w.H), 7.0, device=DEV)]
    moe.moe_layer_backward(z, *W, z, torch.empty((0, w.E), device=DEV), *dW, ws, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert all(not t.any() for t in dW)
