"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact on ids, Phi, offsets, counts, route_row, the gathered buffer and the
fixed-order combine; within the stated tolerance on gates, expert outputs and
the layer output; bitwise run-to-run and across transfer-slice sizes.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from combine_top_route_counting_b200 import inputs
from tests.helpers import (OUT_TOL, Y_TOL, bf16_to_f64, bits, expert_weights_host, literal_rms_err,
                           rms_floor_err, sha)

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(__file__), "golden")
DEV = "cuda"


def _sched_gpu(moe, ids_dev, P, N, k, E, pad=256):
    sh = moe.shape(P, N, E, k, pad=pad)
    b = moe.alloc_schedule_outputs(sh)
    b["phi"].fill_(-7)
    moe.moe_schedule(ids_dev, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    torch.cuda.synchronize()
    return {k_: v.cpu().numpy() for k_, v in b.items()}


def _assert_sched_equal(g, o):
    rows = int(o["offsets"][-1])
    assert (g["offsets"] == o["offsets"]).all()
    assert (g["counts"] == o["counts"]).all()
    assert (g["route_row"] == o["route_row"]).all()
    assert (g["phi"][:rows] == o["phi"]).all()
    assert int(g["dev_status"][0]) == 0


# ---------------------------------------------------------------- schedule
def test_schedule_handworked(cuda_lib):
    moe = cuda_lib
    for c in json.load(open(os.path.join(GOLD, "schedule_handworked.json")))["cases"]:
        ids = torch.tensor(c["ids"], dtype=torch.int32, device=DEV)
        g = _sched_gpu(moe, ids, c["P"], c["N"], c["k"], c["E"], c["pad"])
        rows = c["offsets"][-1]
        assert g["phi"][:rows].tolist() == c["phi"]
        assert g["offsets"].tolist() == c["offsets"]
        assert g["counts"].tolist() == c["counts"]
        assert g["route_row"].tolist() == c["route_row"]


def test_schedule_sweep_945(cuda_lib):
    moe = cuda_lib
    n = 0
    for P, N, E, k, ids in inputs.sweep_cases():
        g = _sched_gpu(moe, ids.to(DEV), P, N, k, E)
        o = oracle.schedule(ids.numpy(), P, N, k, E, 256)
        _assert_sched_equal(g, o)
        n += 1
    assert n == 945


def test_schedule_full_scheduler_workload(cuda_lib):
    moe = cuda_lib
    w = inputs.WORKLOADS["sched"]
    ids = inputs.make_sched_ids(w)
    g = _sched_gpu(moe, ids.to(DEV), w.P, w.N, w.k, w.E)
    o = oracle.schedule(ids.numpy(), w.P, w.N, w.k, w.E, 256)
    _assert_sched_equal(g, o)
    assert o["reads"] == 917504


@pytest.mark.parametrize("case", ["empty", "one_expert", "k_eq_E", "hot", "many_blocks", "P64"])
def test_schedule_edge_cases(cuda_lib, case):
    moe = cuda_lib
    if case == "empty":
        P, N, E, k = 3, 0, 5, 2
        ids = torch.zeros((P, N, k), dtype=torch.int32)
    elif case == "one_expert":
        P, N, E, k = 4, 1000, 1, 1
        ids = torch.zeros((P, N, k), dtype=torch.int32)
    elif case == "k_eq_E":
        P, N, E, k = 2, 300, 6, 6
        ids = inputs.make_ids_uniform(P, N, E, k, seed=11)
    elif case == "hot":  # every route of peer 0 to expert 3, others uniform
        P, N, E, k = 5, 900, 40, 4
        ids = inputs.make_ids_uniform(P, N, E, k, seed=12)
        ids[0, :, 0] = 3
        ids[0, :, 1:] = torch.where(ids[0, :, 1:] == 3, torch.full_like(ids[0, :, 1:], 7),
                                    ids[0, :, 1:])
    elif case == "many_blocks":  # ragged last block, several blocks per peer
        P, N, E, k = 3, 5000, 17, 3
        ids = inputs.make_ids_uniform(P, N, E, k, seed=13)
    else:
        P, N, E, k = 64, 200, 256, 16
        ids = inputs.make_ids_uniform(P, N, E, k, seed=14)
    g = _sched_gpu(moe, ids.to(DEV), P, N, k, E)
    o = oracle.schedule(ids.numpy(), P, N, k, E, 256)
    _assert_sched_equal(g, o)


def test_schedule_bad_expert_id_flags_and_drops(cuda_lib):
    moe = cuda_lib
    P, N, E, k = 2, 50, 8, 2
    ids = inputs.make_ids_uniform(P, N, E, k, seed=21)
    bad = ids.clone()
    bad[1, 7, 1] = 99
    g = _sched_gpu(moe, bad.to(DEV), P, N, k, E)
    assert int(g["dev_status"][0]) & moe.DEV_BAD_EXPERT_ID
    assert g["route_row"][1, 7, 1] == -1
    assert moe.status_from_device_flags(int(g["dev_status"][0])) == 6
    # the other routes still form a valid schedule of their own
    placed = g["route_row"].reshape(-1)
    placed = placed[placed >= 0]
    assert len(np.unique(placed)) == P * N * k - 1


def _boundary_rows(offsets, counts, n_big=3, span=256):
    """Rows a tile-order or boundary bug would hit first: the first and last
    `span` rows of the n_big largest segments, and every non-empty segment's
    first row, last real row and first padding row."""
    off = np.asarray(offsets, np.int64)
    T = np.asarray(counts, np.int64).sum(axis=1)
    rows = []
    for l in np.argsort(-T, kind="stable")[:n_big]:
        a, b = off[l], off[l] + T[l]
        rows += list(range(a, min(a + span, b))) + list(range(max(a, b - span), b))
    for l in np.nonzero(T > 0)[0]:
        a, real_end, seg_end = off[l], off[l] + T[l], off[l + 1]
        rows += [a, real_end - 1] + ([real_end] if real_end < seg_end else [])
    return np.unique(np.asarray(rows, np.int64))


@pytest.mark.parametrize("name", ["kimi", "zipf"])
def test_schedule_and_dispatch_full_config(cuda_lib, name):
    """The whole Phi, offsets, counts and route_row of the Kimi-shape and Zipf
    layers (routing on the GPU, then the schedule on its ids) bit for bit
    against the oracle's schedule of the oracle's own ids; the dispatch bit
    for bit on >= 4,096 rows that include the largest segments' ends and every
    segment's boundary rows."""
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    lg = inputs.make_logits(w)
    sh = moe.shape(**w.shape())
    ids = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=DEV)
    gates = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg.to(DEV), ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh)
    b["phi"].fill_(-7)
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    torch.cuda.synchronize()
    o_ids, _, _ = oracle.route_topk(lg, w.k)
    assert (ids.cpu().numpy() == o_ids).all()
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    g = {k_: v.cpu().numpy() for k_, v in b.items()}
    _assert_sched_equal(g, s)
    assert s["reads"] == 2 * w.n_routes
    T = s["counts"].sum(axis=1)
    seg = np.diff(s["offsets"])
    assert (seg % 256 == 0).all() and (seg - T < 256).all() and (seg >= T).all()
    if name == "zipf":
        empties = inputs.empty_experts(w)
        assert (T[empties] == 0).all() and (seg[empties] == 0).all()
        hot = int(np.argmax(T))
        assert T[hot] > 0.10 * w.n_routes
        # the hot expert's routes come from every peer and from many 2,048-route blocks
        rr = s["route_row"]
        in_hot = (rr >= s["offsets"][hot]) & (rr < s["offsets"][hot] + T[hot])
        q = np.nonzero(in_hot.reshape(w.P, -1))
        assert len(np.unique(q[0])) == w.P
        assert len(np.unique(q[1] // 2048)) == (w.N * w.k + 2047) // 2048
    # dispatch on sampled rows
    x = inputs.make_x(w)
    rm = moe.rows_max(sh)
    xg = torch.empty((rm, w.H), dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_dispatch(x.to(DEV), b["phi"], b["offsets"], xg, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows_used = int(s["offsets"][-1])
    pick = _boundary_rows(s["offsets"], s["counts"])
    rng = np.random.default_rng(w.wid)
    extra = rng.choice(rows_used, max(0, 4096 - len(pick)) + 512, replace=False)
    pick = np.unique(np.concatenate([pick, extra]))
    assert len(pick) >= 4096
    got = bits(xg[torch.from_numpy(pick).to(DEV)])
    assert (got == oracle.dispatch_rows(bits(x), w.N, s["phi"], pick)).all()
    del xg
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- routing
@pytest.mark.parametrize("name", ["tiny", "mid", "kimi", "zipf"])
def test_route_topk(cuda_lib, name):
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    lg = inputs.make_logits(w)
    sh = moe.shape(**w.shape())
    ids = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=DEV)
    gates = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg.to(DEV), ids, gates, sh)
    torch.cuda.synchronize()
    o_ids, o_g32, o_g64 = oracle.route_topk(lg, w.k)
    assert (ids.cpu().numpy() == o_ids).all()
    g = gates.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g - o_g64) / o_g64) < 1e-6   # a few fp32 ulp (expf + divide)
    if w.n_empty:
        assert not np.isin(o_ids, inputs.empty_experts(w)).any()


def test_route_topk_ties(cuda_lib):
    moe = cuda_lib
    w = json.load(open(os.path.join(GOLD, "worked_numbers.json")))["topk_ties"]
    row = [float(v) for v in w["logits"]]
    lg = torch.tensor([row] * 3, dtype=torch.float32)
    lg[1] = torch.tensor([0.0] * 5)  # all tied: lowest ids first
    sh = moe.shape(1, 3, 5, w["k"])
    ids = torch.empty((3, w["k"]), dtype=torch.int32, device=DEV)
    gates = torch.empty((3, w["k"]), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg.to(DEV), ids, gates, sh)
    o_ids, _, o_g64 = oracle.route_topk(lg, w["k"])
    assert ids.cpu().numpy()[0].tolist() == w["ids"]
    assert (ids.cpu().numpy() == o_ids).all()
    np.testing.assert_allclose(gates.cpu().numpy(), o_g64, rtol=1e-6)


@pytest.mark.parametrize("E,k", [(64, 4), (384, 8), (1024, 16), (7, 7)])
def test_route_topk_heavy_ties_and_neg_inf(cuda_lib, E, k):
    """Rows with many equal logits (more than 32 reach the threshold: the
    fallback path) and rows with -inf logits, mixed with ordinary rows."""
    moe = cuda_lib
    g = torch.Generator().manual_seed(E + k)
    T = 300
    lg = torch.randn((T, E), generator=g)
    lg[0::5] = 0.0                                    # all tied
    lg[1::5, : E // 2] = float("-inf")                # half the experts unreachable
    lg[2::5] = torch.randint(0, 3, (len(range(2, T, 5)), E), generator=g).float()  # coarse ties
    lg[3::5, 1:] = float("-inf")                      # one finite logit, the rest -inf
    sh = moe.shape(1, T, E, k)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gates = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg.to(DEV), ids, gates, sh)
    torch.cuda.synchronize()
    o_ids, _, o_g64 = oracle.route_topk(lg, k)
    assert (ids.cpu().numpy() == o_ids).all()
    g_ = gates.cpu().numpy().astype(np.float64)
    ok = o_g64 > 0
    assert np.all(np.abs(g_[ok] - o_g64[ok]) / o_g64[ok] < 1e-6)
    assert np.all(g_[~ok] == 0)


@pytest.mark.parametrize("E,k", [(16, 2), (48, 8), (64, 1), (128, 5), (160, 8), (256, 3),
                                 (320, 8), (512, 8), (384, 12), (256, 16), (36, 4), (100, 8),
                                 (388, 8), (96, 9)])
def test_route_topk_shapes(cuda_lib, E, k):
    """Every routing kernel variant (four lanes per token for E % 16 == 0 and
    k <= 8, at each chunk count; eight lanes for other multiples of 4 or
    k > 8; one warp per token otherwise) on a ragged token count: random rows,
    rows whose winners all fall in one lane's chunks (more candidates in that
    lane than its slots), tied rows and rows with -inf logits."""
    moe = cuda_lib
    g = torch.Generator().manual_seed(1000 * E + k)
    T = 300
    lg = torch.randn((T, E), generator=g)
    lane0 = [c * 4 + j for c in range(0, (E + 3) // 4, 4) for j in range(4) if c * 4 + j < E]
    lg[4::7, lane0] += 8.0                           # winners crowd the first lane of a quad
    lg[5::7] = 0.5                                   # all tied
    lg[6::7, ::3] = float("-inf")                    # a third of the experts unreachable
    sh = moe.shape(1, T, E, k)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gates = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg.to(DEV), ids, gates, sh)
    torch.cuda.synchronize()
    o_ids, _, o_g64 = oracle.route_topk(lg, k)
    assert (ids.cpu().numpy() == o_ids).all()
    g_ = gates.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g_ - o_g64) / o_g64) < 1e-6


# ---------------------------------------------------------------- stages on small layers
def _stage_run(moe, w, W1, W3, W2, lg, x):
    """Run every stage through its own entry point; return device tensors."""
    sh = moe.shape(**w.shape())
    T, k = w.n_tokens, w.k
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gates = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg, ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh)
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    rm = moe.rows_max(sh)
    xg = torch.empty((rm, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch(x, b["phi"], b["offsets"], xg, b["dev_status"], sh)
    h = torch.empty((rm, w.I), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((rm, w.H), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn(xg, W1, W3, W2, b["offsets"], b["counts"], h, y, b["dev_status"], sh)
    out = torch.empty((T, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(y, b["route_row"], gates, out, b["dev_status"], sh)
    torch.cuda.synchronize()
    return dict(ids=ids, gates=gates, xg=xg, h=h, y=y, out=out, **b)


def _check_combine_stage(moe, w, s, o_g32, toks):
    """moe_combine on seeded stand-in expert outputs y [rows, H] with the oracle's
    route_row and gates, against the oracle's fixed-order fp32 combine: bit-exact."""
    sh = moe.shape(**w.shape())
    rows = int(s["offsets"][-1])
    y = inputs.make_expert_outputs(w, max(rows, 1))
    rr = torch.from_numpy(np.ascontiguousarray(s["route_row"].reshape(-1, w.k))).to(DEV)
    gt = torch.from_numpy(np.ascontiguousarray(o_g32.reshape(-1, w.k))).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(y.to(DEV), rr, gt, out, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    toks = np.asarray(list(toks))
    rrt = s["route_row"].reshape(-1, w.k)[toks]
    used = np.unique(rrt)
    exp = oracle.combine_f32(y.numpy()[used], np.searchsorted(used, rrt), o_g32.reshape(-1, w.k)[toks], w.k)
    assert (bits(out)[toks] == exp).all()


def test_tiny_all_stages_vs_oracle(cuda_lib):
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny"]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = inputs.make_weights(w)
    r = _stage_run(moe, w, W1.to(DEV), W3.to(DEV), W2.to(DEV), lg.to(DEV), x.to(DEV))
    assert int(r["dev_status"].item()) == 0
    o_ids, o_g32, o_g64 = oracle.route_topk(lg, w.k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    g = {k_: r[k_].cpu().numpy() for k_ in ("phi", "offsets", "counts", "route_row")}
    g["dev_status"] = r["dev_status"].cpu().numpy()
    _assert_sched_equal(g, s)
    rows = int(s["offsets"][-1])
    # dispatch: bit-exact on every row in use, padding rows zero
    o_xg = oracle.dispatch_rows(bits(x), w.N, s["phi"], np.arange(rows))
    assert (bits(r["xg"][:rows]) == o_xg).all()
    # FFN on every row that carries a route
    real = np.nonzero(s["phi"][:, 0] >= 0)[0]
    ex = oracle.expert_of_rows(s["offsets"], real)
    Wd = expert_weights_host(W1, W3, W2, range(w.E))
    o_h, o_y = oracle.ffn_rows(o_xg[real], ex, *Wd, H=w.H, I=w.I)
    gh = bits(r["h"][torch.from_numpy(real).to(DEV)])
    assert (gh == o_h).mean() > 0.995
    gy = r["y"][torch.from_numpy(real).to(DEV)].cpu().numpy()
    assert rms_floor_err(gy, o_y) < Y_TOL
    # combine: bit-exact against the fixed-order definition, both sides fed the
    # same seeded stand-in expert outputs and the oracle's own gates and route_row
    _check_combine_stage(moe, w, s, o_g32, range(w.n_tokens))
    # end to end against the oracle's fp64 layer output
    res = oracle.layer_tokens(lg, bits(x), Wd, w.P, w.N, w.k, w.E, w.H, w.I, range(w.n_tokens))
    assert rms_floor_err(bf16_to_f64(bits(r["out"])), res["out64"]) < OUT_TOL


def test_ffn_no_counts_computes_padding_rows(cuda_lib):
    """Without counts the FFN also computes padding tiles: zero rows give zero h and y."""
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny"]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = [t.to(DEV) for t in inputs.make_weights(w)]
    r = _stage_run(moe, w, W1, W3, W2, lg.to(DEV), x.to(DEV))
    sh = moe.shape(**w.shape())
    rows = int(r["offsets"][-1].item())
    h2 = torch.full_like(r["h"], 7.0)
    y2 = torch.full_like(r["y"], 7.0)
    moe.moe_expert_ffn(r["xg"], W1, W3, W2, r["offsets"], None, h2, y2, r["dev_status"], sh)
    torch.cuda.synchronize()
    pad = torch.from_numpy(np.nonzero(r["phi"][:rows, 0].cpu().numpy() < 0)[0]).to(DEV)
    assert (y2[pad] == 0).all() and (h2[pad].float() == 0).all()
    real = torch.from_numpy(np.nonzero(r["phi"][:rows, 0].cpu().numpy() >= 0)[0]).to(DEV)
    assert torch.equal(y2[real], r["y"][real]) and torch.equal(h2[real], r["h"][real])


def test_ffn_counts_leave_padding_blocks_of_y_unwritten(cuda_lib):
    """With counts, GEMM2 writes y for every row that carries a route and skips
    the 32-row blocks wholly past their expert's last route (padding rows
    nothing reads); the rows it writes equal the count-less run's."""
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny"]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = [t.to(DEV) for t in inputs.make_weights(w)]
    r = _stage_run(moe, w, W1, W3, W2, lg.to(DEV), x.to(DEV))
    sh = moe.shape(**w.shape())
    rows = int(r["offsets"][-1].item())
    h2 = torch.empty_like(r["h"])
    y2 = torch.full_like(r["y"], 7.0)
    moe.moe_expert_ffn(r["xg"], W1, W3, W2, r["offsets"], r["counts"], h2, y2, r["dev_status"], sh)
    torch.cuda.synchronize()
    assert int(r["dev_status"].item()) == 0
    phi = r["phi"][:rows, 0].cpu().numpy()
    real = np.nonzero(phi >= 0)[0]
    yd, y2h = r["y"].cpu(), y2.cpu()
    assert torch.equal(y2h[real], yd[real])
    off = r["offsets"].cpu().numpy()
    cnt = r["counts"].cpu().numpy().sum(axis=1)
    skipped = 0
    for l in range(w.E):
        end = off[l] + cnt[l]
        for b0 in range((end + 31) // 32 * 32, off[l + 1], 32):  # blocks wholly past the routes
            assert (y2h[b0:b0 + 32] == 7.0).all()
            skipped += 1
    assert skipped > 0, "the case has padding blocks past an expert's last route"


@pytest.mark.parametrize("name,pad", [("tiny", 256), ("mid", 256), ("tiny", 128)])
def test_ffn_gather_equals_dispatch_then_ffn(cuda_lib, name, pad):
    """The FFN that pulls its rows from x by Phi reproduces dispatch + FFN bit for bit."""
    moe = cuda_lib
    w0 = inputs.WORKLOADS[name]
    w = inputs.Workload(w0.name, w0.wid, P=w0.P, N=w0.N, E=w0.E, k=w0.k, H=w0.H, I=w0.I, pad=pad)
    lg, x = inputs.make_logits(w0), inputs.make_x(w0)
    W1, W3, W2 = [t.to(DEV) for t in inputs.make_weights(w0)]
    r = _stage_run(moe, w, W1, W3, W2, lg.to(DEV), x.to(DEV))
    sh = moe.shape(**w.shape())
    h2 = torch.full_like(r["h"], 3.0)
    y2 = torch.full_like(r["y"], 3.0)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_expert_ffn_gather(x.to(DEV), r["phi"], W1, W3, W2, r["offsets"], r["counts"], h2, y2,
                              st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = int(r["offsets"][-1].item())
    real = torch.from_numpy(np.nonzero(r["phi"][:rows, 0].cpu().numpy() >= 0)[0]).to(DEV)
    assert torch.equal(h2[real], r["h"][real]) and torch.equal(y2[real], r["y"][real])


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_ffn_gather_vs_oracle(cuda_lib, name):
    """The FFN that pulls its A rows from x through Phi, against the oracle's
    dispatch and FFN (schedule from the oracle's own routing)."""
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = inputs.make_weights(w)
    sh = moe.shape(**w.shape())
    o_ids, _, _ = oracle.route_topk(lg, w.k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    rm = moe.rows_max(sh)
    rows = int(s["offsets"][-1])
    phi = torch.full((rm, 2), -1, dtype=torch.int32)
    phi[:rows] = torch.from_numpy(s["phi"])
    offs = torch.from_numpy(s["offsets"]).to(DEV)
    cnts = torch.from_numpy(np.ascontiguousarray(s["counts"])).to(DEV)
    h = torch.empty((rm, w.I), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((rm, w.H), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_expert_ffn_gather(x.to(DEV), phi.to(DEV), W1.to(DEV), W3.to(DEV), W2.to(DEV), offs,
                              cnts, h, y, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    real = np.nonzero(s["phi"][:, 0] >= 0)[0]
    if len(real) > 600:
        rng = np.random.default_rng(w.wid)
        real = np.unique(np.concatenate([real[:64], real[-64:], rng.choice(real, 400, replace=False)]))
    ex = oracle.expert_of_rows(s["offsets"], real)
    o_xg = oracle.dispatch_rows(bits(x), w.N, s["phi"], real)
    o_h, o_y = oracle.ffn_rows(o_xg, ex, *expert_weights_host(W1, W3, W2, ex), H=w.H, I=w.I)
    idx = torch.from_numpy(real).to(DEV)
    assert (bits(h[idx]) == o_h).mean() > 0.995
    assert rms_floor_err(y[idx].cpu().numpy(), o_y) < Y_TOL


def test_ffn_gather_flags_corrupt_phi(cuda_lib):
    """A Phi entry outside [0,P)x[0,N) is reported and its row reads as zeros."""
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny"]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = [t.to(DEV) for t in inputs.make_weights(w)]
    r = _stage_run(moe, w, W1, W3, W2, lg.to(DEV), x.to(DEV))
    sh = moe.shape(**w.shape())
    phi = r["phi"].clone()
    real = np.nonzero(phi[:, 0].cpu().numpy() >= 0)[0]
    victim = int(real[5])
    phi[victim, 1] = w.N + 3  # token index out of range
    h2 = torch.zeros_like(r["h"])
    y2 = torch.zeros_like(r["y"])
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_expert_ffn_gather(x.to(DEV), phi, W1, W3, W2, r["offsets"], r["counts"], h2, y2, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.DEV_BAD_SCHEDULE
    assert (y2[victim] == 0).all()
    other = int(real[6])
    assert torch.equal(y2[other], r["y"][other])


def test_mid_stages_sampled(cuda_lib):
    moe = cuda_lib
    w = inputs.WORKLOADS["mid"]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = inputs.make_weights(w)
    r = _stage_run(moe, w, W1.to(DEV), W3.to(DEV), W2.to(DEV), lg.to(DEV), x.to(DEV))
    assert int(r["dev_status"].item()) == 0
    o_ids, _, o_g64 = oracle.route_topk(lg, w.k)
    assert (r["ids"].cpu().numpy() == o_ids).all()
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    g = {k_: r[k_].cpu().numpy() for k_ in ("phi", "offsets", "counts", "route_row", "dev_status")}
    _assert_sched_equal(g, s)
    rows = int(s["offsets"][-1])
    o_xg = oracle.dispatch_rows(bits(x), w.N, s["phi"], np.arange(rows))
    assert (bits(r["xg"][:rows]) == o_xg).all()
    # FFN on sampled rows: first/last row of several experts plus random rows
    rng = np.random.default_rng(5)
    real = np.nonzero(s["phi"][:, 0] >= 0)[0]
    pick = np.unique(np.concatenate([real[:3], real[-3:], rng.choice(real, 250, replace=False)]))
    ex = oracle.expert_of_rows(s["offsets"], pick)
    Wd = expert_weights_host(W1, W3, W2, ex)
    o_h, o_y = oracle.ffn_rows(o_xg[pick], ex, *Wd, H=w.H, I=w.I)
    idx = torch.from_numpy(pick).to(DEV)
    assert (bits(r["h"][idx]) == o_h).mean() > 0.995
    assert rms_floor_err(r["y"][idx].cpu().numpy(), o_y) < Y_TOL
    # combine bit-exact on sampled tokens (seeded stand-in expert outputs)
    _, o_g32, _ = oracle.route_topk(lg, w.k)
    _check_combine_stage(moe, w, s, o_g32, inputs.sample_tokens(w.n_tokens, 300, seed=2))


# ---------------------------------------------------------------- whole layer
_LAYER_CACHE = {}


def _layer_inputs(name):
    if name not in _LAYER_CACHE:
        _LAYER_CACHE.clear()
        torch.cuda.empty_cache()
        w = inputs.WORKLOADS[name]
        big = w.H * w.I * w.E > 1e9
        lg, x = inputs.make_logits(w), inputs.make_x(w)
        W = inputs.make_weights(w, device=DEV if big else "cpu")
        _LAYER_CACHE[name] = (w, lg, x, W)
    return _LAYER_CACHE[name]


def _layer_gpu(moe, w, lg_d, x_d, Wd, minibatch=0, ws=None):
    sh = moe.shape(**w.shape())
    if ws is None:
        ws = torch.empty(moe.layer_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=DEV)
    moe.moe_layer_forward(lg_d, x_d, *Wd, out, ws, st, sh, minibatch_tokens=minibatch)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out, ws


def _layer_tokens_for(w, lg, n_tok):
    """n_tok tokens: those owning the first and last real rows of the three
    largest expert segments and the last real row of every tenth segment,
    then seeded random tokens."""
    o_ids, _, _ = oracle.route_topk(lg, w.k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    T = s["counts"].sum(axis=1)
    off = s["offsets"].astype(np.int64)
    rows = []
    for l in np.argsort(-T, kind="stable")[:3]:
        rows += list(range(off[l], off[l] + 8)) + list(range(off[l] + T[l] - 8, off[l] + T[l]))
    rows += [off[l] + T[l] - 1 for l in np.nonzero(T > 0)[0][::10]]
    phi = s["phi"][np.asarray(rows, np.int64)]
    toks = set((phi[:, 0].astype(np.int64) * w.N + phi[:, 1]).tolist())
    rng = np.random.default_rng(w.wid)
    while len(toks) < n_tok:
        toks.add(int(rng.integers(w.n_tokens)))
    return sorted(toks)


@pytest.mark.parametrize("name,n_tok", [("tiny", 512), ("mid", 96), ("kimi", 256), ("zipf", 256)])
def test_layer_vs_oracle(cuda_lib, name, n_tok):
    moe = cuda_lib
    w, lg, x, W = _layer_inputs(name)
    Wd = [t.to(DEV) for t in W]
    out, ws = _layer_gpu(moe, w, lg.to(DEV), x.to(DEV), Wd)
    if name in ("kimi", "zipf"):
        toks = _layer_tokens_for(w, lg, n_tok)
    else:
        toks = inputs.sample_tokens(w.n_tokens, n_tok, seed=w.wid)
    o_ids, _, _ = oracle.route_topk(lg[toks], w.k)
    # weights go to the host one group of experts at a time
    Wh = lambda ex: expert_weights_host(*Wd, ex)
    res = oracle.layer_tokens(lg, bits(x), Wh, w.P, w.N, w.k, w.E, w.H, w.I, toks)
    got = bf16_to_f64(bits(out[torch.tensor(toks, device=DEV)]))
    err = rms_floor_err(got, res["out64"])
    print(f"{name}: rms-floor err {err:.3e}, literal max|d|/rms {literal_rms_err(got, res['out64']):.3e}")
    assert err < OUT_TOL
    if name == "zipf":
        ids_all = res["ids"]
        assert not np.isin(ids_all, inputs.empty_experts(w)).any()
        counts = np.bincount(ids_all.reshape(-1), minlength=w.E)
        assert counts.max() > 0.10 * ids_all.size, "a hot expert takes >10% of routes"
        s = res["sched"]
        assert (np.diff(s["offsets"])[inputs.empty_experts(w)] == 0).all()
        top3 = np.argsort(-counts, kind="stable")[:3]
        assert all(np.isin(top3[i], o_ids) for i in range(3)), "sampled tokens reach the hot experts"


@pytest.mark.parametrize("name", ["tiny", "mid", "kimi", "zipf"])
def test_layer_bitwise_deterministic_and_slice_invariant(cuda_lib, name):
    moe = cuda_lib
    w, lg, x, W = _layer_inputs(name)
    Wd = [t.to(DEV) for t in W]
    lg_d, x_d = lg.to(DEV), x.to(DEV)
    out0, ws = _layer_gpu(moe, w, lg_d, x_d, Wd)
    h0 = sha(out0)
    for _ in range(2):
        out1, _ = _layer_gpu(moe, w, lg_d, x_d, Wd, ws=ws)
        assert sha(out1) == h0
    slices = [w.minibatch] if w.minibatch else []
    if w.N >= 4 * 2368 // 3:
        slices = sorted(set(slices + [2368]))
    for T in slices + [max(1, w.N // 3), 97]:
        outT, _ = _layer_gpu(moe, w, lg_d, x_d, Wd, minibatch=T, ws=ws)
        assert sha(outT) == h0, f"transfer slice {T} changed the output"


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_layer_equals_its_stage_entries(cuda_lib, name):
    """The layer (whose GEMM1 lands the dispatch itself when segments are padded
    to 256 rows) gives bit for bit the output of the separate entry points:
    moe_route_topk, moe_schedule, moe_dispatch, moe_expert_ffn, moe_combine."""
    moe = cuda_lib
    w, lg, x, W = _layer_inputs(name)
    Wd = [t.to(DEV) for t in W]
    out, _ = _layer_gpu(moe, w, lg.to(DEV), x.to(DEV), Wd)
    r = _stage_run(moe, w, *Wd, lg.to(DEV), x.to(DEV))
    assert int(r["dev_status"].item()) == 0
    assert torch.equal(out, r["out"])


@pytest.mark.parametrize("minibatch", [0, 1000, 4096, 2368])
def test_layer_host_entry_matches_device_entry(cuda_lib, minibatch):
    """Host buffers in and out, transfers overlapped with compute slice by slice
    (ragged last slice included) and across calls (two input batches
    alternated, so both internal input copies and their reuse are exercised):
    identical to the device-buffer entry."""
    moe = cuda_lib
    w, lg, x, W = _layer_inputs("mid")
    Wd = [t.to(DEV) for t in W]
    perm = torch.randperm(w.n_tokens, generator=torch.Generator().manual_seed(9))
    batches = [(lg, x), (lg[perm].contiguous(), x[perm].contiguous())]
    refs = [_layer_gpu(moe, w, a.to(DEV), b.to(DEV), Wd)[0].cpu() for a, b in batches]
    sh = moe.shape(**w.shape())
    ws = torch.empty(moe.layer_host_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    pinned = [(a.pin_memory(), b.pin_memory()) for a, b in batches]
    outs = [torch.full((w.n_tokens, w.H), 7.0, dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    for c in range(5):  # calls issued back to back, synchronised once at the end
        lg_h, x_h = pinned[c % 2]
        moe.moe_layer_forward_host(lg_h, x_h, *Wd, outs[c], ws, st, sh, minibatch_tokens=minibatch)
    torch.cuda.current_stream().synchronize()
    assert int(st.item()) == 0
    for c in range(5):
        assert torch.equal(outs[c], refs[c % 2]), f"call {c}"


@pytest.mark.parametrize("minibatch", [0, 2368])
def test_layer_host_async_entry_matches_device_entry(cuda_lib, minibatch):
    """The async-output host entry: six calls back to back (two input batches
    alternated, so both device input copies and both device output copies are
    reused), one synchronous call in between; each call's host output, read
    after its own event, equals the device-buffer entry's."""
    moe = cuda_lib
    w, lg, x, W = _layer_inputs("mid")
    Wd = [t.to(DEV) for t in W]
    perm = torch.randperm(w.n_tokens, generator=torch.Generator().manual_seed(9))
    batches = [(lg, x), (lg[perm].contiguous(), x[perm].contiguous())]
    refs = [_layer_gpu(moe, w, a.to(DEV), b.to(DEV), Wd)[0].cpu() for a, b in batches]
    sh = moe.shape(**w.shape())
    ws = torch.empty(moe.layer_host_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    pinned = [(a.pin_memory(), b.pin_memory()) for a, b in batches]
    n = 7
    outs = [torch.full((w.n_tokens, w.H), 7.0, dtype=torch.bfloat16).pin_memory() for _ in range(n)]
    evs = [torch.cuda.Event() for _ in range(n)]
    for e in evs:
        e.record()  # creates the event
    torch.cuda.synchronize()
    for c in range(n):
        lg_h, x_h = pinned[c % 2]
        if c == 3:
            moe.moe_layer_forward_host(lg_h, x_h, *Wd, outs[c], ws, st, sh,
                                       minibatch_tokens=minibatch)
            evs[c].record()
        else:
            moe.moe_layer_forward_host_async(lg_h, x_h, *Wd, outs[c], ws, st, sh, evs[c],
                                             minibatch_tokens=minibatch)
    for c in range(n):
        evs[c].synchronize()
        assert torch.equal(outs[c], refs[c % 2]), f"call {c}"
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_layer_concurrent_streams(cuda_lib):
    """Two layer calls running at the same time on two streams (own workspaces):
    each GEMM launch takes its own tile counter, so both outputs equal the
    single-stream result bit for bit."""
    moe = cuda_lib
    w, lg, x, W = _layer_inputs("mid")
    Wd = [t.to(DEV) for t in W]
    lg_d, x_d = lg.to(DEV), x.to(DEV)
    ref, _ = _layer_gpu(moe, w, lg_d, x_d, Wd)
    sh = moe.shape(**w.shape())
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [torch.empty(moe.layer_workspace_bytes(sh), dtype=torch.uint8, device=DEV) for _ in streams]
    sts = [torch.zeros(1, dtype=torch.int32, device=DEV) for _ in streams]
    outs = [torch.empty_like(ref) for _ in streams]
    torch.cuda.synchronize()
    for _ in range(3):
        for s_, ws_, st_, o_ in zip(streams, wss, sts, outs):
            with torch.cuda.stream(s_):
                moe.moe_layer_forward(lg_d, x_d, *Wd, o_, ws_, st_, sh, stream=s_)
    torch.cuda.synchronize()
    for st_, o_ in zip(sts, outs):
        assert int(st_.item()) == 0
        assert torch.equal(o_, ref)


def test_ffn_launch_waiting_on_an_event_while_another_stream_queues_300(cuda_lib):
    """A GEMM launch held back on one stream (it waits for an event recorded
    after a spin kernel) is undisturbed by 300 FFN calls (600 GEMM launches)
    that another stream enqueues and runs meanwhile, cycling through every
    counter of the pool: its output equals the one computed alone."""
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny"]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    W1, W3, W2 = [t.to(DEV) for t in inputs.make_weights(w)]
    r = _stage_run(moe, w, W1, W3, W2, lg.to(DEV), x.to(DEV))
    sh = moe.shape(**w.shape())
    ref_h, ref_y = r["h"].clone(), r["y"].clone()
    gate, a, b = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = torch.cuda.Event()
    h_a, y_a = torch.zeros_like(ref_h), torch.zeros_like(ref_y)
    h_b, y_b = torch.zeros_like(ref_h), torch.zeros_like(ref_y)
    st_a = torch.zeros(1, dtype=torch.int32, device=DEV)
    st_b = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    with torch.cuda.stream(gate):
        torch.cuda._sleep(300_000_000)  # well over 100 ms at any SM clock
        ev.record(gate)
    a.wait_event(ev)
    moe.moe_expert_ffn(r["xg"], W1, W3, W2, r["offsets"], r["counts"], h_a, y_a, st_a, sh,
                       stream=a)
    for _ in range(300):
        moe.moe_expert_ffn(r["xg"], W1, W3, W2, r["offsets"], r["counts"], h_b, y_b, st_b, sh,
                           stream=b)
    torch.cuda.synchronize()
    assert int(st_a.item()) == 0 and int(st_b.item()) == 0
    real = torch.from_numpy(np.nonzero(r["phi"][:int(r["offsets"][-1].item()), 0].cpu().numpy() >= 0)[0]).to(DEV)
    for h_, y_ in ((h_a, y_a), (h_b, y_b)):
        assert torch.equal(h_[real], ref_h[real]) and torch.equal(y_[real], ref_y[real])


def test_layer_pad128_single_cta_path(cuda_lib):
    """Segments padded to 128 rows run the single-CTA (128x256 tile) FFN kernels."""
    moe = cuda_lib
    w0 = inputs.WORKLOADS["tiny"]
    w = inputs.Workload("tiny_pad128", w0.wid, P=2, N=100, E=w0.E, k=w0.k, H=w0.H, I=w0.I, pad=128)
    lg = torch.randn((w.n_tokens, w.E), generator=torch.Generator().manual_seed(77))
    x = torch.randn((w.n_tokens, w.H), generator=torch.Generator().manual_seed(78)).to(torch.bfloat16)
    W1, W3, W2 = inputs.make_weights(w0)
    Wd = [t.to(DEV) for t in (W1, W3, W2)]
    out, _ = _layer_gpu(moe, w, lg.to(DEV), x.to(DEV), Wd)
    Wh = expert_weights_host(W1, W3, W2, range(w.E))
    res = oracle.layer_tokens(lg, bits(x), Wh, w.P, w.N, w.k, w.E, w.H, w.I, range(w.n_tokens),
                              pad=128)
    assert rms_floor_err(bf16_to_f64(bits(out)), res["out64"]) < OUT_TOL
    assert all(int(v) % 128 == 0 for v in res["sched"]["offsets"])
    assert any(int(v) % 256 != 0 for v in res["sched"]["offsets"])


@pytest.mark.parametrize("P,N,E,k,H,I", [
    (64, 3, 1024, 16, 256, 128),    # most peers, experts and routes per token
    (1, 1, 8, 2, 256, 128),          # a single token
    (3, 131, 5, 5, 512, 256),        # k = E, ragged token count
    (2, 700, 1, 1, 256, 384),        # one expert takes everything
])
def test_layer_edge_shapes(cuda_lib, P, N, E, k, H, I):
    moe = cuda_lib
    w = inputs.Workload("edge", 7, P=P, N=N, E=E, k=k, H=H, I=I)
    g = torch.Generator().manual_seed(P * 1000 + N)
    lg = torch.randn((w.n_tokens, E), generator=g)
    x = torch.randn((w.n_tokens, H), generator=g).to(torch.bfloat16)
    W1 = (torch.randn((E, H, I), generator=g) * 0.02).to(torch.bfloat16)
    W3 = (torch.randn((E, H, I), generator=g) * 0.02).to(torch.bfloat16)
    W2 = (torch.randn((E, I, H), generator=g) * 0.02).to(torch.bfloat16)
    Wd = [t.to(DEV) for t in (W1, W3, W2)]
    out, _ = _layer_gpu(moe, w, lg.to(DEV), x.to(DEV), Wd)
    toks = inputs.sample_tokens(w.n_tokens, 64, seed=3)
    o_ids, _, _ = oracle.route_topk(lg[toks], k)
    Wh = expert_weights_host(W1, W3, W2, np.unique(o_ids))
    res = oracle.layer_tokens(lg, bits(x), Wh, P, N, k, E, H, I, toks)
    got = bf16_to_f64(bits(out[torch.tensor(toks, device=DEV)]))
    assert rms_floor_err(got, res["out64"]) < OUT_TOL


def test_layer_no_tokens(cuda_lib):
    """N = 0: nothing to route; the call succeeds and touches no output."""
    moe = cuda_lib
    sh = moe.shape(2, 0, 8, 2, 256, 128)
    ws = torch.empty(moe.layer_workspace_bytes(sh), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    e = torch.empty((0,), device=DEV)
    W = torch.zeros((8, 256, 128), dtype=torch.bfloat16, device=DEV)
    W2 = torch.zeros((8, 128, 256), dtype=torch.bfloat16, device=DEV)
    moe.moe_layer_forward(e.float().reshape(0, 8), e.to(torch.bfloat16).reshape(0, 256), W, W, W2,
                          e.to(torch.bfloat16).reshape(0, 256), ws, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
