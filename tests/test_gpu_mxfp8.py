"""GPU parity of the MXFP8 quantisation kernels (through the C ABI) against the
oracle's MX quantisation: E4M3 codes and E8M0 scales bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_route_counting_b200 import inputs
from tests.helpers import bf16_to_f64, bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _crafted_rows(n_rows=64, K=512, seed=4):
    """bf16 rows whose 32-blocks span the whole bf16 range: zero blocks, bf16
    subnormals, huge magnitudes, negative zeros, exact powers of two, blocks
    whose largest scaled values saturate."""
    g = torch.Generator().manual_seed(seed)
    base = torch.randn((n_rows, K), generator=g, dtype=torch.float32)
    mags = torch.exp2(torch.randint(-140, 126, (n_rows, K // 32), generator=g).float())
    x = (base.view(n_rows, K // 32, 32) * mags.unsqueeze(-1)).view(n_rows, K)
    x[0] = 0.0
    x[1, :32] = -0.0
    x[2, :32] = torch.exp2(torch.arange(32).float() - 20)           # powers of two
    x[3, :32] = 1.99 * 2.0 ** 10                                   # bf16 2040: scaled 510, clamped to 448
    x[3, 5] = 1.0
    x[4] = 2.0 ** -133 * torch.arange(1, K + 1).float() % 127      # bf16 subnormals
    x[5] = 3.0e38 * torch.sign(base[5])
    return x.to(torch.bfloat16)


def _oracle_mx(b16: torch.Tensor):
    return oracle.mx_quantize(bf16_to_f64(bits(b16)))


def test_mx_quantize_rows_bit_exact(cuda_lib):
    moe = cuda_lib
    x = _crafted_rows()
    q = torch.empty(x.shape, dtype=torch.uint8, device=DEV)
    s = torch.empty((x.shape[0], x.shape[1] // 32), dtype=torch.uint8, device=DEV)
    moe.moe_mx_quantize_rows(x.to(DEV), q, s)
    torch.cuda.synchronize()
    oq, os_ = _oracle_mx(x)
    assert (s.cpu().numpy() == os_).all()
    assert (q.cpu().numpy() == oq).all()
    assert (os_[0] == 0).all() and (oq[3, :32] == 0x7E).sum() >= 20  # zero and saturated blocks


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_dispatch_mxfp8_bit_exact(cuda_lib, name):
    moe = cuda_lib
    w = inputs.WORKLOADS[name]
    sh = moe.shape(**w.shape())
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    ids = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=DEV)
    gates = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg.to(DEV), ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh)
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    rm = moe.rows_max(sh)
    xq = torch.full((rm, w.H), 0x55, dtype=torch.uint8, device=DEV)
    xs = torch.full((rm, w.H // 32), 0x55, dtype=torch.uint8, device=DEV)
    moe.moe_dispatch_mxfp8(x.to(DEV), b["phi"], b["offsets"], xq, xs, b["dev_status"], sh)
    torch.cuda.synchronize()
    assert int(b["dev_status"].item()) == 0
    o_ids, _, _ = oracle.route_topk(lg, w.k)
    s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    rows = int(s["offsets"][-1])
    o_xg = oracle.dispatch_rows(bits(x), w.N, s["phi"], np.arange(rows))
    oq, os_ = oracle.mx_quantize(bf16_to_f64(o_xg))
    assert (xq[:rows].cpu().numpy() == oq).all()
    assert (xs[:rows].cpu().numpy() == os_).all()
    pad = s["phi"][:, 0] < 0
    assert (xs[:rows].cpu().numpy()[pad] == 0).all()


def test_dispatch_mxfp8_kimi_sampled_rows(cuda_lib):
    moe = cuda_lib
    w = inputs.WORKLOADS["kimi"]
    sh = moe.shape(**w.shape())
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    ids = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=DEV)
    gates = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=DEV)
    moe.moe_route_topk(lg.to(DEV), ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh)
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    rm = moe.rows_max(sh)
    xq = torch.empty((rm, w.H), dtype=torch.uint8, device=DEV)
    xs = torch.empty((rm, w.H // 32), dtype=torch.uint8, device=DEV)
    moe.moe_dispatch_mxfp8(x.to(DEV), b["phi"], b["offsets"], xq, xs, b["dev_status"], sh)
    torch.cuda.synchronize()
    assert int(b["dev_status"].item()) == 0
    o_ids, _, _ = oracle.route_topk(lg, w.k)
    o_s = oracle.schedule(o_ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, 256)
    rows = int(o_s["offsets"][-1])
    pick = np.unique(np.concatenate([[0, rows - 1], np.random.default_rng(6).choice(rows, 2000)]))
    o_xg = oracle.dispatch_rows(bits(x), w.N, o_s["phi"], pick)
    oq, os_ = oracle.mx_quantize(bf16_to_f64(o_xg))
    idx = torch.from_numpy(pick).to(DEV)
    assert (xq[idx].cpu().numpy() == oq).all()
    assert (xs[idx].cpu().numpy() == os_).all()
