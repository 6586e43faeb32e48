"""Failure detection on the GPU without a fault: bounded device waits and the
error paths of the C ABI."""
import ctypes

import pytest
import torch

from combine_top_route_counting_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_lib):
    moe = cuda_lib
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_selftest_bounded_wait(st, 20_000_000)  # 20 ms on an mbarrier nothing completes
    torch.cuda.synchronize()
    assert int(st.item()) & moe.DEV_TIMEOUT
    assert moe.status_from_device_flags(int(st.item())) == 5
    # the context is still usable
    a = torch.arange(10, device="cuda")
    assert int(a.sum().item()) == 45


def test_schedule_grid_barrier_times_out_and_context_survives(cuda_lib):
    """The schedule's one-launch kernel with a barrier expecting one block more
    than it launched: every block gives up after 20 ms and raises
    MOE_DEV_TIMEOUT; the next ordinary schedule on the same buffers is exact."""
    import oracle
    moe = cuda_lib
    P, N, E, k = 8, 1024, 64, 4
    ids = inputs.make_ids_uniform(P, N, E, k, seed=41)
    sh = moe.shape(P, N, E, k)
    b = moe.alloc_schedule_outputs(sh)
    ids_d = ids.to("cuda")
    moe.moe_selftest_schedule_barrier(ids_d, b["phi"], b["offsets"], b["counts"], b["route_row"],
                                      b["ws"], b["dev_status"], sh, 20_000_000)
    torch.cuda.synchronize()
    assert int(b["dev_status"].item()) & moe.DEV_TIMEOUT
    b["dev_status"].zero_()
    moe.moe_schedule(ids_d, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    torch.cuda.synchronize()
    assert int(b["dev_status"].item()) == 0
    o = oracle.schedule(ids.numpy(), P, N, k, E, 256)
    rows = int(o["offsets"][-1])
    assert (b["phi"][:rows].cpu().numpy() == o["phi"]).all()
    assert (b["route_row"].cpu().numpy() == o["route_row"]).all()


def test_host_side_errors(cuda_lib):
    moe = cuda_lib
    sh = moe.shape(1, 16, 8, 2, 256, 128)
    L = moe.load()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    # null pointers
    assert L.moe_route_topk(None, None, None, ctypes.byref(sh), None) == 1
    # unsupported shapes
    bad = moe.shape(1, 16, 8, 9)  # k > E
    assert moe.rows_max(bad) == -1
    assert moe.layer_workspace_bytes(moe.shape(1, 16, 8, 2, 200, 128)) == 0  # H % 256 != 0
    # workspace too small
    w = inputs.WORKLOADS["tiny"]
    x = torch.zeros((w.n_tokens, w.H), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((w.n_tokens, w.E), dtype=torch.float32, device="cuda")
    W1 = torch.zeros((w.E, w.H, w.I), dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros((w.E, w.I, w.H), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    shw = moe.shape(**w.shape())
    with pytest.raises(moe.MoeError) as e:
        moe.moe_layer_forward(lg, x, W1, W1, W2, out, ws, st, shw)
    assert e.value.status == 3
    with pytest.raises(TypeError):
        moe.moe_layer_forward(lg.cpu(), x, W1, W1, W2, out, ws, st, shw)


def test_corrupt_schedule_is_flagged_not_faulted(cuda_lib):
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny"]
    sh = moe.shape(**w.shape())
    rm = moe.rows_max(sh)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    # offsets beyond rows_max: dispatch and FFN refuse and flag
    offsets = torch.full((w.E + 1,), rm + 256, dtype=torch.int32, device="cuda")
    offsets[0] = 0
    phi = torch.full((rm, 2), -1, dtype=torch.int32, device="cuda")
    x = torch.zeros((w.n_tokens, w.H), dtype=torch.bfloat16, device="cuda")
    xg = torch.zeros((rm, w.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_dispatch(x, phi, offsets, xg, st, sh)
    W1 = torch.zeros((w.E, w.H, w.I), dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros((w.E, w.I, w.H), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((rm, w.I), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((rm, w.H), dtype=torch.float32, device="cuda")
    moe.moe_expert_ffn(xg, W1, W1, W2, offsets, None, h, y, st, sh)
    # route_row out of range: combine skips the slot and flags
    rr = torch.full((w.n_tokens, w.k), rm + 5, dtype=torch.int32, device="cuda")
    g = torch.ones((w.n_tokens, w.k), dtype=torch.float32, device="cuda")
    out = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(y, rr, g, out, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.DEV_BAD_SCHEDULE
    assert (out.float() == 0).all()


def test_backward_corrupt_schedule_is_flagged_not_faulted(cuda_lib):
    """Offsets that are not multiples of the 256-row tile (or run past rows_max)
    make every backward GEMM refuse its work and flag MOE_DEV_BAD_SCHEDULE; the
    reverse dispatch and router gradient skip out-of-range rows. Nothing hangs."""
    moe = cuda_lib
    w = inputs.WORKLOADS["tiny_bwd"]
    sh = moe.shape(**w.shape())
    rm = moe.rows_max(sh)
    dev = "cuda"
    for bad_offsets in ([0, 100] + [100] * (w.E - 1), [0] + [rm + 256] * w.E):
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        offsets = torch.tensor(bad_offsets, dtype=torch.int32, device=dev)
        z16 = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device=dev)
        z32 = lambda *s: torch.zeros(s, dtype=torch.float32, device=dev)
        W1, W2 = z16(w.E, w.H, w.I), z16(w.E, w.I, w.H)
        dab, hg, part, dxg = z16(rm, 2 * w.I), z16(rm, w.I), z32(rm, w.I // 128), z32(rm, w.H)
        moe.moe_expert_ffn_dgrad(z16(rm, w.H), z32(rm), z16(rm, 2 * w.I), z16(rm, w.I), W1, W1, W2,
                                 offsets, None, dab, hg, part, dxg, st, sh)
        dW1, dW3 = torch.full((w.E, w.H, w.I), 5.0, device=dev), torch.full((w.E, w.H, w.I), 5.0, device=dev)
        dW2 = torch.full((w.E, w.I, w.H), 5.0, device=dev)
        moe.moe_expert_ffn_wgrad(z16(rm, w.H), z16(rm, w.H), dab, hg, offsets, None, dW1, dW3, dW2,
                                 st, sh)
        torch.cuda.synchronize()
        assert int(st.item()) & moe.DEV_BAD_SCHEDULE
        assert (dW1 == 5.0).all() and (dW2 == 5.0).all()  # nothing written
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    rr = torch.full((w.n_tokens, w.k), rm + 5, dtype=torch.int32, device=dev)
    ids = torch.zeros((w.n_tokens, w.k), dtype=torch.int32, device=dev)
    g = torch.ones((w.n_tokens, w.k), dtype=torch.float32, device=dev)
    dx = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=dev)
    moe.moe_reverse_dispatch(torch.zeros((rm, w.H), device=dev), rr, dx, st, sh)
    dl = torch.full((w.n_tokens, w.E), 3.0, device=dev)
    moe.moe_router_backward(torch.zeros((rm, w.I // 128), device=dev), rr, ids, g, dl, st, sh)
    torch.cuda.synchronize()
    assert int(st.item()) & moe.DEV_BAD_SCHEDULE
    assert (dx.float() == 0).all() and (dl == 0).all()
    # the context is still usable
    assert int(torch.arange(10, device=dev).sum().item()) == 45
