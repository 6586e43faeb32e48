"""The schedule entry point that allocates nothing (moe_schedule_static_ws).

It serves callers that cannot give the library a scratch buffer (a plugin
handed only its inputs and outputs, a serving loop that bans cudaMalloc on
its hot path). Its results must equal those of moe_schedule, which takes the
caller's workspace, bit for bit, call after call, even though every call
reuses the same fixed device array. This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from combine_top_route_counting_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(moe, ids, sh, static):
    b = moe.alloc_schedule_outputs(sh)
    b["phi"].fill_(-7)
    if static:
        moe.moe_schedule_static_ws(ids, b["phi"], b["offsets"], b["counts"], b["route_row"],
                                   b["dev_status"], sh)
    else:
        moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                         b["dev_status"], sh)
    torch.cuda.synchronize()
    rows = int(b["offsets"][-1].item())
    return {"phi": b["phi"][:rows].cpu(), "offsets": b["offsets"].cpu(),
            "counts": b["counts"].cpu(), "route_row": b["route_row"].cpu(),
            "dev_status": b["dev_status"].cpu()}


def test_static_scratch_schedule_matches_workspace_schedule(cuda_lib):
    moe = cuda_lib
    wl = inputs.WORKLOADS["sched"]
    cases = [
        (wl.P, wl.N, wl.E, wl.k, inputs.make_sched_ids(wl)),        # the full scheduler workload
        (3, 777, 50, 4, inputs.make_ids_uniform(3, 777, 50, 4, seed=31)),  # smaller, after it
    ]
    for P, N, E, k, ids in cases:
        sh = moe.shape(P, N, E, k)
        ids_d = ids.to(DEV)
        ref = _run(moe, ids_d, sh, static=False)
        for _ in range(2):  # two calls in a row on the shared array
            got = _run(moe, ids_d, sh, static=True)
            for key in ref:
                assert torch.equal(got[key], ref[key]), key
            assert int(got["dev_status"][0]) == 0


def test_static_scratch_rejects_oversized_shapes(cuda_lib):
    moe = cuda_lib
    # P * ceil(N*k/2048) * E = 64 * 512 * 1024 words > 1,048,576: refused before any launch
    sh = moe.shape(64, 131072, 1024, 8)
    L = moe.load()
    p = ctypes.c_void_p(256)
    n0 = moe.launch_count()
    assert L.moe_schedule_static_ws(p, p, p, p, p, p, ctypes.byref(sh), None) == 3
    assert moe.launch_count() == n0
