"""Host logic of bench.py on CPU: the world-size-2 path with gloo ranks (max over
ranks, barrier, teardown), argument checks, and the reference arm's rank gate."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    ready = bench.init_dist(world, rank, backend="gloo")
    vals = bench.reduce_max([10.0 * (rank + 1), 5.0 - rank, 1.5], ready)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, vals))


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1] == [20.0, 5.0, 1.5]


def test_single_rank_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max([1.0, 2.0], False) == [1.0, 2.0]
    assert bench.init_dist(1, 0) is False


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0


def test_warmup_floor():
    sys.path.insert(0, ROOT)
    import bench
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "1"])


def test_algorithmic_work_kimi():
    sys.path.insert(0, ROOT)
    import bench
    from combine_top_route_counting_b200 import inputs
    w = inputs.WORKLOADS["kimi"]
    wk = bench.algorithmic_work(w, rows_used=492288, rows_real=w.n_routes)
    # 6 * routes * H * I flops over both GEMMs (real routes)
    assert wk["ffn_gemm1"]["flops"] + wk["ffn_gemm2"]["flops"] == 6 * w.n_routes * w.H * w.I
    assert abs(wk["ffn_gemm1"]["flops"] + wk["ffn_gemm2"]["flops"] - 4.04e13) / 4.04e13 < 0.01
    assert wk["dispatch"]["bytes"] == w.n_routes * w.H * 2 + 492288 * w.H * 2
