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


def test_assembled_line_meets_the_contract():
    """The JSON line bench.py prints, assembled from synthetic measurements of
    every leg: the contract's keys and types, throughput arithmetic, and both
    rooflines (so a slip in the post-processing cannot cost a GPU run's line)."""
    import argparse
    import json

    sys.path.insert(0, ROOT)
    import bench
    from combine_top_route_counting_b200 import inputs, moe

    args = argparse.Namespace(steps=20, warmup=3, e2e_steps=20, bwd_steps=10)
    w = inputs.WORKLOADS["kimi"]
    stage_ms = dict(zip(moe.STAGES, (0.065, 0.053, 2.39, 21.6, 13.4, 2.21)))
    bwd = dict(train_ms=1232.0, bwd_ms=79.8, launches=160,
               stages=dict(zip(moe.BWD_STAGES, (2.45, 13.25, 23.79, 2.22, 0.063, 12.68, 25.38))))
    e2e = dict(ms=830.0, h2d=910163968, d2h=822083584, chk=0.0)
    mx = dict(ms=1.94, rows=492544)
    peaks = bench.load_peaks()
    line = bench.assemble_line(args, w, 1, 794.0, stage_ms, 180, e2e, 0, 0, 1188.0, mx, bwd,
                               492544, peaks)
    line = json.loads(json.dumps(line))
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches"):
        assert key in line, key
    assert line["value"] == pytest.approx(w.n_tokens * 20 / 0.794)
    assert line["ms_per_step"] == pytest.approx(39.7)
    assert line["config"]["workload"].startswith("kimi")
    r = line["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(2 * w.n_routes * w.H * 2 * w.I / 21.6e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["peak"] == peaks["bf16"]                                     # led by the burst peak
    assert r["frac_sustained"] == pytest.approx(r["achieved"] / peaks["bf16_sus"])
    assert line["stages"]["ffn_gemm2"]["frac_bf16_burst"] < line["stages"]["ffn_gemm2"]["frac_bf16"]
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert line["e2e"]["value"] == pytest.approx(w.n_tokens * 20 / 0.830)
    b = line["backward"]
    assert b["roofline"]["kernel"] == "wgrad_w13" and b["roofline"]["bound"] == "tensor"
    assert b["value"] == pytest.approx(w.n_tokens / 0.0798)
    assert line["mxfp8"]["dispatch_mxfp8"]["frac_hbm"] > 0
    assert line["phi_build_us"] == pytest.approx(53.0)


def test_assembled_line_reports_the_mxfp8_layer_leg():
    """The opt-in MXFP8 layer leg: throughput, and the GEMMs against the fp8
    peak (twice the measured sustained bf16 peak), the dispatch against HBM."""
    import argparse

    sys.path.insert(0, ROOT)
    import bench
    from combine_top_route_counting_b200 import inputs, moe

    args = argparse.Namespace(steps=10, warmup=3, e2e_steps=10, bwd_steps=10)
    w = inputs.WORKLOADS["kimi"]
    stage_ms = dict(zip(moe.STAGES, (0.065, 0.053, 2.39, 21.6, 13.4, 2.21)))
    mxl = dict(ms=250.0, stage_ms=dict(zip(moe.STAGES, (0.065, 0.053, 1.94, 11.0, 7.0, 2.21))))
    peaks = bench.load_peaks()
    line = bench.assemble_line(args, w, 1, 397.0, stage_ms, 90, None, 0, 0, None, None, None,
                               492544, peaks, mxl=mxl)
    m = line["mxfp8_layer"]
    assert m["value"] == pytest.approx(w.n_tokens * 10 / 0.250)
    assert m["ms_per_step"] == pytest.approx(25.0)
    g1 = m["stages"]["ffn_gemm1"]
    assert g1["tflops"] == pytest.approx(2 * w.n_routes * w.H * 2 * w.I / 11.0e-3 / 1e12)
    assert g1["frac_fp8"] == pytest.approx(g1["tflops"] / (2 * peaks["bf16_sus"]))
    d = m["stages"]["dispatch"]
    assert d["bytes"] == w.n_routes * w.H * 2 + 492544 * (w.H + w.H // 32)
    assert "mxfp8_layer" not in bench.assemble_line(args, w, 1, 397.0, stage_ms, 90, None, 0, 0,
                                                    None, None, None, 492544, peaks)


def _fake_tree(root, sources):
    csrc = root / "combine_top_route_counting_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, text in sources.items():
        (csrc / name).write_text(text)
    (root / "profiles").mkdir()


def test_recorded_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    """A committed DRAM-traffic record reaches the bench line only while the
    kernel sources hash to the value it was taken with: comments and blank
    lines do not count, any code change does; the bytes scale by routes."""
    sys.path.insert(0, ROOT)
    import bench
    files = ("a.cu", "b.cuh")
    _fake_tree(tmp_path, {"a.cu": "int f() { return 1; }  // one\n", "b.cuh": "/* hdr */\nint g;\n"})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash(files)
    assert bench._recorded_traffic("t.txt", files, 10) is None  # no record
    (tmp_path / "profiles" / "t.txt").write_text(
        f"# comment: ignored\nkernel_source_sha256: {h}\ndram_bytes_per_route: 2.5\n")
    assert bench._recorded_traffic("t.txt", files, 10) == 25.0
    # comments and blank lines leave the hash and the record valid
    (tmp_path / "combine_top_route_counting_b200" / "csrc" / "a.cu").write_text(
        "// new comment\n\nint f() { return 1; }  // other\n")
    assert bench.kernel_source_hash(files) == h
    assert bench._recorded_traffic("t.txt", files, 4) == 10.0
    # a code change invalidates it
    (tmp_path / "combine_top_route_counting_b200" / "csrc" / "a.cu").write_text(
        "int f() { return 2; }\n")
    assert bench.kernel_source_hash(files) != h
    assert bench._recorded_traffic("t.txt", files, 10) is None


def test_committed_traffic_records_parse():
    """The committed GEMM1 and dW1|dW3 records carry a hash and a per-route
    byte figure in the form bench.py reads."""
    for name in ("ffn_gemm1_traffic.txt", "ffn_wgrad13_traffic.txt"):
        kv = {}
        for ln in open(os.path.join(ROOT, "profiles", name)):
            if ":" in ln and not ln.startswith("#"):
                a, b = ln.split(":", 1)
                kv[a.strip()] = b.strip()
        assert len(kv["kernel_source_sha256"]) == 64
        assert float(kv["dram_bytes_per_route"]) > 0
