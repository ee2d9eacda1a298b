"""bench.py host logic on CPU: max-over-ranks timing with two gloo ranks, the
reference (oracle) arm's JSON line, and the work counts the roofline uses."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    v = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
    out[rank] = v
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == 15.0 and out[1] == 15.0


def test_max_over_ranks_single():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, None) == 3.5


def test_reference_arm_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "steps/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_work_counts():
    sys.path.insert(0, ROOT)
    import bench
    g = bench.WORKLOADS["mamba2-130m"]
    assert bench.ns_flops(g) == 1146617856000
    assert bench.elements(g) == 24 * 768 * 1536 + 24 * 3352 * 768
    assert bench.momentum_bytes(g) == 12 * bench.elements(g)


def test_kernel_hash_ignores_comments_but_not_code():
    import bench
    a = "int x = 1; // one\n/* block\ncomment */\n\nint y = 2;\n"
    b = "int x = 1;   // a different note\n\nint y = 2;  \n"
    c = "int x = 3; // one\nint y = 2;\n"
    assert bench._code_only(a) == bench._code_only(b) == "int x = 1;\nint y = 2;"
    assert bench._code_only(c) != bench._code_only(a)
    assert len(bench.gemm_source_hash()) == 16


def test_cpu_baseline_reports_blas_and_a_one_thread_figure():
    import bench
    assert bench.blas_vendor() != ""
    t = bench.oracle_one_thread_seconds([("small", 2, 96, 160)])
    assert 0.0 < t < 30.0
