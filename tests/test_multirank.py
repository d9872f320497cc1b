"""bench.py's replica mode on CPU with world size 2 over gloo: every rank
joins the barrier, the step time is the maximum over ranks and the reported
throughput counts the work of all ranks (weak scaling)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_setup(None)
    bench.barrier(w)
    elapsed = bench.max_over_ranks(10.0 * (r + 1), w)  # rank 1 is the slower one
    value = bench.aggregate_throughput(1.0e12, w, elapsed)
    q.put((r, w, elapsed, value))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_replicas_take_max_time_and_sum_work():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for r, w, elapsed, value in res:
        assert w == world
        assert elapsed == 20.0
        # 2 ranks x 1 TFLOP in 20 ms per step -> 100 TFLOPS
        assert abs(value - 100.0) < 1e-9


def test_gemm_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    """The captured DRAM traffic is reported only while the GEMM sources
    hash as captured: comment and whitespace edits keep the hash, any code
    edit changes it."""
    import bench
    src = tmp_path / "k.cuh"
    src.write_text("// a kernel\n__global__ void k(int *p) { p[0] = 1; /* store */ }\n")
    monkeypatch.setattr(bench, "GEMM_SOURCES", [str(src)])
    h0 = bench.gemm_source_hash()
    src.write_text("// the kernel, reworded\n__global__   void k(int *p)\n{ p[0] = 1; /* one store */ }\n")
    assert bench.gemm_source_hash() == h0
    src.write_text("// a kernel\n__global__ void k(int *p) { p[0] = 2; /* store */ }\n")
    assert bench.gemm_source_hash() != h0
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", {"source_sha256_12": h0, "bytes_per_launch": 1.0})
    assert bench.gemm_traffic() is None


def test_gemm_source_hash_covers_the_launch_code(tmp_path, monkeypatch):
    """The hash also covers the host functions that choose the GEMM's tile
    order, grid and tensor-map boxes (run_gemm and the tensor-map builders in
    nvfp4_api.cu): a change there invalidates the captured traffic, a change
    elsewhere in that file does not."""
    import bench
    entries = {os.path.basename(p): f for p, f in bench.GEMM_SOURCES}
    assert {"gemm_kernel.cuh", "gemm_pair_kernel.cuh", "ptx_sm100.cuh", "nvfp4_api.cu"} <= set(entries)
    assert "run_gemm" in entries["nvfp4_api.cu"]
    assert all(os.path.exists(p) for p, _ in bench.GEMM_SOURCES)
    src = tmp_path / "api.cu"
    body = ("int other(int a)\n{\n    return a + 1;\n}\n\n"
            "int run_gemm(int m, int n)\n{\n    const int grid = m * n;\n    return grid;\n}\n")
    src.write_text(body)
    monkeypatch.setattr(bench, "GEMM_SOURCES", [(str(src), ("run_gemm",))])
    h0 = bench.gemm_source_hash()
    src.write_text(body.replace("a + 1", "a + 2"))
    assert bench.gemm_source_hash() == h0
    src.write_text(body.replace("m * n", "m * n + 1"))
    assert bench.gemm_source_hash() != h0
