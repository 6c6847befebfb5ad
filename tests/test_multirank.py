"""The benchmark's multi-process plumbing on CPU: two gloo ranks, each timing
its own replica; the reported time is the maximum over ranks."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ws, r, local = bench.dist_env()
    bench.barrier(ws)
    t = bench.max_over_ranks(10.0 + 5.0 * rank, ws)
    bench.barrier(ws)
    q.put((r, ws, local, t))
    dist.destroy_process_group()


def test_two_ranks_report_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2, 0, 15.0), (1, 2, 1, 15.0)]


def test_single_process_defaults():
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_work_counts_match_the_stated_flops():
    from workloads import FULL_DIMS
    # per-row GEMM flops 770.7 M plus 4 * 56 * 128 flops per (query, key) pair
    f = bench.block_flops(FULL_DIMS, 8192)
    assert abs(f - (2 * 8192 * (5376 * 21504 + 7168 * 5376 + 5376 * 28672 + 14336 * 5376)
                    + 4 * 56 * 128 * 8192 ** 2)) < 1
    assert abs(f / 1e12 - 8.238) < 0.01


def test_recorded_traffic_is_used_only_for_the_recorded_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu summary of the bench's
    workload, and only while the kernel's source file still hashes to the
    recorded SHA-256."""
    import hashlib
    src = tmp_path / "k.cu"
    src.write_text("// a kernel\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles").mkdir()
    rec = tmp_path / "profiles" / "dram_traffic_config4.txt"
    rec.write_text(f"# comment line\nattention {digest} 123456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "attention", "k.cu")
    (tmp_path / "audio_generation_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "audio_generation_b200" / "csrc" / "k.cu").write_bytes(src.read_bytes())
    assert bench.measured_traffic("attention") == 123456.0
    assert bench.measured_traffic("attention", 4) == 123456.0
    assert bench.measured_traffic("attention", 3) is None  # no record for that workload
    (tmp_path / "audio_generation_b200" / "csrc" / "k.cu").write_text("// changed\n")
    assert bench.measured_traffic("attention") is None


def test_algorithmic_bytes_per_kernel():
    from workloads import FULL_DIMS
    b = bench.kernel_bytes(FULL_DIMS, 8192)
    H, A, F, V = 5376, 7168, 14336, 8192
    assert b["attention"] == 4 * V * A * 2
    assert b["ffn_up"] == V * H * 2 + 2 * F * H * 2 + V * F * 2
    assert b["norm_modulate_1"] == V * 12 * H
