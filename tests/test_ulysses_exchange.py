"""The head <-> sequence exchange of the sequence-parallel block between real
processes (gloo, world size 2 and 4, CPU tensors): after seq_to_heads every
rank holds every row of its heads in packed order; heads_to_seq gives each rank
its rows of every head, in head order; the two are inverse to each other."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from audio_generation_b200.ulysses import heads_to_seq, seq_to_heads


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        NH, S, D = 4 * world, 6 * world, 3
        full = torch.arange(NH * S * D, dtype=torch.float32).view(NH, S, D)  # [heads, rows, D]
        Sr, NHl = S // world, NH // world
        mine = full[:, rank * Sr:(rank + 1) * Sr].clone()
        a2a = lambda out, inp: dist.all_to_all_single(out, inp)
        got = seq_to_heads(mine, world, a2a)
        ok1 = torch.equal(got, full[rank * NHl:(rank + 1) * NHl])
        # o [S, NHl * D] of this rank's heads -> this rank's rows of every head
        o_heads = full[rank * NHl:(rank + 1) * NHl].permute(1, 0, 2).reshape(S, NHl * D)
        back = heads_to_seq(o_heads, world, a2a)
        want = full[:, rank * Sr:(rank + 1) * Sr].permute(1, 0, 2).reshape(Sr, NH * D)
        ok2 = torch.equal(back, want)
        q.put((rank, bool(ok1), bool(ok2)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_between_processes(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert res == [(r, True, True) for r in range(world)]


def test_fused_exchange_receive_areas_and_peer_table():
    """Host side of the fused exchange: the receive areas hold q, k, v and o at
    256-byte aligned offsets with the right sizes, and make_peers lays out one
    destination per rank (raw addresses accepted) and rejects more than 8."""
    from audio_generation_b200 import h3
    from audio_generation_b200.ulysses import receive_offsets, receive_shapes
    from workloads import FULL_DIMS

    S, P = 16384, 8
    shapes = receive_shapes(FULL_DIMS, S, P)
    assert shapes == [(7, S, 128)] * 3 + [(S // 8, 7168)]
    offs, size = receive_offsets(FULL_DIMS, S, P)
    assert all(o % 256 == 0 for o in offs)
    sizes = [2 * int(np.prod(s)) for s in shapes]
    assert [b - a for a, b in zip(offs, offs[1:] + [size])] == sizes  # no gaps: all multiples of 256
    base = [0x7f0000000000 + j * (1 << 32) for j in range(P)]
    lists = [[b + o for b in base] for o in offs]
    p = h3.make_peers(3, *lists)
    assert p.n_ranks == 8 and p.rank == 3
    assert [p.q[j] for j in range(P)] == lists[0] and [p.o[j] for j in range(P)] == lists[3]
    with pytest.raises(ValueError):
        h3.make_peers(0, *[[1] * 9] * 4)


def test_symmetric_receive_buffers_address_arithmetic(monkeypatch):
    """symmetric_receive_buffers on a fake symmetric-memory backend (CPU): the
    views sit at the receive offsets of this rank's area, and every rank's peer
    addresses are its buffer base plus the area's offset in the allocation plus
    the view's offset."""
    import types
    import torch.distributed as dist
    from audio_generation_b200 import ulysses as U
    from workloads import Dims

    dims = Dims(hidden=256, heads=8, head_dim=128, ffn=384, time_embed_dim=64, time_hidden=128)
    S, P, rank = 64, 4, 2
    pool = torch.zeros(1 << 20, dtype=torch.uint8)
    lead = 512  # the area starts this far into the (fake) symmetric allocation

    def empty(size, dtype=None, device=None):
        return pool[lead:lead + size]

    bases = [0x10000000 * (j + 1) for j in range(P)]
    bases[rank] = pool.data_ptr()
    hdl = types.SimpleNamespace(buffer_ptrs=bases, rank=rank)
    fake = types.SimpleNamespace(empty=empty, rendezvous=lambda t, g: hdl)
    monkeypatch.setitem(__import__("sys").modules, "torch.distributed._symmetric_memory", fake)
    monkeypatch.setattr(dist, "get_world_size", lambda group=None: P)
    monkeypatch.setattr(dist, "group", types.SimpleNamespace(WORLD="world"), raising=False)
    views, lists, h = U.symmetric_receive_buffers(dims, S, group="g", device="cpu")
    offs, size = U.receive_offsets(dims, S, P)
    assert [tuple(v.shape) for v in views] == [tuple(s) for s in U.receive_shapes(dims, S, P)]
    for v, off in zip(views, offs):
        assert v.data_ptr() == pool.data_ptr() + lead + off
    for lst, off in zip(lists, offs):
        assert lst == [b + lead + off for b in bases]
