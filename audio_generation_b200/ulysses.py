"""Sequence-parallel block forward: rows split across ranks, heads across ranks
for attention (a head <-> sequence all-to-all before and after it).

The batch axis of the transformer is a pure replication axis ("MiniMaxH3Transformer3DModel"
page, `forward`: every batch element is one attention document over one packed
sequence), so one long sequence is the unit that needs more than one GPU. Every
step of the block except attention is row-local (norm + modulate, QKV + QK-norm
+ RoPE, the output projection and the FFN with their residuals), so each rank
runs those on its own contiguous chunk of S / P rows. Attention needs every row
but is independent per head: an all-to-all turns "my rows, all heads" into "all
rows, my NH / P heads" for q, k and v, each rank runs the attention kernel on
its heads over the whole sequence (with the full layout, so the padding
document is the same), and a second all-to-all turns the output back into "my
rows, all heads".

Every step runs in this library's kernels through the C ABI; this module only
allocates, reshapes and exchanges buffers. Two forms of the exchange:

* fused (``forward_fused``): the QKV kernel's epilogue stores each head's rows
  straight into the receive buffer of the rank that owns the head
  (h3_qkv_rope_to_heads), and the attention kernel stores each row's output
  straight into the receive buffer of the rank that owns the row
  (h3_attention_to_rows). The receive buffers are this GPU's or peers' memory
  (``symmetric_receive_buffers`` maps them through torch's symmetric memory);
  the ranks only synchronise between the phases (``barrier``). No copy or
  collective runs on the data path.
* through a callable ``all_to_all(out, inp)`` that splits dim 0 of ``inp``
  evenly across ranks, as ``torch.distributed.all_to_all_single`` (NCCL) does
  (``forward``).

The stages of :class:`UlyssesBlock` are public so that a caller that holds every
rank's buffers (one process, one GPU) can run the ranks in turn.

Requirements: S % P == 0, heads % P == 0 and P <= 8 for the fused form.
"""

from __future__ import annotations

from typing import Callable, Optional

import numpy as np
import torch

from . import h3


def seq_to_heads(t: torch.Tensor, world: int, all_to_all: Callable) -> torch.Tensor:
    """[NH, Sr, D] (this rank's rows, every head) -> [NH / P, P * Sr, D] (every
    row, this rank's heads; rows in rank order, i.e. packed order)."""
    NH, Sr, D = t.shape
    inp = t.contiguous()
    out = torch.empty_like(inp)
    all_to_all(out, inp)  # out[j] = rank j's rows of this rank's heads
    return out.view(world, NH // world, Sr, D).transpose(0, 1).reshape(NH // world, world * Sr, D)


def heads_to_seq(o: torch.Tensor, world: int, all_to_all: Callable) -> torch.Tensor:
    """[S, NHl * D] (every row, this rank's heads) -> [S / P, P * NHl * D] (this
    rank's rows, every head in head order)."""
    S, W = o.shape
    Sr = S // world
    inp = o.contiguous()
    out = torch.empty_like(inp)
    all_to_all(out, inp)  # out[j] = head group j of this rank's rows
    return out.view(world, Sr, W).transpose(0, 1).reshape(Sr, world * W)


def _device_layout(dims_c, tags, pos, t_idx, n_t, device):
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    keep = [i32(np.nonzero(tags == m)[0]) for m in (0, 2, 1)]
    lay = h3.h3_layout_prepare(dims_c, len(tags), n_t, f32(pos.reshape(-1, 3)), i32(tags),
                               i32(t_idx), *keep)
    return lay


class UlyssesBlock:
    """One rank's part of the block over a packed sequence split into P chunks.

    ``layout`` is the whole sequence's host layout (tags, pos, t_idx, timestep
    arrays); ``weights`` has the block's device tensors (w_qkv, q_norm, k_norm,
    w_o, w13, w2, ada_table) and ``tmod`` is the shared [n_t, 6, H] modulation.
    """

    def __init__(self, dims, layout, rank: int, world: int, device,
                 all_to_all: Optional[Callable] = None, receive=None):
        S, NH = layout.S, dims.heads
        if S % world or NH % world:
            raise ValueError("the sequence length and the head count must divide by the ranks")
        self.dims, self.rank, self.world, self.device = dims, rank, world, device
        self.all_to_all = all_to_all
        self.d = h3.make_dims(dims)
        self.Sr = S // world
        self.NHl = NH // world
        # attention over every row for NH / P heads: same dims with fewer heads
        self.d_local = h3.make_dims(dims)
        self.d_local.heads = self.NHl
        tags, pos, t_idx = (np.asarray(a) for a in (layout.tags, layout.pos, layout.t_idx))
        self.full = _device_layout(self.d, tags, pos, t_idx, layout.n_t, device)
        r0, r1 = rank * self.Sr, (rank + 1) * self.Sr
        self.chunk = _device_layout(self.d, tags[r0:r1], pos[r0:r1], t_idx[r0:r1], layout.n_t,
                                    device)
        H, A, F, D = dims.hidden, dims.attn_width, dims.ffn, dims.head_dim
        bf = lambda *sh: torch.empty(sh, dtype=torch.bfloat16, device=device)
        self.h = bf(1, self.Sr, H)
        self.q, self.k, self.v = bf(1, NH, self.Sr, D), bf(1, NH, self.Sr, D), bf(1, NH, self.Sr, D)
        self.ol = bf(1, S, self.NHl * D)
        self.g = bf(1, self.Sr, F)
        # receive buffers of the fused exchange: q, k, v [NH / P, S, D] (every
        # row of this rank's heads) and o [S / P, NH D] (this rank's rows)
        if receive is None:
            receive = (bf(self.NHl, S, D), bf(self.NHl, S, D), bf(self.NHl, S, D),
                       bf(self.Sr, NH * D))
        self.recv = receive

    def pre_attention(self, w, tmod, x):
        """norm1 + modulate and QKV + QK-norm + RoPE on this rank's rows: x [1, Sr, H]."""
        h3.h3_norm_modulate(self.d, self.chunk, 1, 0, x, w.ada_table, tmod, self.h)
        h3.h3_qkv_rope(self.d, self.chunk, 1, self.h, w.w_qkv, w.q_norm, w.k_norm, self.q, self.k,
                       self.v)
        return self.q[0], self.k[0], self.v[0]

    def attention(self, ql, kl, vl):
        """Attention of this rank's NH / P heads over every row: [NHl, S, D] -> [S, NHl D]."""
        h3.h3_attention(self.d_local, self.full, 1, ql[None], kl[None], vl[None], self.ol)
        return self.ol[0]

    def post_attention(self, w, tmod, o, x):
        """Output projection + gated residual, norm2 + modulate, FFN + gated residual on
        this rank's rows: o [Sr, NH D], x [1, Sr, H] updated in place."""
        h3.h3_out_residual(self.d, self.chunk, 1, o[None], w.w_o, w.ada_table, tmod, x)
        h3.h3_norm_modulate(self.d, self.chunk, 1, 1, x, w.ada_table, tmod, self.h)
        h3.h3_ffn_up(self.d, self.chunk, 1, self.h, w.w13, self.g)
        h3.h3_ffn_down_residual(self.d, self.chunk, 1, self.g, w.w2, w.ada_table, tmod, x)

    def pre_attention_to_heads(self, w, tmod, x, peers):
        """norm1 + modulate on this rank's rows, then QKV + QK-norm + RoPE with
        every head's rows stored into its owner's receive buffer."""
        h3.h3_norm_modulate(self.d, self.chunk, 1, 0, x, w.ada_table, tmod, self.h)
        h3.h3_qkv_rope_to_heads(self.d, self.chunk, self.h, w.w_qkv, w.q_norm, w.k_norm, peers)

    def attention_to_rows(self, peers):
        """Attention of this rank's heads over every row (its receive buffers),
        every row's output stored into its owner's receive buffer."""
        q, k, v, _ = self.recv
        h3.h3_attention_to_rows(self.d, self.full, q, k, v, peers)

    def forward_fused(self, w, tmod, x, peers, barrier: Callable):
        """The whole block with the fused exchange; ``barrier()`` orders the
        phases across ranks (every rank's stores complete before any rank reads
        them)."""
        self.pre_attention_to_heads(w, tmod, x, peers)
        barrier()
        self.attention_to_rows(peers)
        barrier()
        self.post_attention(w, tmod, self.recv[3][None], x)

    def forward(self, w, tmod, x):
        """The whole block on this rank's rows, exchanging with the other ranks."""
        if self.all_to_all is None:
            raise ValueError("forward needs an all_to_all exchange")
        q, k, v = self.pre_attention(w, tmod, x)
        ql, kl, vl = (seq_to_heads(t, self.world, self.all_to_all) for t in (q, k, v))
        o = heads_to_seq(self.attention(ql, kl, vl), self.world, self.all_to_all)
        self.post_attention(w, tmod, o, x)

    def close(self):
        self.full.close()
        self.chunk.close()


def receive_shapes(dims, S: int, world: int):
    """Shapes of one rank's q, k, v and o receive buffers (bf16)."""
    NHl, D = dims.heads // world, dims.head_dim
    return [(NHl, S, D)] * 3 + [(S // world, dims.heads * D)]


def receive_offsets(dims, S: int, world: int):
    """Byte offsets of q, k, v and o inside one rank's receive area, each
    256-byte aligned, and the area's size."""
    offs, at = [], 0
    for shp in receive_shapes(dims, S, world):
        offs.append(at)
        n = 2
        for d in shp:
            n *= d
        at += (n + 255) // 256 * 256
    return offs, at


def symmetric_receive_buffers(dims, S: int, group=None, device=None):
    """Receive buffers in torch's symmetric memory, one area per rank at the
    same offsets: returns (this rank's q, k, v, o views, the peers of every
    rank's areas as lists of addresses (q, k, v, o), the handle)."""
    import torch.distributed as dist
    import torch.distributed._symmetric_memory as symm_mem

    world = dist.get_world_size(group)
    offs, size = receive_offsets(dims, S, world)
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    area = symm_mem.empty(size, dtype=torch.uint8, device=device)
    hdl = symm_mem.rendezvous(area, group if group is not None else dist.group.WORLD)
    views = []
    for off, shp in zip(offs, receive_shapes(dims, S, world)):
        n = 1
        for d in shp:
            n *= d
        views.append(area[off:off + 2 * n].view(torch.bfloat16).view(*shp))
    ptrs = [int(p) for p in hdl.buffer_ptrs]
    # the area may sit at an offset inside the symmetric allocation: the same
    # offset on every rank
    base = area.data_ptr() - ptrs[hdl.rank]
    lists = [[p + base + off for p in ptrs] for off in offs]
    return tuple(views), lists, hdl


def host_barrier(group=None) -> Callable:
    """Phase barrier between ranks: this GPU's work done, then the ranks meet."""
    import torch.distributed as dist

    def barrier():
        torch.cuda.current_stream().synchronize()
        dist.barrier(group=group)
    return barrier


def nccl_all_to_all(group=None) -> Callable:
    """The exchange between GPUs: torch.distributed.all_to_all_single (NCCL)."""
    import torch.distributed as dist

    def a2a(out, inp):
        dist.all_to_all_single(out, inp, group=group)
    return a2a
