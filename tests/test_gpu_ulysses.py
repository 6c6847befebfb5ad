"""Sequence-parallel block (audio_generation_b200.ulysses) with P ranks emulated
on one GPU: each rank's row-local steps on its chunk of rows, attention on
NH / P heads over every row, and the head <-> sequence exchange done either by
copies between the ranks' buffers or fused into the producing kernels (the QKV
epilogue and the attention epilogue store into the owning rank's receive
buffer, here a buffer of the same GPU). Every output element is computed by the
same kernels in the same order as in the single-GPU block, so the result must be
bit-identical to h3_block_forward.
"""

import numpy as np
import pytest
import torch

from audio_generation_b200 import h3
from audio_generation_b200.ulysses import UlyssesBlock
from tests.h3_testlib import DevLayout, DevWeights, dev_bf16, host_bits
from tests.test_gpu_block import amplified_weights, gpu_tmod
from workloads import (FULL_DIMS, Dims, activations, block_weights, config_layout, make_layout,
                       normal_bf16, prologue_weights)

pytestmark = pytest.mark.gpu


def emulate(dims, L, w, tmod, xb, P):
    dev = torch.device("cuda", 0)
    dw = DevWeights(w)
    ranks = [UlyssesBlock(dims, L, r, P, dev) for r in range(P)]
    Sr, NHl = L.S // P, dims.heads // P
    xs = [dev_bf16(np.ascontiguousarray(xb[:, r * Sr:(r + 1) * Sr])) for r in range(P)]
    qkv = [rk.pre_attention(dw, tmod, x) for rk, x in zip(ranks, xs)]
    outs = []
    for j, rk in enumerate(ranks):  # rank j: every row of heads [j NHl, (j + 1) NHl)
        ql, kl, vl = (torch.cat([qkv[r][t][j * NHl:(j + 1) * NHl] for r in range(P)], dim=1)
                      for t in range(3))
        outs.append(rk.attention(ql, kl, vl).clone())
    for r, (rk, x) in enumerate(zip(ranks, xs)):  # rank r: its rows of every head group
        o = torch.cat([outs[j][r * Sr:(r + 1) * Sr] for j in range(P)], dim=1)
        rk.post_attention(dw, tmod, o, x)
    torch.cuda.synchronize()
    for rk in ranks:
        assert h3.h3_layout_error(rk.full) == h3.H3_OK
        rk.close()
    return np.concatenate([host_bits(x) for x in xs], axis=1)


def emulate_fused(dims, L, w, tmod, xb, P):
    """The fused exchange: every rank's stores go straight into the receive
    buffers of the ranks (all on this GPU); the phases run rank after rank, so
    every rank's stores are complete before any rank reads them."""
    dw = DevWeights(w)
    dev = torch.device("cuda", 0)
    ranks = [UlyssesBlock(dims, L, r, P, dev) for r in range(P)]
    Sr = L.S // P
    # fill the receive buffers with a marker: every element must be overwritten
    for rk in ranks:
        for t in rk.recv:
            t.fill_(float("nan"))
    recv = [rk.recv for rk in ranks]
    peers = [h3.make_peers(r, *[[recv[j][i] for j in range(P)] for i in range(4)])
             for r in range(P)]
    xs = [dev_bf16(np.ascontiguousarray(xb[:, r * Sr:(r + 1) * Sr])) for r in range(P)]
    for r, rk in enumerate(ranks):
        rk.pre_attention_to_heads(dw, tmod, xs[r], peers[r])
    for r, rk in enumerate(ranks):
        rk.attention_to_rows(peers[r])
    for r, rk in enumerate(ranks):
        rk.post_attention(dw, tmod, rk.recv[3][None], xs[r])
    torch.cuda.synchronize()
    for rk in ranks:
        assert h3.h3_layout_error(rk.full) == h3.H3_OK
        # every element of the receive buffers was stored by some rank
        assert not any(bool(torch.isnan(t).any()) for t in rk.recv)
        rk.close()
    return np.concatenate([host_bits(x) for x in xs], axis=1)


def reference(dims, L, w, tmod, xb):
    dl = DevLayout(dims, L)
    x = dev_bf16(xb)
    ws_b = h3.h3_workspace_size(dl.dims, 1, L.S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    h3.h3_block_forward(dl.dims, DevWeights(w).c, dl.handle, tmod, x, 1, ws, ws_b)
    torch.cuda.synchronize()
    return host_bits(x)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("P", [2, 4])
def test_ulysses_small_matches_the_block_bit_for_bit(P, fused):
    dims = Dims(hidden=256, heads=8, head_dim=128, ffn=384, time_embed_dim=64, time_hidden=128)
    segs = [("text", 0, 100), ("pad", 28), ("video", (2, 8, 16), 0, 2), ("audio", 0, 124)]
    L = make_layout(segs, seed=[31])
    assert L.S % P == 0
    w = amplified_weights(dims, 31)
    tm = torch.from_numpy((np.random.default_rng(32).standard_normal((L.n_t, 6, dims.hidden))
                           * 0.3).astype(np.float32)).cuda()
    xb = normal_bf16((1, L.S, dims.hidden), [33], 1.0)
    got = (emulate_fused if fused else emulate)(dims, L, w, tm, xb, P)
    ref = reference(dims, L, w, tm, xb)
    np.testing.assert_array_equal(got, ref)
    assert not np.array_equal(ref, xb)


@pytest.mark.parametrize("fused", [False, True])
def test_ulysses_full_width_eight_ranks_matches_the_block_bit_for_bit(fused):
    """56 heads over 8 ranks (7 heads each), the padded 16384-row layout."""
    dims = FULL_DIMS
    L = config_layout(3)
    w = block_weights(dims, 3, 0)
    pw = prologue_weights(dims, 3)
    tmod = gpu_tmod(dims, L.timestep, pw)
    xb = activations(dims, 3, L.S)
    got = (emulate_fused if fused else emulate)(dims, L, w, tmod, xb, 8)
    ref = reference(dims, L, w, tmod, xb)
    np.testing.assert_array_equal(got, ref)
