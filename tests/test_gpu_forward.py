"""The whole transformer forward (h3_forward) on the GPU against the float64
oracle's denoiser_forward: input projections, text refiner, block stack,
norm_out and the two heads; velocities compared element by element
(rel-L2 <= 1e-2, max-abs <= 5e-2), in the order of the index tensors.

Source: "MiniMaxH3Transformer3DModel" (diffusers v0.43.0 docs), constructor
parameters in_channels, audio_in_channels, patch_size, text_dim,
num_refiner_layers, final_norm_eps, the mixed-precision note, and `forward`.
"""

from types import SimpleNamespace

import numpy as np
import pytest
import torch

from audio_generation_b200 import h3
from oracle import h3_oracle as O
from tests.h3_testlib import DevLayout, DevWeights, assert_close, dev_bf16, dev_f32, rel_l2
from tests.test_gpu_block import amplified_weights
from workloads import (FULL_DIMS, TINY_DIMS, Dims, block_weights, config_layout, denoiser_inputs,
                       denoiser_weights, f32_to_bf16_bits, make_layout, random_layout)

pytestmark = pytest.mark.gpu


def gpu_forward(dims, L, dw, blocks, video, audio, text, B):
    dl = DevLayout(dims, L)
    io = h3.make_io_dims(dims)
    keep = [dev_f32(dw.w_patch_video), dev_f32(dw.w_patch_audio), dev_bf16(dw.w_text),
            dev_f32(dw.w_t1), dev_f32(dw.w_t2), dev_f32(dw.w_proj), dev_f32(dw.w_out),
            dev_f32(dw.out_table), dev_f32(dw.w_head_video), dev_f32(dw.w_head_audio)]
    iw = h3.make_io_weights(*keep)
    ref = [DevWeights(w) for w in dw.refiner]
    blk = [DevWeights(w) for w in blocks]
    vo = torch.full((B, len(L.video_idx), dims.video_channels), float("nan"), device="cuda")
    ao = torch.full((B, len(L.audio_idx), dims.audio_in_channels), float("nan"), device="cuda")
    ws_b = h3.h3_forward_workspace_size(dl.dims, io, dl.handle, B)
    assert ws_b > 0
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    h3.h3_forward(dl.dims, io, iw, [w.c for w in ref], [w.c for w in blk], dl.handle,
                  dev_f32(L.timestep), B, dev_f32(video), dev_f32(audio), dev_bf16(text), vo, ao,
                  ws, ws_b)
    torch.cuda.synchronize()
    assert h3.h3_layout_error(dl.handle) == h3.H3_OK
    return vo.double().cpu().numpy(), ao.double().cpu().numpy()


def oracle_forward(dims, L, dw, blocks, video, audio, text, b=0):
    return O.denoiser_forward(video[b], audio[b], text[b], dw, lambda i: blocks[i], len(blocks),
                              L, dims, dims.final_norm_eps)


def _check(got, ref, what):
    assert np.all(np.isfinite(got)), what
    assert_close(got, ref, what=what)


def test_forward_tiny_workload():
    dims = TINY_DIMS
    L = config_layout(1)
    dw = denoiser_weights(dims, 1)
    blocks = [block_weights(dims, 1, i) for i in range(3)]
    video, audio, text = denoiser_inputs(dims, 1, L)
    vo, ao = gpu_forward(dims, L, dw, blocks, video, audio, text, 1)
    rv, ra = oracle_forward(dims, L, dw, blocks, video, audio, text)
    _check(vo[0], rv, "video velocity")
    _check(ao[0], ra, "audio velocity")


def _amplified_case(seed, S, dims, n_blocks=2, pad_runs=2, text=True):
    L = random_layout(S, seed, pad_runs=pad_runs, max_run=40, n_t=3)
    if not text:  # no text rows: relabel them as audio
        tags = np.where(L.tags == 1, 2, L.tags).astype(np.int32)
        L = type(L)(tags=tags, pos=L.pos, t_idx=L.t_idx, timestep=L.timestep,
                    video_idx=np.nonzero(tags == 0)[0].astype(np.int32),
                    audio_idx=np.nonzero(tags == 2)[0].astype(np.int32),
                    text_idx=np.zeros(0, np.int32))
    g = np.random.default_rng([seed, 88])
    H, E = dims.hidden, dims.time_embed_dim
    dw = SimpleNamespace(
        w_patch_video=(g.standard_normal((H, dims.video_channels)) * 0.1).astype(np.float32),
        w_patch_audio=(g.standard_normal((H, dims.audio_in_channels)) * 0.1).astype(np.float32),
        w_text=f32_to_bf16_bits((g.standard_normal((H, dims.text_dim)) * 0.05).astype(np.float32)),
        refiner=[amplified_weights(dims, 500 + seed * 10 + i, std=0.05, table_std=0.2)
                 for i in range(2)],
        w_t1=(g.standard_normal((dims.time_hidden, dims.freq_dim)) * 0.05).astype(np.float32),
        w_t2=(g.standard_normal((E, dims.time_hidden)) * 0.05).astype(np.float32),
        w_proj=(g.standard_normal((6 * H, E)) * 0.05).astype(np.float32),
        w_out=(g.standard_normal((2 * H, E)) * 0.05).astype(np.float32),
        out_table=(g.standard_normal((2, 2, H)) * 0.2).astype(np.float32),
        w_head_video=(g.standard_normal((dims.video_channels, H)) * 0.05).astype(np.float32),
        w_head_audio=(g.standard_normal((dims.audio_in_channels, H)) * 0.05).astype(np.float32))
    blocks = [amplified_weights(dims, 600 + seed * 10 + i, std=0.05, table_std=0.2)
              for i in range(n_blocks)]
    return L, dw, blocks


@pytest.mark.parametrize("S,seed,B,text", [(300, 1, 2, True), (97, 2, 1, True),
                                           (200, 3, 1, False)])
def test_forward_small_amplified(S, seed, B, text):
    """Small widths with weights large enough that the refiner and the blocks
    move the stream far beyond bf16 resolution, on ragged layouts with padding;
    B = 2 checks the batch replicas, one case has no text rows."""
    dims = Dims(hidden=256, heads=2, head_dim=128, ffn=384, time_embed_dim=64, time_hidden=128,
                text_dim=128, in_channels=8, audio_in_channels=64)
    L, dw, blocks = _amplified_case(seed, S, dims, text=text)
    g = np.random.default_rng([seed, 89])
    video = g.standard_normal((B, len(L.video_idx), dims.video_channels)).astype(np.float32)
    audio = g.standard_normal((B, len(L.audio_idx), dims.audio_in_channels)).astype(np.float32)
    txt = f32_to_bf16_bits(g.standard_normal((B, len(L.text_idx), dims.text_dim)).astype(np.float32))
    vo, ao = gpu_forward(dims, L, dw, blocks, video, audio, txt, B)
    for b in range(B):
        rv, ra = oracle_forward(dims, L, dw, blocks, video, audio, txt, b)
        _check(vo[b], rv, f"video velocity b={b}")
        _check(ao[b], ra, f"audio velocity b={b}")
        # the stack matters: without its blocks the velocities differ far
        # beyond the tolerance
        r0v, _ = O.denoiser_forward(video[b], audio[b], txt[b], dw, lambda i: blocks[i], 0, L,
                                    dims, dims.final_norm_eps)
        assert rel_l2(r0v, rv) > 0.1


def test_forward_full_width_ragged():
    """Full constructor widths (hidden 5376, text_dim 5120, 96 / 32 latent
    channels) on a 1500-row layout with padding runs, two refiner blocks and two
    stack blocks."""
    dims = FULL_DIMS
    segs = [("text", 0, 200), ("pad", 37), ("video", (3, 8, 16), 0, 3), ("pad", 100),
            ("audio", 0, 500), ("pad", 279)]
    L = make_layout(segs, seed=[77])
    assert L.S == 1500
    dw = denoiser_weights(dims, 7)
    blocks = [block_weights(dims, 7, i) for i in range(2)]
    video, audio, text = denoiser_inputs(dims, 7, L)
    vo, ao = gpu_forward(dims, L, dw, blocks, video, audio, text, 1)
    rv, ra = oracle_forward(dims, L, dw, blocks, video, audio, text)
    _check(vo[0], rv, "full-width video velocity")
    _check(ao[0], ra, "full-width audio velocity")


def test_forward_core_residual_store_and_reuse():
    """H3_CORE_STORE gives the plain forward's velocities and the stack's
    residual (output minus input, valid rows in packed order); H3_CORE_REUSE with
    fresh latents matches the oracle's reuse of that residual."""
    dims = Dims(hidden=256, heads=2, head_dim=128, ffn=384, time_embed_dim=64, time_hidden=128,
                text_dim=128, in_channels=8, audio_in_channels=64)
    L, dw, blocks = _amplified_case(4, 250, dims)
    g = np.random.default_rng(90)
    video = g.standard_normal((1, len(L.video_idx), dims.video_channels)).astype(np.float32)
    audio = g.standard_normal((1, len(L.audio_idx), dims.audio_in_channels)).astype(np.float32)
    txt = f32_to_bf16_bits(g.standard_normal((1, len(L.text_idx), dims.text_dim)).astype(np.float32))
    dl = DevLayout(dims, L)
    io = h3.make_io_dims(dims)
    keep = [dev_f32(dw.w_patch_video), dev_f32(dw.w_patch_audio), dev_bf16(dw.w_text),
            dev_f32(dw.w_t1), dev_f32(dw.w_t2), dev_f32(dw.w_proj), dev_f32(dw.w_out),
            dev_f32(dw.out_table), dev_f32(dw.w_head_video), dev_f32(dw.w_head_audio)]
    iw = h3.make_io_weights(*keep)
    ref = [DevWeights(w) for w in dw.refiner]
    blk = [DevWeights(w) for w in blocks]
    V = L.n_valid
    res = torch.zeros((1, V, dims.hidden), device="cuda")
    ws_b = h3.h3_forward_workspace_size(dl.dims, io, dl.handle, 1)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")

    def run(v, a, mode):
        vo = torch.empty((1, len(L.video_idx), dims.video_channels), device="cuda")
        ao = torch.empty((1, len(L.audio_idx), dims.audio_in_channels), device="cuda")
        h3.h3_forward(dl.dims, io, iw, [w.c for w in ref], [w.c for w in blk], dl.handle,
                      dev_f32(L.timestep), 1, dev_f32(v), dev_f32(a), dev_bf16(txt), vo, ao, ws,
                      ws_b, core_residual=res, core_mode=mode)
        torch.cuda.synchronize()
        assert h3.h3_layout_error(dl.handle) == h3.H3_OK
        return vo.double().cpu().numpy()[0], ao.double().cpu().numpy()[0]

    v_run, a_run = run(video, audio, h3.H3_CORE_RUN)
    v_st, a_st = run(video, audio, h3.H3_CORE_STORE)
    np.testing.assert_array_equal(v_st, v_run)
    np.testing.assert_array_equal(a_st, a_run)
    ores = np.zeros((L.S, dims.hidden))
    O.denoiser_forward(video[0], audio[0], txt[0], dw, lambda i: blocks[i], len(blocks), L, dims,
                       dims.final_norm_eps, core_residual=ores)
    valid = np.nonzero(L.tags >= 0)[0]
    _check(res.double().cpu().numpy()[0], ores[valid], "core residual")
    v2 = (video * 0.5 + 0.2).astype(np.float32)
    a2 = (audio * -0.7).astype(np.float32)
    v_re, a_re = run(v2, a2, h3.H3_CORE_REUSE)
    rv, ra = O.denoiser_forward(v2[0], a2[0], txt[0], dw, lambda i: blocks[i], len(blocks), L,
                                dims, dims.final_norm_eps, core_residual=ores, reuse=True)
    _check(v_re, rv, "reused video velocity")
    _check(a_re, ra, "reused audio velocity")
