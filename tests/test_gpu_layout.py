"""a0 / a1 on the GPU: layout tables and packed-row gather / scatter are
bit-exact against the oracle."""

import numpy as np
import pytest
import torch

from audio_generation_b200 import h3
from oracle import h3_oracle as O
from tests.h3_testlib import DevLayout, dev_bf16, dev_i32, dev_f32, host_bits
from workloads import TINY_DIMS, FULL_DIMS, config_layout, random_layout, make_layout

pytestmark = pytest.mark.gpu


def _export(dl):
    S = dl.L.S
    perm = np.zeros(max(S, 1), np.int32)
    tc = np.zeros(max((S + 127) // 128, 1), np.uint8)
    nv = h3.h3_layout_export(dl.handle, perm, tc)
    return perm[:S], tc[:(S + 127) // 128], nv


@pytest.mark.parametrize("which", ["cfg1", "cfg3", "cfg5", "rand300", "rand1", "rand129",
                                   "allpad", "nopad"])
def test_layout_tables_bit_exact(which):
    if which == "cfg1":
        L = config_layout(1)
    elif which == "cfg3":
        L = config_layout(3)
    elif which == "cfg5":
        L = config_layout(5)
    elif which == "rand300":
        L = random_layout(300, 1, pad_runs=4)
    elif which == "rand1":
        L = random_layout(1, 2, pad_runs=0)
    elif which == "rand129":
        L = random_layout(129, 3, pad_runs=3, max_run=60)
    elif which == "allpad":
        L = make_layout([("pad", 200)], seed=[0])
    else:
        L = make_layout([("text", 0, 17), ("video", (2, 3, 5), 0, 2), ("audio", 0, 9)], seed=[1])
    dl = DevLayout(TINY_DIMS, L)
    perm, tc, nv = _export(dl)
    assert nv == L.n_valid
    np.testing.assert_array_equal(perm, O.compaction_perm(L.tags))
    np.testing.assert_array_equal(tc, O.tile_classes(L.tags))
    assert h3.h3_layout_error(dl.handle) == h3.H3_OK


def test_empty_layout():
    L = make_layout([], seed=[0])
    dl = DevLayout(TINY_DIMS, L)
    perm, tc, nv = _export(dl)
    assert nv == 0 and perm.size == 0 and tc.size == 0


@pytest.mark.parametrize("breakage", ["tag", "tidx", "pos", "dup", "range", "wrongtag", "count"])
def test_layout_rejects_malformed(breakage):
    L = config_layout(1)
    if breakage == "tag":
        L.tags = L.tags.copy(); L.tags[3] = 3
    elif breakage == "tidx":
        L.t_idx = L.t_idx.copy(); L.t_idx[5] = L.n_t
    elif breakage == "pos":
        L.pos = L.pos.copy(); L.pos[2, 1] = np.inf
    elif breakage == "dup":
        L.video_idx = L.video_idx.copy(); L.video_idx[1] = L.video_idx[0]
    elif breakage == "range":
        L.audio_idx = L.audio_idx.copy(); L.audio_idx[0] = L.S + 5
    elif breakage == "wrongtag":
        L.text_idx = L.text_idx.copy(); L.text_idx[0] = L.video_idx[0]
    elif breakage == "count":
        L.text_idx = L.text_idx[:-1]
    assert O.layout_check(L) == O.LAYOUT_BAD
    with pytest.raises(h3.H3Error) as ei:
        DevLayout(TINY_DIMS, L)
    assert ei.value.status == h3.H3_ERR_LAYOUT


@pytest.mark.parametrize("cfg,B,E", [(1, 2, 512), (3, 1, 5376), (1, 1, 8)])
def test_pack_unpack_bit_exact(cfg, B, E):
    L = config_layout(cfg)
    dl = DevLayout(TINY_DIMS, L)
    g = np.random.default_rng([cfg, B, E])
    vid = g.integers(0, 65536, size=(B, len(L.video_idx), E)).astype(np.uint16)
    aud = g.integers(0, 65536, size=(B, len(L.audio_idx), E)).astype(np.uint16)
    txt = g.integers(0, 65536, size=(B, len(L.text_idx), E)).astype(np.uint16)
    dv, da, dt = dev_bf16(vid), dev_bf16(aud), dev_bf16(txt)
    x = torch.full((B, L.S, E), float("nan"), dtype=torch.bfloat16, device="cuda")
    h3.h3_pack_rows(dl.handle, B, E, dv, da, dt, x)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bits(x), O.pack_rows(L, vid, aud, txt, E))
    ov = torch.empty_like(dv); oa = torch.empty_like(da); ot = torch.empty_like(dt)
    h3.h3_unpack_rows(dl.handle, B, E, x, ov, oa, ot)
    torch.cuda.synchronize()
    rv, ra, rt = O.unpack_rows(L, host_bits(x))
    np.testing.assert_array_equal(host_bits(ov), rv)
    np.testing.assert_array_equal(host_bits(oa), ra)
    np.testing.assert_array_equal(host_bits(ot), rt)
    np.testing.assert_array_equal(host_bits(ov), vid)


def test_pack_rejects_bad_arguments():
    L = config_layout(1)
    dl = DevLayout(TINY_DIMS, L)
    x = torch.zeros((1, L.S, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(h3.H3Error) as ei:
        h3.h3_pack_rows(dl.handle, 1, 12, x, x, x, x)  # row width not a multiple of 8
    assert ei.value.status == h3.H3_ERR_SHAPE
    with pytest.raises(h3.H3Error) as ei:
        h3.h3_pack_rows(dl.handle, 1, 16, None, x, x, x)
    assert ei.value.status == h3.H3_ERR_ARG
    with pytest.raises(h3.H3Error) as ei:
        h3.h3_pack_rows(dl.handle, 1, 16, x.data_ptr() + 2, x, x, x)
    assert ei.value.status == h3.H3_ERR_ALIGN
