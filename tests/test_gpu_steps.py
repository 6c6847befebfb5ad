"""Each step of the block on the GPU (through its own C-ABI entry point)
against the oracle's definition of that step, on seeded inputs.

Inputs are chosen so that each step's own contribution is large next to bf16
rounding (e.g. modulation and gates of order 1), so a wrong term, sign, index
or operand shows up in the comparison.
"""

import numpy as np
import pytest
import torch

from audio_generation_b200 import h3
from oracle import h3_oracle as O
from tests.h3_testlib import (DevLayout, assert_close, dev_bf16, dev_f32, host_f64, rel_l2,
                              host_bits)
from workloads import (FULL_DIMS, TINY_DIMS, Dims, block_weights, config_layout, normal_bf16,
                       prologue_weights, random_layout, make_layout)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_cfg1_B2": (TINY_DIMS, lambda: config_layout(1), 2),
    "tiny_rand333": (TINY_DIMS, lambda: random_layout(333, 5, pad_runs=3, max_run=70), 1),
    "full_rand300": (FULL_DIMS, lambda: random_layout(300, 6, pad_runs=2, max_run=50), 1),
    "tiny_rand1500": (TINY_DIMS, lambda: random_layout(1500, 7, pad_runs=4, max_run=300), 1),
}
# Attention-only cases at full width with more work items (pairs of query tiles
# x 56 heads) than one wave of the GPU; "full_sparse1500" keeps only two key
# tiles and has all-padding pairs of query tiles.
ATTN_CASES = {
    "full_rand1500": (FULL_DIMS, lambda: random_layout(1500, 8, pad_runs=3, max_run=200), 1),
    "full_sparse1500": (FULL_DIMS, lambda: make_layout([("text", 0, 100), ("pad", 1372),
                                                        ("audio", 0, 28)]), 1),
}


def _tmod(n_t, H, seed, std=0.5):
    g = np.random.default_rng([seed, 77])
    return (g.standard_normal((n_t, 6, H)) * std).astype(np.float32)


def _setup(case):
    dims, mk, B = CASES[case]
    L = mk()
    dl = DevLayout(dims, L)
    w = block_weights(dims, 50, 0)
    return dims, L, dl, w, B


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("which", [0, 1])
def test_norm_modulate(case, which):
    dims, L, dl, w, B = _setup(case)
    H = dims.hidden
    xb = normal_bf16((B, L.S, H), [1, which, L.S], 1.5, 0.3)
    tm = _tmod(L.n_t, H, 3)
    x, h = dev_bf16(xb), torch.empty((B, L.S, H), dtype=torch.bfloat16, device="cuda")
    h3.h3_norm_modulate(dl.dims, dl.handle, B, which, x, dev_f32(w.ada_table), dev_f32(tm), h)
    torch.cuda.synchronize()
    got = host_f64(h)
    m = O.row_modulation(L.tags, L.t_idx, w.ada_table, tm)
    c = 3 * which
    valid = L.tags >= 0
    for b in range(B):
        ref = O.norm_modulate(O.bf16_to_f64(xb[b]), m[:, c], m[:, c + 1], dims.norm_eps)
        assert_close(got[b, valid], ref[valid], what=f"norm b={b}", storage_rounding=True)
        assert np.all(got[b, ~valid] == 0.0)


@pytest.mark.parametrize("case", list(CASES))
def test_qkv_rope(case):
    dims, L, dl, w, B = _setup(case)
    H, NH, D = dims.hidden, dims.heads, dims.head_dim
    hb = normal_bf16((B, L.S, H), [2, L.S], 1.0)
    q = torch.empty((B, NH, L.S, D), dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    h3.h3_qkv_rope(dl.dims, dl.handle, B, dev_bf16(hb), dev_bf16(w.w_qkv), dev_bf16(w.q_norm),
                   dev_bf16(w.k_norm), q, k, v)
    torch.cuda.synchronize()
    for b in range(B):
        rq, rk, rv = O.qkv_project(O.bf16_to_f64(hb[b]), L.pos, w.w_qkv, w.q_norm, w.k_norm, dims)
        for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
            g = host_f64(got[b]).transpose(1, 0, 2)  # [S, NH, D]
            assert_close(g, ref, what=f"{name} b={b}", storage_rounding=True)


def _attention_inputs(dims, L, B, seed, q_scale=1.0):
    NH, D = dims.heads, dims.head_dim
    qb = normal_bf16((B, NH, L.S, D), [3, seed, 0], q_scale)
    kb = normal_bf16((B, NH, L.S, D), [3, seed, 1], 1.0)
    vb = normal_bf16((B, NH, L.S, D), [3, seed, 2], 1.0)
    return qb, kb, vb


@pytest.mark.parametrize("case,q_scale", [("tiny_cfg1_B2", 1.0), ("tiny_rand333", 1.0),
                                          ("tiny_rand333", 6.0), ("full_rand300", 1.0),
                                          ("tiny_rand1500", 1.0), ("tiny_rand1500", 6.0),
                                          ("full_rand1500", 1.0), ("full_sparse1500", 1.0),
                                          ("full_sparse1500", 6.0)])
def test_attention(case, q_scale):
    if case in ATTN_CASES:
        dims, mk, B = ATTN_CASES[case]
        L = mk()
        dl = DevLayout(dims, L)
    else:
        dims, L, dl, w, B = _setup(case)
    NH, D = dims.heads, dims.head_dim
    qb, kb, vb = _attention_inputs(dims, L, B, 11, q_scale)
    o = torch.full((B, L.S, NH * D), float("nan"), dtype=torch.bfloat16, device="cuda")
    h3.h3_attention(dl.dims, dl.handle, B, dev_bf16(qb), dev_bf16(kb), dev_bf16(vb), o)
    torch.cuda.synchronize()
    got = host_f64(o)
    pad = L.tags < 0
    tc = O.tile_classes(L.tags)
    allpad_rows = np.repeat(tc == 1, 128)[:L.S]
    for b in range(B):
        t = lambda a: O.bf16_to_f64(a[b]).transpose(1, 0, 2)
        ref = O.attention(t(qb), pad, t(kb), t(vb), pad)
        assert_close(got[b, ~pad], ref[~pad], what=f"attention b={b}", storage_rounding=True)
        assert np.all(got[b, allpad_rows] == 0.0)
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("case", list(CASES))
def test_out_residual(case):
    dims, L, dl, w, B = _setup(case)
    H, A = dims.hidden, dims.attn_width
    ob = normal_bf16((B, L.S, A), [4, L.S], 1.0)
    xb = normal_bf16((B, L.S, H), [5, L.S], 1.0)
    tm = _tmod(L.n_t, H, 4, std=1.0)
    x = dev_bf16(xb)
    h3.h3_out_residual(dl.dims, dl.handle, B, dev_bf16(ob), dev_bf16(w.w_o), dev_f32(w.ada_table),
                       dev_f32(tm), x)
    torch.cuda.synchronize()
    got = host_f64(x)
    m = O.row_modulation(L.tags, L.t_idx, w.ada_table, tm)
    valid = L.tags >= 0
    for b in range(B):
        x0 = O.bf16_to_f64(xb[b])
        ref = O.out_project_residual(x0, O.bf16_to_f64(ob[b]), m[:, 2], w.w_o)
        assert_close(got[b, valid], ref[valid], what="x1", storage_rounding=True)
        assert_close(got[b, valid] - x0[valid], ref[valid] - x0[valid], what="x1 - x",
                     mabs=np.inf)
        np.testing.assert_array_equal(host_bits(x)[b, ~valid], xb[b, ~valid])


@pytest.mark.parametrize("case", list(CASES))
def test_ffn_up(case):
    dims, L, dl, w, B = _setup(case)
    H, Fd = dims.hidden, dims.ffn
    hb = normal_bf16((B, L.S, H), [6, L.S], 1.0)
    g = torch.empty((B, L.S, Fd), dtype=torch.bfloat16, device="cuda")
    h3.h3_ffn_up(dl.dims, dl.handle, B, dev_bf16(hb), dev_bf16(w.w13), g)
    torch.cuda.synchronize()
    got = host_f64(g)
    for b in range(B):
        ref = O.ffn_gate(O.bf16_to_f64(hb[b]), w.w13, Fd)
        assert_close(got[b], ref, what="g", storage_rounding=True)


@pytest.mark.parametrize("case", list(CASES))
def test_ffn_down_residual(case):
    dims, L, dl, w, B = _setup(case)
    H, Fd = dims.hidden, dims.ffn
    gb = normal_bf16((B, L.S, Fd), [7, L.S], 1.0)
    xb = normal_bf16((B, L.S, H), [8, L.S], 1.0)
    tm = _tmod(L.n_t, H, 5, std=1.0)
    x = dev_bf16(xb)
    h3.h3_ffn_down_residual(dl.dims, dl.handle, B, dev_bf16(gb), dev_bf16(w.w2),
                            dev_f32(w.ada_table), dev_f32(tm), x)
    torch.cuda.synchronize()
    got = host_f64(x)
    m = O.row_modulation(L.tags, L.t_idx, w.ada_table, tm)
    valid = L.tags >= 0
    for b in range(B):
        x0 = O.bf16_to_f64(xb[b])
        ref = O.ffn_down_residual(x0, O.bf16_to_f64(gb[b]), m[:, 5], w.w2)
        assert_close(got[b, valid], ref[valid], what="x2", storage_rounding=True)
        assert_close(got[b, valid] - x0[valid], ref[valid] - x0[valid], what="x2 - x1",
                     mabs=np.inf)
        np.testing.assert_array_equal(host_bits(x)[b, ~valid], xb[b, ~valid])


# fp32 outputs: a K-term fp32 dot product carries relative error ~ sqrt(K) * 2^-24;
# 1e-4 relative L2 leaves two orders of magnitude of margin at K = 5376.
TMOD_REL = 1e-4


@pytest.mark.parametrize("dims,n_t", [(TINY_DIMS, 256), (TINY_DIMS, 64), (TINY_DIMS, 65),
                                      (FULL_DIMS, 2), (FULL_DIMS, 3), (FULL_DIMS, 17),
                                      (FULL_DIMS, 64), (FULL_DIMS, 70), (FULL_DIMS, 300)])
def test_timestep_modulation(dims, n_t):
    """n_t < 65: skinny fp32 GEMMs on the CUDA cores (chunks of eight timesteps,
    ragged last chunk at 17); n_t >= 65: tensor-core GEMMs over three-way bf16
    splits of the fp32 operands (same fp32-level tolerance)."""
    pw = prologue_weights(dims, 1 if dims is TINY_DIMS else 2)
    g = np.random.default_rng(n_t)
    t = g.random(n_t).astype(np.float32)
    t[0] = 0.0
    t[-1] = 1.0
    d = h3.make_dims(dims)
    ws_b = h3.h3_timestep_workspace_size(d, n_t)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    tmod = torch.empty((n_t, 6, dims.hidden), dtype=torch.float32, device="cuda")
    h3.h3_timestep_modulation(d, n_t, dev_f32(t), dev_f32(pw.w_t1), dev_f32(pw.w_t2),
                              dev_f32(pw.w_proj), tmod, ws, ws_b)
    torch.cuda.synchronize()
    ref = O.timestep_modulation(t, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim, dims.hidden)
    got = tmod.double().cpu().numpy()
    assert rel_l2(got, ref) < TMOD_REL


def test_timestep_modulation_many_timesteps_sampled_rows():
    """2048 per-row timesteps at full width (split-operand tensor-core form):
    rows are independent, so sampled rows are checked against the oracle run on
    their timesteps alone."""
    dims, n_t = FULL_DIMS, 2048
    pw = prologue_weights(dims, 2)
    g = np.random.default_rng(2048)
    t = g.random(n_t).astype(np.float32)
    d = h3.make_dims(dims)
    ws_b = h3.h3_timestep_workspace_size(d, n_t)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    tmod = torch.empty((n_t, 6, dims.hidden), dtype=torch.float32, device="cuda")
    h3.h3_timestep_modulation(d, n_t, dev_f32(t), dev_f32(pw.w_t1), dev_f32(pw.w_t2),
                              dev_f32(pw.w_proj), tmod, ws, ws_b)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 255, 256, 1000, 2047])
    ref = O.timestep_modulation(t[rows], pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim, dims.hidden)
    got = tmod[torch.as_tensor(rows, device="cuda")].double().cpu().numpy()
    assert rel_l2(got, ref) < TMOD_REL
