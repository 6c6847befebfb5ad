"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties one oracle function to a fact the pages or the mathematics
fix: values the page prints, closed forms, library routines on a special
case, brute force on tiny inputs, and invariants of the method (RoPE scores
depend only on position differences; padding rows never change other rows;
rows permute with their positions, tags and timesteps).
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import h3_oracle as O
from workloads import (FULL_DIMS, TINY_DIMS, Dims, activations, block_weights,
                       config_layout, prologue_weights, random_layout, make_layout,
                       bf16_bits_to_f32, f32_to_bf16_bits)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F = np.float64

# A small block for fast invariant checks: 2 heads of 128 (attn width 256 >
# hidden 128), ffn 256.
SMALL = Dims(hidden=128, heads=2, head_dim=128, ffn=256, time_embed_dim=64, time_hidden=128)


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _tmod_random(n_t, H, seed, std=0.5):
    g = np.random.default_rng(seed)
    return g.standard_normal((n_t, 6, H)) * std


def _weights_big_gates(dims, seed):
    """Block weights ~N(0, 0.1^2) and AdaLN table ~N(0, 0.3^2), so that the
    block visibly moves x at these small widths."""
    w = block_weights(dims, 77, seed)
    g = np.random.default_rng([seed, 5])
    for name in ("w_qkv", "w_o", "w13", "w2"):
        a = getattr(w, name)
        setattr(w, name, f32_to_bf16_bits(g.standard_normal(a.shape).astype(np.float32) * 0.1))
    w.ada_table = (g.standard_normal(w.ada_table.shape) * 0.3).astype(np.float32)
    return w


# ---------------------------------------------------------------- golden values

def _golden():
    out = {}
    with open(os.path.join(GOLDEN, "h3_constructor_defaults.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            out[k] = float(v)
    return out


def test_golden_constructor_defaults_match_full_dims():
    g = _golden()
    d = FULL_DIMS
    assert d.heads == g["num_attention_heads"]
    assert d.head_dim == g["attention_head_dim"]
    assert d.hidden == g["hidden_size"]
    assert d.ffn == g["ffn_dim"]
    assert d.freq_dim == g["freq_dim"]
    assert d.time_hidden == g["time_embed_hidden_dim"]
    assert d.time_embed_dim == g["time_embed_dim"]
    assert d.rope_freq_dim == g["rope_freq_dim"]
    assert d.rope_theta == g["rope_theta"]
    assert d.norm_eps == g["norm_eps"] and d.qk_norm_eps == g["qk_norm_eps"]
    assert 2 * 3 * d.rope_freq_dim == g["rotated_channels"]
    assert d.attn_width == g["attn_width"] and d.attn_width > d.hidden


def test_projection_shapes_full_width():
    """56 * 128 != 5376: QKV is 5376 -> 21504 and O is 7168 -> 5376."""
    d = FULL_DIMS
    H, A, Fd = d.hidden, d.attn_width, d.ffn
    assert (3 * A, H) == (21504, 5376)
    assert (H, A) == (5376, 7168)
    assert (2 * Fd, H) == (28672, 5376) and (H, Fd) == (5376, 14336)
    # The oracle splits the head-interleaved weight into three [A, H] blocks.
    wq, wk, wv = O.split_qkv_weight(np.zeros((3 * A, 8)), d.heads, d.head_dim)
    assert wq.shape == wk.shape == wv.shape == (A, 8)
    w1, w3 = O.split_w13(np.zeros((2 * Fd, 8)), Fd)
    assert w1.shape == w3.shape == (Fd, 8)


def test_split_qkv_weight_head_interleaving_by_hand():
    NH, D = 3, 4
    rows = np.arange(3 * NH * D)[:, None].astype(F)
    wq, wk, wv = O.split_qkv_weight(rows, NH, D)
    for n in range(NH):
        for d in range(D):
            assert wq[n * D + d, 0] == n * 3 * D + d
            assert wk[n * D + d, 0] == n * 3 * D + D + d
            assert wv[n * D + d, 0] == n * 3 * D + 2 * D + d


def test_split_w13_block_interleaving_by_hand():
    Fd = 256
    rows = np.arange(2 * Fd)[:, None].astype(F)
    w1, w3 = O.split_w13(rows, Fd)
    for f in range(Fd):
        j, r = divmod(f, 128)
        assert w1[f, 0] == 256 * j + r
        assert w3[f, 0] == 256 * j + 128 + r


# ---------------------------------------------------------------- storage

def test_bf16_roundtrip_and_rne():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 3.0e38], np.float32)
    bits = f32_to_bf16_bits(vals)
    back = O.bf16_to_f64(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: ties go to the even mantissa (1.0).
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2 ** -6
    assert back[3] == -2.5 and back[4] == 0.0
    np.testing.assert_array_equal(bf16_bits_to_f32(bits).astype(F), back)
    np.testing.assert_array_equal(O.round_bf16(vals.astype(F)), back)
    # agrees with torch's own float -> bfloat16 conversion
    tb = torch.tensor(vals).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(tb, back)


# ---------------------------------------------------------------- prologue (a2)

def test_sinusoid_closed_forms():
    t = np.array([0.0, 0.25, 1.0])
    s = O.timestep_sinusoid(t, 256)
    assert s.shape == (3, 256)
    np.testing.assert_array_equal(s[0, :128], 1.0)
    np.testing.assert_array_equal(s[0, 128:], 0.0)
    np.testing.assert_allclose(s[:, :128] ** 2 + s[:, 128:] ** 2, 1.0, atol=1e-15)
    # f_0 = 1 and f_64 = 10^4^(-1/2) = 0.01
    assert abs(s[2, 0] - math.cos(1.0)) < 1e-15
    assert abs(s[2, 64] - math.cos(0.01)) < 1e-15
    assert abs(s[1, 128 + 64] - math.sin(0.25 * 0.01)) < 1e-15


def test_silu_closed_forms():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert abs(O.silu(np.array([50.0]))[0] - 50.0) < 1e-12
    assert abs(O.silu(np.array([-50.0]))[0]) < 1e-18
    x = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(O.silu(x), torch.nn.functional.silu(torch.tensor(x)).numpy(),
                               rtol=1e-14, atol=1e-15)


def test_timestep_modulation_matches_torch_modules():
    d = TINY_DIMS
    pw = prologue_weights(d, 1)
    t = np.array([0.0, 0.1, 0.9], np.float32)
    got = O.timestep_modulation(t, pw.w_t1, pw.w_t2, pw.w_proj, d.freq_dim, d.hidden)
    lin = torch.nn.functional.linear
    half = d.freq_dim // 2
    f = torch.exp(-math.log(10000.0) * torch.arange(half, dtype=torch.float64) / half)
    arg = torch.tensor(t, dtype=torch.float64)[:, None] * f
    emb = torch.cat([torch.cos(arg), torch.sin(arg)], 1)
    a = torch.nn.functional.silu(lin(emb, torch.tensor(pw.w_t1, dtype=torch.float64)))
    temb = lin(a, torch.tensor(pw.w_t2, dtype=torch.float64))
    ref = lin(torch.nn.functional.silu(temb), torch.tensor(pw.w_proj, dtype=torch.float64))
    np.testing.assert_allclose(got.reshape(3, -1), ref.numpy(), rtol=1e-12, atol=1e-14)
    assert got.shape == (3, 6, d.hidden)


def test_row_modulation_by_loop():
    H = 8
    g = np.random.default_rng(3)
    table = g.standard_normal((3, 6, H))
    tmod = g.standard_normal((5, 6, H))
    tags = np.array([0, 2, -1, 1, 1, 0])
    tidx = np.array([4, 0, 3, 2, 2, 1])
    m = O.row_modulation(tags, tidx, table, tmod)
    for r in range(6):
        if tags[r] < 0:
            np.testing.assert_array_equal(m[r], 0.0)
        else:
            for c in range(6):
                for i in range(H):
                    assert m[r, c, i] == table[tags[r], c, i] + tmod[tidx[r], c, i]


# ---------------------------------------------------------------- norms (a3, a4, a7)

def test_layer_norm_closed_form_and_torch():
    x = np.full((2, 64), 3.25)
    np.testing.assert_array_equal(O.layer_norm(x, 1e-5), 0.0)
    g = np.random.default_rng(0)
    x = g.standard_normal((5, 512)) * 3 + 1
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (512,), eps=1e-5).numpy()
    np.testing.assert_allclose(O.layer_norm(x, 1e-5), ref, rtol=1e-12, atol=1e-12)
    # modulation = 0 reduces norm_modulate to the plain norm
    z = np.zeros(512)
    np.testing.assert_array_equal(O.norm_modulate(x, z, z, 1e-5), O.layer_norm(x, 1e-5))


def test_rms_norm_closed_form_and_torch():
    w = np.linspace(0.5, 1.5, 128)
    c = -2.0
    x = np.full((1, 128), c)
    got = O.rms_norm(x, w, 1e-5)
    np.testing.assert_allclose(got[0], math.copysign(1.0, c) * w * abs(c) / math.sqrt(c * c + 1e-5),
                               rtol=1e-15)
    g = np.random.default_rng(1)
    x = g.standard_normal((7, 3, 128))
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (128,), weight=torch.tensor(w),
                                       eps=1e-5).numpy()
    np.testing.assert_allclose(O.rms_norm(x, w, 1e-5), ref, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- RoPE (a4)

def _inv():
    return O.rope_inv_freq(16, 1e4)


def test_rope_inv_freq_values():
    inv = _inv()
    assert inv.shape == (16,) and inv[0] == 1.0
    assert abs(inv[8] - 0.01) < 1e-15  # 10^4^(-1/2)
    assert np.all(np.diff(inv) < 0)


def test_rope_zero_position_is_identity_and_tail_untouched():
    g = np.random.default_rng(2)
    x = g.standard_normal((6, 2, 128))
    np.testing.assert_array_equal(O.rope_apply(x, np.zeros((6, 3)), _inv()), x)
    pos = g.integers(1, 40, size=(6, 3)).astype(F)
    y = O.rope_apply(x, pos, _inv())
    np.testing.assert_array_equal(y[:, :, 96:], x[:, :, 96:])   # 2*3*16 channels rotate
    assert np.all(np.abs(y[:, :, :96] - x[:, :, :96]).max(axis=(0, 1)) > 0)


def test_rope_preserves_pair_norms():
    g = np.random.default_rng(3)
    x = g.standard_normal((10, 1, 128))
    pos = g.standard_normal((10, 3)) * 20
    y = O.rope_apply(x, pos, _inv())
    for a in range(3):
        for j in range(16):
            c0, c1 = 32 * a + j, 32 * a + j + 16
            np.testing.assert_allclose(y[:, 0, c0] ** 2 + y[:, 0, c1] ** 2,
                                       x[:, 0, c0] ** 2 + x[:, 0, c1] ** 2, rtol=1e-12)


def test_rope_scores_depend_only_on_position_difference():
    g = np.random.default_rng(4)
    q = g.standard_normal((1, 1, 128))
    k = g.standard_normal((1, 1, 128))
    for _ in range(5):
        p, pk = g.integers(-30, 30, size=(2, 3)).astype(F)
        delta = g.integers(-100, 100, size=3).astype(F)
        s0 = (O.rope_apply(q, p[None], _inv()) * O.rope_apply(k, pk[None], _inv())).sum()
        s1 = (O.rope_apply(q, (p + delta)[None], _inv())
              * O.rope_apply(k, (pk + delta)[None], _inv())).sum()
        assert abs(s0 - s1) < 1e-10 * (1 + abs(s0))


def test_rope_axes_share_one_inv_freq():
    """Position p on axis a rotates channel block a exactly as p on axis 0 rotates block 0."""
    g = np.random.default_rng(5)
    x = g.standard_normal((1, 1, 128))
    blk = x[:, :, 0:32].copy()
    for a in (1, 2):
        xa = np.zeros_like(x)
        xa[:, :, 32 * a:32 * a + 32] = blk
        pa = np.zeros((1, 3))
        pa[0, a] = 7.0
        p0 = np.array([[7.0, 0, 0]])
        ya = O.rope_apply(xa, pa, _inv())
        y0 = O.rope_apply(np.concatenate([blk, np.zeros((1, 1, 96))], 2), p0, _inv())
        np.testing.assert_allclose(ya[:, :, 32 * a:32 * a + 32], y0[:, :, 0:32], rtol=1e-14)


# ---------------------------------------------------------------- attention (a5)

def _brute_attention(q, doc_q, k, v, doc_k):
    """Pure-Python loops: explicit scores, explicit softmax, explicit sum."""
    n, NH, D = q.shape
    S = k.shape[0]
    out = np.zeros((n, NH * D))
    for i in range(n):
        for h in range(NH):
            scores = []
            for j in range(S):
                if doc_k[j] != doc_q[i]:
                    continue
                s = sum(q[i, h, c] * k[j, h, c] for c in range(D)) / math.sqrt(D)
                scores.append((j, s))
            mx = max(s for _, s in scores)
            ws = [(j, math.exp(s - mx)) for j, s in scores]
            tot = sum(wt for _, wt in ws)
            for c in range(D):
                out[i, h * D + c] = sum(wt * v[j, h, c] for j, wt in ws) / tot
    return out


def test_attention_matches_brute_force_small():
    g = np.random.default_rng(6)
    S, NH, D = 11, 2, 8
    q = g.standard_normal((S, NH, D))
    k = g.standard_normal((S, NH, D))
    v = g.standard_normal((S, NH, D))
    doc = np.array([0, 0, 1, 0, 0, 1, 1, 0, 0, 0, 1]) == 1
    got = O.attention(q, doc, k, v, doc)
    np.testing.assert_allclose(got, _brute_attention(q, doc, k, v, doc), rtol=1e-12, atol=1e-13)


def test_attention_matches_torch_sdpa_with_boolean_mask():
    g = np.random.default_rng(7)
    S, NH, D = 64, 3, 128
    q, k, v = (g.standard_normal((S, NH, D)) for _ in range(3))
    doc = g.random(S) < 0.2
    got = O.attention(q, doc, k, v, doc)
    mask = torch.tensor(doc[:, None] == doc[None, :])
    t = lambda a: torch.tensor(a).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)
    ref = ref[0].permute(1, 0, 2).reshape(S, NH * D).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_attention_closed_forms():
    g = np.random.default_rng(8)
    S, D = 9, 128
    q = g.standard_normal((S, 1, D))
    kk = np.repeat(g.standard_normal((1, 1, D)), S, axis=0)   # equal keys
    v = g.standard_normal((S, 1, D))
    doc = np.zeros(S, bool)
    np.testing.assert_allclose(O.attention(q, doc, kk, v, doc),
                               np.repeat(v.mean(axis=0).reshape(1, D), S, 0), rtol=1e-12)
    # a query whose document holds one key returns that key's value
    doc = np.zeros(S, bool)
    doc[4] = True
    o = O.attention(q, doc, g.standard_normal((S, 1, D)), v, doc)
    np.testing.assert_allclose(o[4], v[4, 0], rtol=1e-15)


# ---------------------------------------------------------------- block invariants

def _small_case(S=48, seed=0, pad_runs=2, n_t=None):
    L = random_layout(S, seed, pad_runs=pad_runs, max_run=10, n_t=n_t)
    w = _weights_big_gates(SMALL, seed)
    x = O.bf16_to_f64(activations(SMALL, 77, S, B=1, key=seed))
    tmod = _tmod_random(L.n_t, SMALL.hidden, seed + 100, std=0.3)
    return L, w, x, tmod


def test_block_moves_valid_rows_and_keeps_padding_rows_exactly():
    L, w, x, tmod = _small_case()
    y = O.block_forward(x, w, L, tmod, SMALL)
    pad = L.tags < 0
    assert pad.any() and (~pad).any()
    np.testing.assert_array_equal(y[0, pad], x[0, pad])
    assert np.abs(y[0, ~pad] - x[0, ~pad]).mean() > 0.05


def test_block_padding_rows_never_change_valid_outputs():
    L, w, x, tmod = _small_case(seed=1)
    pad = L.tags < 0
    y = O.block_forward(x, w, L, tmod, SMALL)
    g = np.random.default_rng(11)
    x2 = x.copy()
    x2[0, pad] = g.standard_normal((pad.sum(), SMALL.hidden)) * 5
    L2 = random_layout(L.S, 1, pad_runs=2, max_run=10)
    L2.pos = L.pos.copy()
    L2.pos[pad] = g.integers(0, 99, size=(pad.sum(), 3))
    L2.t_idx = L.t_idx.copy()
    L2.t_idx[pad] = g.integers(0, L.n_t, size=pad.sum())
    y2 = O.block_forward(x2, w, L2, tmod, SMALL)
    np.testing.assert_array_equal(y2[0, ~pad], y[0, ~pad])          # bit-identical
    # deleting the padding rows altogether leaves valid outputs unchanged
    keep = ~pad
    L3 = make_layout([], seed=[0])
    L3.tags, L3.pos, L3.t_idx = L.tags[keep], L.pos[keep], L.t_idx[keep]
    L3.timestep = L.timestep
    y3 = O.block_forward(x[:, keep], w, L3, tmod, SMALL)
    np.testing.assert_allclose(y3[0], y[0, keep], rtol=1e-12, atol=1e-12)


def test_block_permutation_equivariance():
    L, w, x, tmod = _small_case(seed=2)
    y = O.block_forward(x, w, L, tmod, SMALL)
    perm = np.random.default_rng(12).permutation(L.S)
    Lp = make_layout([], seed=[0])
    Lp.tags, Lp.pos, Lp.t_idx, Lp.timestep = L.tags[perm], L.pos[perm], L.t_idx[perm], L.timestep
    yp = O.block_forward(x[:, perm], w, Lp, tmod, SMALL)
    np.testing.assert_allclose(yp, y[:, perm], rtol=1e-11, atol=1e-11)


def test_block_translation_of_all_positions_leaves_output_unchanged():
    L, w, x, tmod = _small_case(seed=3)
    y = O.block_forward(x, w, L, tmod, SMALL)
    L2 = make_layout([], seed=[0])
    L2.tags, L2.t_idx, L2.timestep = L.tags, L.t_idx, L.timestep
    L2.pos = L.pos + np.array([13.0, -7.0, 101.0], np.float32)
    y2 = O.block_forward(x, w, L2, tmod, SMALL)
    assert _rel(y2 - x, y - x) < 1e-9


def test_block_zero_gates_is_identity_and_gate2_isolates_attention():
    L, w, x, tmod = _small_case(seed=4)
    w0 = _weights_big_gates(SMALL, 4)
    w0.ada_table = w.ada_table.copy()
    w0.ada_table[:, 2] = 0.0
    w0.ada_table[:, 5] = 0.0
    t0 = tmod.copy()
    t0[:, 2] = 0.0
    t0[:, 5] = 0.0
    np.testing.assert_array_equal(O.block_forward(x, w0, L, t0, SMALL), x)
    # with gate2 = 0 the output is x + gate1 * attention-branch alone
    w0.ada_table[:, 2] = w.ada_table[:, 2]
    t0[:, 2] = tmod[:, 2]
    y = O.block_forward(x, w0, L, t0, SMALL)
    pad = L.tags < 0
    m = O.row_modulation(L.tags, L.t_idx, w.ada_table, tmod)
    h = O.norm_modulate(x[0], m[:, 0], m[:, 1], SMALL.norm_eps)
    q, k, v = O.qkv_project(h, L.pos, w.w_qkv, w.q_norm, w.k_norm, SMALL)
    o = O.attention(q, pad, k, v, pad)
    x1 = O.out_project_residual(x[0], o, m[:, 2], w.w_o)
    np.testing.assert_allclose(y[0, ~pad], x1[~pad], rtol=1e-13, atol=1e-13)


def test_block_library_special_case_matches_torch_composition():
    """With modulation scale = shift = 0 and gates = 1 the block is a plain
    pre-norm transformer block; rebuild it from torch CPU primitives."""
    L, w, x, _ = _small_case(seed=5, pad_runs=1)
    d = SMALL
    w.ada_table = np.zeros_like(w.ada_table)
    w.ada_table[:, 2] = 1.0
    w.ada_table[:, 5] = 1.0
    tmod = np.zeros((L.n_t, 6, d.hidden))
    y = O.block_forward(x, w, L, tmod, d)
    T = lambda a: torch.tensor(np.asarray(a, F))
    xt = T(x[0])
    pad = torch.tensor(L.tags < 0)
    wq, wk, wv = (T(a) for a in O.split_qkv_weight(O.bf16_to_f64(w.w_qkv), d.heads, d.head_dim))
    h = torch.nn.functional.layer_norm(xt, (d.hidden,), eps=d.norm_eps)
    def heads(a):
        return a.reshape(L.S, d.heads, d.head_dim)
    qn, kn = T(O.bf16_to_f64(w.q_norm)), T(O.bf16_to_f64(w.k_norm))
    q = torch.nn.functional.rms_norm(heads(h @ wq.T), (d.head_dim,), weight=qn, eps=d.qk_norm_eps)
    k = torch.nn.functional.rms_norm(heads(h @ wk.T), (d.head_dim,), weight=kn, eps=d.qk_norm_eps)
    v = heads(h @ wv.T)
    # RoPE via complex multiplication on (c, c + 16) pairs of each 32-channel axis block
    inv = T(O.rope_inv_freq(16, d.rope_theta))
    def rope(a):
        out = a.clone()
        for ax in range(3):
            ang = T(L.pos[:, ax])[:, None] * inv[None]
            z = torch.complex(a[:, :, 32 * ax:32 * ax + 16], a[:, :, 32 * ax + 16:32 * ax + 32])
            z = z * torch.polar(torch.ones_like(ang), ang)[:, None, :]
            out[:, :, 32 * ax:32 * ax + 16] = z.real
            out[:, :, 32 * ax + 16:32 * ax + 32] = z.imag
        return out
    q, k = rope(q), rope(k)
    mask = pad[:, None] == pad[None, :]
    o = torch.nn.functional.scaled_dot_product_attention(
        q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None], v.permute(1, 0, 2)[None],
        attn_mask=mask)[0].permute(1, 0, 2).reshape(L.S, -1)
    x1 = xt + o @ T(O.bf16_to_f64(w.w_o)).T
    h2 = torch.nn.functional.layer_norm(x1, (d.hidden,), eps=d.norm_eps)
    w1, w3 = (T(a) for a in O.split_w13(O.bf16_to_f64(w.w13), d.ffn))
    g = torch.nn.functional.silu(h2 @ w1.T) * (h2 @ w3.T)
    x2 = x1 + g @ T(O.bf16_to_f64(w.w2)).T
    ref = torch.where(pad[:, None], xt, x2).numpy()
    np.testing.assert_allclose(y[0], ref, rtol=1e-10, atol=1e-10)


def test_block_rows_evaluator_matches_full_block():
    L, w, x, tmod = _small_case(S=70, seed=6)
    y = O.block_forward(x, w, L, tmod, SMALL)
    rows = np.array([0, 5, 17, 33, 69])
    yr = O.block_forward_rows(x[0], w, L, lambda ti, c: tmod[ti, :c], SMALL, rows, chunk=16)
    np.testing.assert_allclose(yr, y[0, rows], rtol=1e-12, atol=1e-12)


def test_batch_elements_are_independent_documents():
    L, w, x, tmod = _small_case(seed=7)
    xb = np.concatenate([x, x[:, ::-1] * 0.5], 0)
    y = O.block_forward(xb, w, L, tmod, SMALL)
    np.testing.assert_array_equal(y[0], O.block_forward(x, w, L, tmod, SMALL)[0])
    np.testing.assert_array_equal(y[1], O.block_forward(xb[1:], w, L, tmod, SMALL)[0])


def test_stack_is_blocks_in_sequence():
    L, w, x, tmod = _small_case(seed=8)
    ws = [_weights_big_gates(SMALL, 20 + i) for i in range(3)]
    y = O.stack_forward(x, lambda i: ws[i], 3, L, tmod, SMALL)
    z = x
    for i in range(3):
        z = O.block_forward(z, ws[i], L, tmod, SMALL)
    np.testing.assert_array_equal(y, z)


def test_bf16_storage_floor_is_inside_the_tolerance():
    """The bf16-storage emulation of the tiny workload sits well inside
    rel-L2 1e-2 / max-abs 5e-2 of the float64 block, for one block and for 50."""
    d = TINY_DIMS
    L = config_layout(1)
    pw = prologue_weights(d, 1)
    tmod = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, d.freq_dim, d.hidden)
    x = O.bf16_to_f64(activations(d, 1, L.S))
    w = block_weights(d, 1)
    y = O.block_forward(x, w, L, tmod, d)
    ye = O.block_forward(x, w, L, tmod, d, emulate=True)
    assert _rel(ye, y) < 2e-3 and np.abs(ye - y).max() < 2e-2


# ---------------------------------------------------------------- layout (a0, a1)

def test_layout_check_accepts_config_layouts():
    for cfg in (1, 2, 3, 5):
        assert O.layout_check(config_layout(cfg)) == O.LAYOUT_OK


@pytest.mark.parametrize("breakage", ["tag", "tidx", "pos", "dup", "range", "wrongtag", "count"])
def test_layout_check_rejects_each_malformation(breakage):
    L = config_layout(1)
    if breakage == "tag":
        L.tags = L.tags.copy(); L.tags[3] = 3
    elif breakage == "tidx":
        L.t_idx = L.t_idx.copy(); L.t_idx[5] = L.n_t
    elif breakage == "pos":
        L.pos = L.pos.copy(); L.pos[2, 1] = np.nan
    elif breakage == "dup":
        L.video_idx = L.video_idx.copy(); L.video_idx[1] = L.video_idx[0]
    elif breakage == "range":
        L.audio_idx = L.audio_idx.copy(); L.audio_idx[0] = L.S
    elif breakage == "wrongtag":
        L.text_idx = L.text_idx.copy(); L.text_idx[0] = L.video_idx[0]
    elif breakage == "count":
        L.text_idx = L.text_idx[:-1]
    assert O.layout_check(L) == O.LAYOUT_BAD


def test_tile_classes_of_config3_layout():
    L = config_layout(3)
    tc = O.tile_classes(L.tags)
    assert tc.shape == (128,)
    # padding runs start at rows 960 (crosses tiles 7 and 8), 7296, 14848, 16256
    assert tc[7] == 2 and tc[8] == 2
    assert tc[57] == 1 and tc[116] == 1 and tc[127] == 1
    assert int((tc == 0).sum()) == 128 - 5
    assert L.S - L.n_valid == 512


def test_compaction_perm_is_stable_partition():
    L = random_layout(300, 4, pad_runs=5)
    p = O.compaction_perm(L.tags)
    assert sorted(p.tolist()) == list(range(300))
    V = L.n_valid
    assert np.all(L.tags[p[:V]] >= 0) and np.all(L.tags[p[V:]] < 0)
    assert np.all(np.diff(p[:V]) > 0) and np.all(np.diff(p[V:]) > 0)


def test_pack_unpack_roundtrip_and_zero_padding():
    L = config_layout(1)
    g = np.random.default_rng(9)
    H, B = 16, 2
    vid = g.integers(0, 65535, size=(B, len(L.video_idx), H)).astype(np.uint16)
    aud = g.integers(0, 65535, size=(B, len(L.audio_idx), H)).astype(np.uint16)
    txt = g.integers(0, 65535, size=(B, len(L.text_idx), H)).astype(np.uint16)
    x = O.pack_rows(L, vid, aud, txt, H)
    np.testing.assert_array_equal(x[:, L.tags < 0], 0)
    np.testing.assert_array_equal(x[:, L.video_idx[3]], vid[:, 3])
    v2, a2, t2 = O.unpack_rows(L, x)
    np.testing.assert_array_equal(v2, vid)
    np.testing.assert_array_equal(a2, aud)
    np.testing.assert_array_equal(t2, txt)


def test_config_layouts_row_counts():
    L1 = config_layout(1)
    assert (L1.S, L1.n_valid, len(L1.text_idx), len(L1.video_idx), len(L1.audio_idx)) == \
        (256, 240, 48, 128, 64)
    L3 = config_layout(3)
    assert (L3.S, L3.n_valid, len(L3.text_idx), len(L3.video_idx), len(L3.audio_idx)) == \
        (16384, 15872, 1024, 12288, 2560)
    L5 = config_layout(5)
    assert L5.n_t == 2 and L5.timestep[0] == 0.0
    assert set(np.unique(L5.t_idx).tolist()) == {0, 1}


# ---------------------------------------------------------------- prologue worked by hand

def test_timestep_modulation_worked_by_hand():
    """A tiny prologue worked out by hand: freq_dim 4 (two frequencies,
    f_0 = 1 and f_1 = (10^4)^(-1/2) = 0.01), time_hidden 2, time_embed_dim 2,
    hidden 2 (six chunks of two), timesteps 0 and 0.5.

    W_t1 = [[1, 0, 0, 0], [0, 0, 2, 100]] reads cos(t), then 2 sin(t) + 100 sin(0.01 t);
    W_t2 = [[1, -1], [-2, 0]];  W_proj row (2c + j) = [c + 1, (-1)^j (j + 1) / 2].

    t = 0:   sinusoid [cos 0, cos 0, sin 0, sin 0] = [1, 1, 0, 0]
             W_t1 -> [1, 0];  SiLU(1) = 1 / (1 + e^-1) = 0.7310585786, SiLU(0) = 0
             W_t2 -> temb = [0.7310585786, -1.4621171573]
             SiLU -> [0.4934919753, -0.2750881685]
             chunk c, column j = (c + 1) 0.4934919753 + (-1)^j (j + 1)/2 (-0.2750881685)
               c = 0: [0.3559478910, 0.7685801438] ... c = 5: [2.8234077675, 3.2360400202]
    t = 0.5: sinusoid [cos .5, cos .005, sin .5, sin .005]
               = [0.8775825619, 0.9999875000, 0.4794255386, 0.0049999792]
             W_t1 -> [0.8775825619, 0.9588510772 + 0.4999979167 = 1.4588489939]
             SiLU -> [0.6198550086, 1.1836467133]
             W_t2 -> temb = [-0.5637917047, -1.2397100173]
             SiLU -> [-0.2044706686, -0.2782981200]
               c = 0: [-0.3436197285, 0.0738274514] ... c = 5: [-1.3659730714, -0.9485258914]

    A dropped or moved SiLU, swapped sin/cos halves, the frequency divisor
    freq_dim instead of freq_dim / 2 (f_1 = 0.1), or a transposed chunk
    reshape each changes these values far beyond the tolerance.
    """
    w_t1 = np.array([[1, 0, 0, 0], [0, 0, 2, 100]], F)
    w_t2 = np.array([[1, -1], [-2, 0]], F)
    w_proj = np.array([[c + 1, (-1) ** j * (j + 1) / 2] for c in range(6) for j in range(2)], F)
    got = O.timestep_modulation(np.array([0.0, 0.5]), w_t1, w_t2, w_proj, 4, 2)
    b0 = (0.49349197528601374, -0.2750881684806041)
    b1 = (-0.20447066856192508, -0.278298119967226)
    want = np.array([[[(c + 1) * b[0] + (-1) ** j * (j + 1) / 2 * b[1] for j in range(2)]
                      for c in range(6)] for b in (b0, b1)])
    assert got.shape == (2, 6, 2)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=0)
    # the first and last chunks, as listed above
    np.testing.assert_allclose(got[0, 0], [0.3559478910, 0.7685801438], atol=1e-9)
    np.testing.assert_allclose(got[0, 5], [2.8234077675, 3.2360400202], atol=1e-9)
    np.testing.assert_allclose(got[1, 0], [-0.3436197285, 0.0738274514], atol=1e-9)
    np.testing.assert_allclose(got[1, 5], [-1.3659730714, -0.9485258914], atol=1e-9)


# ---------------------------------------------------------------- bf16 storage emulation

# The device stores these activations as bf16, in this order, in one block:
# h (norm1 output), q, k, v (after QK-norm and RoPE), P of each head before
# P.V, o, x1, h2, g and x2. The emulation must round at exactly these points.
def test_emulation_rounds_at_the_device_storage_points():
    d = SMALL
    L = make_layout([("text", 0, 20), ("pad", 5), ("video", (2, 2, 4), 0, 2), ("audio", 0, 7)],
                    seed=[3])
    S, H, NH, D, Fd = L.S, d.hidden, d.heads, d.head_dim, d.ffn
    w = _weights_big_gates(d, 4)
    tmod = _tmod_random(L.n_t, H, 5)
    x = O.bf16_to_f64(f32_to_bf16_bits(np.random.default_rng(6).standard_normal((1, S, H))))
    seen = []
    base = O.round_bf16

    def spy(a):
        seen.append(np.shape(a))
        return base(a)

    O.round_bf16 = spy
    try:
        O.block_forward(x, w, L, tmod, d, emulate=False)
        assert seen == []
        O.block_forward(x, w, L, tmod, d, emulate=True)
    finally:
        O.round_bf16 = base
    want = ([(S, H), (S, NH, D), (S, NH, D), (S, NH, D)] + [(S, S)] * NH +
            [(S, NH * D), (S, H), (S, H), (S, Fd), (S, H)])
    assert seen == want


def test_emulated_attention_rounds_p_but_sums_unrounded_p():
    """One query, two keys, D = 1, so s = [0, ln p1] and the weights are
    [1, p1] with p1 = 0.50244140625 = 0.5 (1 + 2^-8 + 2^-10). bf16 keeps 7
    fraction bits: 1.0048828125 lies above the midpoint 1.00390625 between 1
    and 1.0078125, so P rounds to [1, 0.50390625]; the row sum l is taken
    from the unrounded weights, l = 1.50244140625 (the kernel adds fp32 p).

    (a) v = [0, v1] with the exact output p1 v1 / l = 1.00341796875, just below
        the midpoint 1.00390625: unrounded P would store o = 1.0; rounded P
        gives 1.00341796875 * 0.50390625 / 0.50244140625 = 1.006343..., stored
        as 1.0078125.
    (b) the rounded-P output p1r v1 / l = 1.00439453125, just above the
        midpoint: stored as 1.0078125; dividing by the sum of the rounded
        weights (1.50390625) instead would give 1.003417..., stored as 1.0.
    """
    p1, p1r, l = 0.50244140625, 0.50390625, 1.50244140625
    q = np.ones((1, 1, 1))
    k = np.array([0.0, math.log(p1)]).reshape(2, 1, 1)
    doc_q, doc_k = np.zeros(1, bool), np.zeros(2, bool)
    v1a = 1.00341796875 * l / p1
    va = np.array([0.0, v1a]).reshape(2, 1, 1)
    assert O.attention(q, doc_q, k, va, doc_k)[0, 0] == pytest.approx(1.00341796875, rel=1e-12)
    assert O.attention(q, doc_q, k, va, doc_k, emulate=True)[0, 0] == 1.0078125
    v1b = 1.00439453125 * l / p1r
    vb = np.array([0.0, v1b]).reshape(2, 1, 1)
    assert O.attention(q, doc_q, k, vb, doc_k, emulate=True)[0, 0] == 1.0078125
    assert O.round_bf16(np.array(p1r * v1b / (1 + p1r)))[()] == 1.0


def test_emulated_residual_rounds_after_the_add():
    """x1 = bf16(x + gate * (o W_o^T)): with x = 1, gate = 1 and a branch of
    2^-9 (exact in bf16), the sum 1.001953125 is below the midpoint 1.00390625
    and is stored as 1.0; a branch of 3 * 2^-9 gives 1.005859375, stored as
    1.0078125. Rounding the branch alone and adding it unrounded would keep
    1.001953125."""
    w_o = f32_to_bf16_bits(np.array([[2.0 ** -9]], np.float32))
    x = np.ones((1, 1))
    for o, want in ((1.0, 1.0), (3.0, 1.0078125)):
        got = O.out_project_residual(x, np.array([[o]]), np.ones((1, 1)), w_o, emulate=True)
        assert got[0, 0] == want
    got = O.out_project_residual(x, np.array([[1.0]]), np.ones((1, 1)), w_o, emulate=False)
    assert got[0, 0] == 1.001953125


# ---------------------------------------------------------------- the denoiser around the stack

def test_golden_denoiser_defaults_match_full_dims():
    g = _golden()
    d = FULL_DIMS
    assert d.in_channels == g["in_channels"] and d.audio_in_channels == g["audio_in_channels"]
    assert d.patch_size == (g["patch_size_t"], g["patch_size_h"], g["patch_size_w"])
    assert d.video_channels == g["video_row_channels"] == 96
    assert d.text_dim == g["text_dim"]
    assert d.num_refiner_layers == g["num_refiner_layers"]
    assert d.final_norm_eps == g["final_norm_eps"]


def test_timestep_embedding_worked_by_hand():
    """The same tiny prologue as test_timestep_modulation_worked_by_hand: the
    MLP output temb at t = 0 is [SiLU(1) - SiLU(0), -2 SiLU(1)]
    = [0.7310585786, -1.4621171573]; at t = 0.5, [-0.5637917047, -1.2397100173].
    The output modulation W_out . SiLU(temb) then follows from the SiLU values
    listed there."""
    w_t1 = np.array([[1, 0, 0, 0], [0, 0, 2, 100]], F)
    w_t2 = np.array([[1, -1], [-2, 0]], F)
    temb = O.timestep_embedding(np.array([0.0, 0.5]), w_t1, w_t2, 4)
    np.testing.assert_allclose(temb, [[0.7310585786, -1.4621171573],
                                      [-0.5637917047, -1.2397100173]], atol=1e-9)
    w_out = np.array([[1, 0], [0, 1], [1, 1], [2, -1]], F)  # 2 chunks of H = 2
    got = O.output_modulation(np.array([0.0, 0.5]), w_t1, w_t2, w_out, 4, 2)
    b0 = np.array([0.49349197528601374, -0.2750881684806041])
    b1 = np.array([-0.20447066856192508, -0.278298119967226])
    np.testing.assert_allclose(got, np.stack([(w_out @ b).reshape(2, 2) for b in (b0, b1)]),
                               rtol=1e-9)


def test_input_projections_match_torch_linear_and_a_hand_case():
    g = np.random.default_rng(41)
    lat = g.standard_normal((7, 96)).astype(np.float32)
    w = g.standard_normal((64, 96)).astype(np.float32)
    np.testing.assert_allclose(O.patch_project(lat, w), torch.nn.functional.linear(
        torch.tensor(lat, dtype=torch.float64), torch.tensor(w, dtype=torch.float64)).numpy(),
        rtol=1e-12, atol=1e-12)
    # by hand: rows [1, 2] and [0, -1] through [[1, 0], [1, 1], [0, 3]]
    np.testing.assert_array_equal(O.patch_project(np.array([[1.0, 2.0], [0.0, -1.0]]),
                                                  np.array([[1, 0], [1, 1], [0, 3]])),
                                  [[1, 3, 6], [0, -1, -3]])
    enc = f32_to_bf16_bits(np.array([[1.0, -2.0, 0.5]], np.float32))
    wt = f32_to_bf16_bits(np.array([[1, 1, 1], [2, 0, -4]], np.float32))
    np.testing.assert_array_equal(O.text_project(enc, wt), [[-0.5, 0.0]])


def _denoiser_case(seed=0, S=90):
    d = SMALL
    d = Dims(**dict(d.__dict__, text_dim=64, num_refiner_layers=2, in_channels=4,
                    audio_in_channels=8))
    L = random_layout(S, seed, pad_runs=2, max_run=9, n_t=4)
    g = np.random.default_rng([seed, 77])
    from types import SimpleNamespace
    H, E = d.hidden, d.time_embed_dim
    dw = SimpleNamespace(
        w_patch_video=g.standard_normal((H, d.video_channels)) * 0.2,
        w_patch_audio=g.standard_normal((H, d.audio_in_channels)) * 0.2,
        w_text=f32_to_bf16_bits((g.standard_normal((H, d.text_dim)) * 0.1).astype(np.float32)),
        refiner=[_weights_big_gates(d, 200 + i) for i in range(2)],
        w_t1=g.standard_normal((d.time_hidden, d.freq_dim)) * 0.05,
        w_t2=g.standard_normal((E, d.time_hidden)) * 0.05,
        w_proj=g.standard_normal((6 * H, E)) * 0.05,
        w_out=g.standard_normal((2 * H, E)) * 0.05,
        out_table=g.standard_normal((2, 2, H)) * 0.2,
        w_head_video=g.standard_normal((d.video_channels, H)) * 0.1,
        w_head_audio=g.standard_normal((d.audio_in_channels, H)) * 0.1)
    blocks = [_weights_big_gates(d, 300 + i) for i in range(2)]
    video = g.standard_normal((len(L.video_idx), d.video_channels))
    audio = g.standard_normal((len(L.audio_idx), d.audio_in_channels))
    text = f32_to_bf16_bits(g.standard_normal((len(L.text_idx), d.text_dim)).astype(np.float32))
    return d, L, dw, blocks, video, audio, text


def test_output_head_is_layer_norm_modulate_then_linear():
    g = np.random.default_rng(9)
    x = g.standard_normal((5, 32)) * 3 + 1
    sh, sc = g.standard_normal((5, 32)), g.standard_normal((5, 32))
    w = g.standard_normal((6, 32))
    xt = torch.tensor(x)
    ln = torch.nn.functional.layer_norm(xt, (32,), eps=1e-5)
    ref = torch.nn.functional.linear(ln * (1 + torch.tensor(sc)) + torch.tensor(sh),
                                     torch.tensor(w)).numpy()
    np.testing.assert_allclose(O.output_head(x, sh, sc, w, 1e-5), ref, rtol=1e-10, atol=1e-12)
    # a constant row normalises to 0, so the head sees only the shift
    c = np.full((1, 32), 2.5)
    np.testing.assert_allclose(O.output_head(c, sh[:1], sc[:1], w, 1e-5), sh[:1] @ w.T,
                               atol=1e-9)


def test_refiner_attends_text_rows_only_and_ends_in_a_layer_norm():
    d, L, dw, blocks, video, audio, text = _denoiser_case(1)
    H = d.hidden
    tmod = O.timestep_modulation(L.timestep, dw.w_t1, dw.w_t2, dw.w_proj, d.freq_dim, H)
    xt = O.text_project(text, dw.w_text)
    got = O.refine_text(xt, dw.refiner, L, tmod, d, 1e-5)
    # the refiner's blocks equal the block run on the text rows as a sequence of their own
    ti = L.text_idx
    Lt = make_layout([("text", 0, len(ti))], timesteps="given", t_values=L.timestep,
                     t_idx=L.t_idx[ti])
    Lt.pos = L.pos[ti]
    y = xt[None]
    for w in dw.refiner:
        y = O.block_forward(y, w, Lt, tmod, d)
    np.testing.assert_allclose(got, torch.nn.functional.layer_norm(
        torch.tensor(y[0]), (H,), eps=1e-5).numpy(), rtol=1e-10, atol=1e-12)
    # zero gates in the refiner blocks: the output is the LayerNorm of the projection
    z = [dataclasses_replace_gates(w) for w in dw.refiner]
    tz = tmod.copy()
    tz[:, [2, 5]] = 0.0
    np.testing.assert_allclose(O.refine_text(xt, z, L, tz, d, 1e-5), O.layer_norm(xt, 1e-5),
                               rtol=1e-12, atol=1e-12)


def dataclasses_replace_gates(w):
    import copy
    w = copy.copy(w)
    w.ada_table = np.array(w.ada_table, copy=True)
    w.ada_table[:, [2, 5]] = 0.0
    return w


def test_denoiser_with_identity_blocks_is_head_of_normed_projection():
    """With every gate zero (refiner and stack blocks, table and tmod), the
    blocks pass x through, so the velocity of a video row is the head applied
    to norm_out of its patch projection: rebuilt here from torch CPU ops."""
    d, L, dw, blocks, video, audio, text = _denoiser_case(2)
    dw.refiner = [dataclasses_replace_gates(w) for w in dw.refiner]
    blocks = [dataclasses_replace_gates(w) for w in blocks]
    dw.w_proj = np.array(dw.w_proj, copy=True)
    H = d.hidden
    for c in (2, 5):
        dw.w_proj[c * H:(c + 1) * H] = 0.0
    vv, va = O.denoiser_forward(video, audio, text, dw, lambda i: blocks[i], 2, L, d, 1e-5)
    tmo = torch.tensor(O.output_modulation(L.timestep, dw.w_t1, dw.w_t2, dw.w_out, d.freq_dim,
                                           H))
    for lat, idx, m, wp, wh, got in ((video, L.video_idx, 0, dw.w_patch_video, dw.w_head_video, vv),
                                     (audio, L.audio_idx, 1, dw.w_patch_audio, dw.w_head_audio, va)):
        x = torch.nn.functional.linear(torch.tensor(lat), torch.tensor(wp))
        mod = torch.tensor(dw.out_table)[m][None] + tmo[torch.tensor(L.t_idx[idx]).long()]
        h = torch.nn.functional.layer_norm(x, (H,), eps=1e-5) * (1 + mod[:, 1]) + mod[:, 0]
        ref = torch.nn.functional.linear(h, torch.tensor(wh)).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-11)


def test_denoiser_rows_permute_with_their_layout_and_padding_is_inert():
    d, L, dw, blocks, video, audio, text = _denoiser_case(3)
    run = lambda L_: O.denoiser_forward(video, audio, text, dw, lambda i: blocks[i], 2, L_, d, 1e-5)
    vv, va = run(L)
    assert np.linalg.norm(vv) > 0 and np.linalg.norm(va) > 0
    perm = np.random.default_rng(5).permutation(L.S)
    inv = np.argsort(perm)
    Lp = type(L)(tags=L.tags[perm], pos=L.pos[perm], t_idx=L.t_idx[perm], timestep=L.timestep,
                 video_idx=inv[L.video_idx].astype(np.int32),
                 audio_idx=inv[L.audio_idx].astype(np.int32),
                 text_idx=inv[L.text_idx].astype(np.int32))
    vp, ap = run(Lp)
    np.testing.assert_allclose(vp, vv, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(ap, va, rtol=1e-9, atol=1e-11)
    # padding rows: new positions and timestep indices change nothing
    Lq = type(L)(tags=L.tags, pos=L.pos.copy(), t_idx=L.t_idx.copy(), timestep=L.timestep,
                 video_idx=L.video_idx, audio_idx=L.audio_idx, text_idx=L.text_idx)
    pad = L.tags < 0
    assert pad.any()
    Lq.pos[pad] = 17.0
    Lq.t_idx[pad] = 3
    vq, aq = run(Lq)
    np.testing.assert_array_equal(vq, vv)
    np.testing.assert_array_equal(aq, va)


# ---------------------------------------------------------------- token reduction

def test_reduction_pairs_by_hand():
    """A (1, 2, 5) target grid: in each of the two h rows, w = (0, 1) and
    (2, 3) pair and w = 4 stays single; a conditioning frame, text, audio and a
    pair across different timesteps never pair."""
    L = make_layout([("text", 0, 3), ("video", (2, 2, 5), 0, 2), ("audio", 0, 4)],
                    timesteps="given", t_values=np.array([0.0, 0.5], np.float32),
                    t_idx=np.zeros(27, np.int32))
    target = (L.tags == 0) & (L.pos[:, 0] == 1)   # frame 1 is the target, frame 0 a reference
    heads = O.reduction_pairs(L, target)
    # rows: text 0..2, frame 0 at 3..12, frame 1 at 13..22 (h 0: 13..17, h 1: 18..22)
    np.testing.assert_array_equal(heads, [13, 15, 18, 20])
    red, rows = O.reduced_layout(L, heads)
    assert red.S == 27 - 4
    j = int(np.nonzero(rows[:, 0] == 13)[0][0])
    assert rows[j, 1] == 14 and np.allclose(red.pos[j], [1, 0, 0.5])
    L.t_idx[14] = 1  # the second row of the first pair moves to another timestep
    np.testing.assert_array_equal(O.reduction_pairs(L, target), [15, 18, 20])
    assert O.reduction_pairs(L, np.zeros(L.S, bool)).size == 0


def test_merge_and_restore():
    g = np.random.default_rng(3)
    x = g.standard_normal((6, 4))
    rows = np.array([[0, 1], [2, -1], [3, 4], [5, -1]])
    m = O.merge_rows(x, rows)
    np.testing.assert_allclose(m[0], 0.5 * (x[0] + x[1]))
    np.testing.assert_array_equal(m[1], x[2])
    # no change in the reduced rows restores the bypass exactly
    np.testing.assert_allclose(O.restore_rows(x, m, rows), x, rtol=0, atol=1e-15)
    # a change of a merged row reaches both rows of its pair
    d = np.zeros_like(m)
    d[2] = [1, 2, 3, 4]
    out = O.restore_rows(x, m + d, rows)
    np.testing.assert_allclose(out[3] - x[3], [1, 2, 3, 4], atol=1e-14)
    np.testing.assert_allclose(out[4] - x[4], [1, 2, 3, 4], atol=1e-14)
    np.testing.assert_allclose(np.delete(out, [3, 4], 0), np.delete(x, [3, 4], 0), atol=1e-15)


def _reduction_case(seed=0):
    segs = [("text", 0, 9), ("video", (3, 2, 6), 0, 3), ("pad", 5), ("audio", 0, 11)]
    L0 = make_layout(segs, seed=[seed])
    target = (L0.tags == 0) & (L0.pos[:, 0] >= 1)  # video frames 1, 2; frame 0 a reference
    t_idx = (target | (L0.tags == 2)).astype(np.int32)
    L = make_layout(segs, timesteps="given", t_values=np.array([0.0, 0.6], np.float32),
                    t_idx=t_idx)
    assert O.reduction_pairs(L, target).size == 12
    ws = [_weights_big_gates(SMALL, 40 + i) for i in range(4)]
    tmod = _tmod_random(L.n_t, SMALL.hidden, seed)
    x = O.bf16_to_f64(f32_to_bf16_bits(np.random.default_rng([seed, 1]).standard_normal(
        (1, L.S, SMALL.hidden)).astype(np.float32)))
    return L, target, ws, tmod, x


def test_reduced_stack_without_reduction_is_the_stack():
    L, target, ws, tmod, x = _reduction_case(1)
    full = O.stack_forward(x, lambda i: ws[i], 4, L, tmod, SMALL)
    np.testing.assert_array_equal(
        O.stack_forward_reduced(x, lambda i: ws[i], 4, L, tmod, SMALL, target, 2, 2), full)
    # no target rows: every row maps to itself, and the restore x + (x_red - x)
    # gives x_red up to the rounding of that sum
    np.testing.assert_allclose(
        O.stack_forward_reduced(x, lambda i: ws[i], 4, L, tmod, SMALL, np.zeros(L.S, bool), 1, 3),
        full, rtol=1e-12, atol=1e-12)
    red = O.stack_forward_reduced(x, lambda i: ws[i], 4, L, tmod, SMALL, target, 1, 3)
    assert _rel(red, full) > 1e-3  # the reduction changes the result
    pad = L.tags < 0
    np.testing.assert_array_equal(red[0, pad], x[0, pad])


def test_reduced_blocks_with_zero_gates_restore_the_bypass():
    """Reduced blocks whose gates are all zero leave the merged rows unchanged, so
    the restore gives back the bypass exactly, and the stack equals the full
    stack without those blocks."""
    import copy
    L, target, ws, tmod, x = _reduction_case(2)
    z = []
    for w in ws:
        w = copy.copy(w)
        w.ada_table = np.array(w.ada_table, copy=True)
        z.append(w)
    for i in (1, 2):
        z[i].ada_table[:, [2, 5]] = 0.0
    tz = tmod.copy()
    tz[:, [2, 5]] = 0.0
    got = O.stack_forward_reduced(x, lambda i: z[i], 3, L, tz, SMALL, target, 1, 3)
    ref = O.block_forward(x, z[0], L, tz, SMALL)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_reduced_stack_one_pair_by_hand():
    """Two target rows that pair and nothing else: the reduced block sees one
    row (a document of one key: its attention output is its own v), and the
    restore adds that row's update to both rows."""
    L = make_layout([("video", (1, 1, 2), 0, 1)], timesteps="given",
                    t_values=np.array([0.5], np.float32), t_idx=np.zeros(2, np.int32))
    target = np.ones(2, bool)
    w = _weights_big_gates(SMALL, 9)
    tmod = _tmod_random(1, SMALL.hidden, 9)
    x = np.random.default_rng(4).standard_normal((1, 2, SMALL.hidden))
    got = O.stack_forward_reduced(x, lambda i: w, 1, L, tmod, SMALL, target, 0, 1)
    m = 0.5 * (x[0, 0] + x[0, 1])
    Lm = make_layout([("video", (1, 1, 1), 0, 1)], timesteps="given",
                     t_values=np.array([0.5], np.float32), t_idx=np.zeros(1, np.int32))
    Lm.pos[0] = [0.0, 0.0, 0.5]
    y = O.block_forward(m[None, None], w, Lm, tmod, SMALL)[0, 0]
    np.testing.assert_allclose(got[0, 0], x[0, 0] + (y - m), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got[0, 1], x[0, 1] + (y - m), rtol=1e-12, atol=1e-12)


def test_core_reuse_with_the_same_latents_is_the_full_forward():
    """Reusing the core residual of a forward for the same latents gives that
    forward's velocities (the residual is the stack's output minus its input);
    with fresh latents only the projections and heads change."""
    d, L, dw, blocks, video, audio, text = _denoiser_case(4)
    res = np.zeros((L.S, d.hidden))
    vv, va = O.denoiser_forward(video, audio, text, dw, lambda i: blocks[i], 2, L, d, 1e-5,
                                core_residual=res)
    assert np.linalg.norm(res) > 0
    rv, ra = O.denoiser_forward(video, audio, text, dw, lambda i: blocks[i], 2, L, d, 1e-5,
                                core_residual=res, reuse=True)
    np.testing.assert_allclose(rv, vv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ra, va, rtol=1e-12, atol=1e-12)
    # fresh latents: head(norm_out(projection + residual)), rebuilt by hand
    v2 = video * 0.5 + 0.1
    rv2, _ = O.denoiser_forward(v2, audio, text, dw, lambda i: blocks[i], 2, L, d, 1e-5,
                                core_residual=res, reuse=True)
    tmo = O.output_modulation(L.timestep, dw.w_t1, dw.w_t2, dw.w_out, d.freq_dim, d.hidden)
    m = np.asarray(dw.out_table)[0][None] + tmo[L.t_idx[L.video_idx]]
    xr = v2 @ np.asarray(dw.w_patch_video).T + res[L.video_idx]
    np.testing.assert_allclose(rv2, O.output_head(xr, m[:, 0], m[:, 1], dw.w_head_video, 1e-5),
                               rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- 8-bit GEMM inputs

def test_e4m3_rounding_matches_torch_and_the_format():
    """In-range values against torch's float8_e4m3fn conversion (round to
    nearest even), plus the format's landmarks by hand: 448 the largest finite
    value, 2^-9 the smallest subnormal, steps of 2^(k-3) in [2^k, 2^(k+1))."""
    g = np.random.default_rng(8)
    x = np.concatenate([g.standard_normal(20000) * 50, g.uniform(-448, 448, 20000),
                        g.standard_normal(5000) * 0.01, np.linspace(-3, 3, 4001)])
    ref = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3_round(x.astype(np.float32)), ref)
    assert O.e4m3_round(np.array([500.0, -1e6]))[0] == 448.0
    assert O.e4m3_round(np.array([-1e6]))[0] == -448.0
    np.testing.assert_array_equal(O.e4m3_round(np.array([2.0 ** -9, 2.0 ** -10, 1.5 * 2.0 ** -10])),
                                  [2.0 ** -9, 0.0, 2.0 ** -9])
    # 1.0625 is halfway between 1 and 1.125: ties to the even code (1.0)
    np.testing.assert_array_equal(O.e4m3_round(np.array([1.0625, 1.1875, 17.0, 19.0])),
                                  [1.0, 1.25, 16.0, 20.0])


def test_e4m3_decode_matches_torch_on_every_byte():
    """All 256 code bytes against torch's float8_e4m3fn reinterpretation; every
    finite code's value lies on the e4m3 grid (e4m3_round keeps it); the NaN
    codes are 0x7F and 0xFF only; the largest finite value is 448."""
    b = np.arange(256, dtype=np.uint8)
    got = O.e4m3_decode(b)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(got[fin], ref[fin])
    assert set(np.nonzero(np.isnan(got))[0]) == {0x7F, 0xFF}
    np.testing.assert_array_equal(O.e4m3_round(got[fin]), got[fin])
    assert np.nanmax(got) == 448.0 and O.e4m3_decode(np.array([1]))[0] == 2.0 ** -9
    assert np.signbit(O.e4m3_decode(np.array([0x80]))[0])


def test_row_quantization_round_trip():
    g = np.random.default_rng(9)
    a = (g.standard_normal((7, 300)) * np.array([1e-3, 1, 30, 0, 5, 1e4, 2])[:, None])
    codes, s = O.quantize_rows_e4m3(a)
    assert s.dtype == np.float32 and s[3] == 1.0 and np.all(codes[3] == 0)
    assert np.all(np.abs(codes) <= 448) and np.all(np.max(np.abs(codes), 1)[[0, 1, 2, 4, 5, 6]] == 448)
    back = O.dequantize_rows(codes, s)
    ok = np.abs(a) > 2.0 ** -6 * s[:, None]  # normal range: relative error <= 2^-4
    assert np.all(np.abs(back - a)[ok] <= 2.0 ** -4 * np.abs(a)[ok] * (1 + 1e-6))


def test_fp8_block_is_close_to_the_block_and_keeps_padding():
    """The 8-bit block moves x like the block, within the quantization error
    (a few % of the update), and leaves padding rows unchanged."""
    L = random_layout(64, 3, pad_runs=2, max_run=9)
    w = _weights_big_gates(SMALL, 12)
    tmod = _tmod_random(L.n_t, SMALL.hidden, 4)
    x = np.random.default_rng(5).standard_normal((1, L.S, SMALL.hidden))
    y = O.block_forward(x, w, L, tmod, SMALL)
    y8 = O.block_forward_fp8(x, w, L, tmod, SMALL)
    pad = L.tags < 0
    np.testing.assert_array_equal(y8[0, pad], x[0, pad])
    d, d8 = y[0, ~pad] - x[0, ~pad], y8[0, ~pad] - x[0, ~pad]
    r = _rel(d8, d)
    assert 1e-3 < r < 0.08, r
    # with the O and W2 inputs in 8 bits too: still near the block, a little
    # further from it, padding unchanged
    y8a = O.block_forward_fp8(x, w, L, tmod, SMALL, out_down=True)
    np.testing.assert_array_equal(y8a[0, pad], x[0, pad])
    ra = _rel(y8a[0, ~pad] - x[0, ~pad], d)
    assert r < ra < 0.1, (r, ra)
