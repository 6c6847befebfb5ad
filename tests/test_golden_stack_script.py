"""The config-5 golden script's head-parallel attention equals the oracle's
attention, and its row sample covers every padding edge and mixed tile.

Source: "MiniMaxH3Transformer3DModel" (diffusers v0.43.0 docs), overview:
every head attends over the row's document independently; padding rows form
their own document.
"""

import numpy as np

from oracle import h3_oracle as O
from tests.golden.make_stack_config5_golden import head_parallel_attention, sample_rows
from workloads import config_layout, random_layout


def test_head_parallel_attention_equals_oracle():
    g = np.random.default_rng(11)
    for n, S, NH, workers in ((7, 19, 5, 2), (300, 40, 11, 4), (16, 16, 3, 8)):
        q = g.standard_normal((n, NH, 128))
        k = g.standard_normal((S, NH, 128))
        v = g.standard_normal((S, NH, 128))
        dk = g.random(S) < 0.2
        dq = g.random(n) < 0.2
        dk[0], dk[1] = False, True
        ref = O.attention(q, dq, k, v, dk)
        got = head_parallel_attention(workers)(q, dq, k, v, dk)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_head_parallel_block_equals_oracle_block():
    from workloads import TINY_DIMS, activations, block_weights, prologue_weights
    dims = TINY_DIMS
    L = config_layout(1)
    w = block_weights(dims, 1, 0)
    pw = prologue_weights(dims, 1)
    x = O.bf16_to_f64(activations(dims, 1, L.S))
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim,
                               dims.hidden)
    ref = O.block_forward(x, w, L, tm, dims)
    base = O.attention
    try:
        O.attention = head_parallel_attention(4)
        got = O.block_forward(x, w, L, tm, dims)
    finally:
        O.attention = base
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_sample_rows_cover_padding_edges_and_mixed_tiles():
    L = config_layout(5)
    rows = sample_rows(L)
    assert 64 <= rows.size <= 80 and np.all(np.diff(rows) > 0)
    pad = L.tags < 0
    edges = np.nonzero(np.diff(pad.astype(np.int8)))[0]
    for e in edges:
        assert e in rows and e + 1 in rows
    assert pad[rows].sum() >= 7 and (~pad[rows]).sum() >= 50
    for tag in (0, 1, 2):
        assert np.any(L.tags[rows] == tag)
    # rows of both mixed tiles (7 and 8: the first padding run straddles them)
    assert np.any((rows >= 896) & (rows < 960)) and np.any((rows >= 1088) & (rows < 1152))
    L2 = random_layout(500, 3, pad_runs=3)
    assert sample_rows(L2).size >= 64


def test_head_parallel_pieces_keep_the_bf16_storage_emulation():
    """The --emulate golden: the pieces pass the emulation through (P rounded
    per row, as the whole attention does), and the block in its bf16-storage,
    fp32-stream reading is unchanged by the piecewise attention."""
    g = np.random.default_rng(12)
    q = g.standard_normal((40, 3, 128))
    k = g.standard_normal((33, 3, 128))
    v = g.standard_normal((33, 3, 128))
    dk = g.random(33) < 0.2
    dq = g.random(40) < 0.2
    dk[0], dk[1] = False, True
    ref = O.attention(q, dq, k, v, dk, emulate=True)
    got = head_parallel_attention(3, q_chunk=16)(q, dq, k, v, dk, emulate=True)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    assert not np.allclose(ref, O.attention(q, dq, k, v, dk), rtol=1e-6)  # emulation is on

    from workloads import TINY_DIMS, activations, block_weights, prologue_weights
    dims = TINY_DIMS
    L = config_layout(1)
    w = block_weights(dims, 1, 0)
    pw = prologue_weights(dims, 1)
    x = O.bf16_to_f64(activations(dims, 1, L.S))
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim,
                               dims.hidden)
    ref = O.block_forward(x, w, L, tm, dims, emulate=True, stream_f32=True)
    base = O.attention
    try:
        O.attention = head_parallel_attention(4)
        got = O.block_forward(x, w, L, tm, dims, emulate=True, stream_f32=True)
    finally:
        O.attention = base
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)
    # the fp32 stream: x1 and the output are fp32 values, not bf16 ones
    assert np.array_equal(got, got.astype(np.float32).astype(np.float64))
    assert not np.array_equal(got, O.round_bf16(got))
