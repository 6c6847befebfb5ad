"""The 8-bit (e4m3) QKV and W1 || W3 GEMM inputs on the GPU against the oracle.

Source: "MiniMax H3 Inference Engine voor Mac computers", sections "Profiling
en diagnostische pads" and "Sampler en DiT controls" (8-bit MLP and QKV
projections, one activation scale per row). The oracle quantizes at the same
points (oracle.h3_oracle.block_forward_fp8), so the GPU block is held to the
same tolerance as the bf16 block against it; the weight codes and scales, whose
inputs are exact on both sides, are compared bit for bit.

Each 8-bit step through its own entry point: the GEMM steps on the same codes
on both sides (random code bytes and scales from the input generator, decoded
by the oracle) at the block's tolerance; the norm + quantize step bit for bit
on its codes, except at near-ties, where each differing code is checked to be
the other neighbour of a value that lies next to the midpoint between two e4m3
values: within 2^-14 relative plus the fp32 rounding of h's two terms (the
device forms h in fp32, the oracle in float64 then rounded to fp32).

The whole 8-bit block is not a continuous function of its rounded
intermediates: an e4m3 code is an integer decided by floating point, one code
step is 6-12 % of a value, and a one-ulp change of a stored bf16 x1 element can
move an h2 code by a step, which moves that row's FFN output. The block is
compared with the oracle's 8-bit block in its bf16-storage emulation (bf16 where
the device stores bf16; h and h2 go from fp32 straight to codes on both sides,
o and g are quantized from their bf16 values): rel-L2 on x_out and on the update
within 1e-2, and the largest difference within 5e-2, each plus the spread of the
oracle itself between its two storage readings (float64 and emulated bf16
intermediates), which measures how far code flips alone move this output. With
QKV and W1 || W3 in 8 bits that spread is ~1 % (rel-L2 of x_out) on the
amplified cases; with O and W2 too, ~2 %.
"""

import numpy as np
import pytest
import torch

from audio_generation_b200 import h3
from oracle import h3_oracle as O
from tests.h3_testlib import (MAX_ABS, REL_L2, DevLayout, DevWeights, assert_close, dev_bf16,
                              dev_f32, host_bits, host_f64, rel_l2)
from tests.test_gpu_block import amplified_weights, gpu_tmod
from workloads import (FULL_DIMS, TINY_DIMS, Dims, activations, block_weights, config_layout,
                       f32_to_bf16_bits, make_layout, normal_bf16, prologue_weights,
                       random_code_bytes, random_layout, random_scales)

pytestmark = pytest.mark.gpu


def gpu_codes(w_bits):
    rows, K = w_bits.shape
    codes = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, dtype=torch.float32, device="cuda")
    h3.h3_quantize_e4m3_rows(dev_bf16(w_bits), rows, K, codes, scales)
    return codes, scales


def test_weight_codes_and_scales_bit_exact():
    g = np.random.default_rng(3)
    w = g.standard_normal((37, 512)).astype(np.float32) * np.geomspace(1e-4, 30, 37)[:, None]
    w[5] = 0.0
    w[9, 17] = 1e4  # one large entry sets its row's scale
    bits = f32_to_bf16_bits(w)
    codes, scales = gpu_codes(bits)
    torch.cuda.synchronize()
    got = codes.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()
    ref_codes, ref_scales = O.quantize_rows_e4m3(O.bf16_to_f64(bits).astype(np.float32))
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_scales)
    np.testing.assert_array_equal(got, ref_codes)


SMALL = Dims(hidden=256, heads=2, head_dim=128, ffn=384, time_embed_dim=64, time_hidden=128)
STEP_CASES = {
    "small_rand333_B2": (SMALL, lambda: random_layout(333, 5, pad_runs=3, max_run=70), 2),
    "full_rand300": (FULL_DIMS, lambda: random_layout(300, 6, pad_runs=2, max_run=50), 1),
}


def _dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def _codes_and_scales(rows, K, seed, lo, hi):
    return random_code_bytes((rows, K), [seed, rows, K]), random_scales(rows, [seed, 1], lo, hi)


def _values(codes, scales):
    return O.e4m3_decode(codes) * scales.astype(np.float64)[:, None]


@pytest.mark.parametrize("case", list(STEP_CASES))
def test_qkv_rope_e4m3_step(case):
    dims, mk, B = STEP_CASES[case]
    L = mk()
    dl = DevLayout(dims, L)
    w = block_weights(dims, 51, 0)
    H, NH, D, S = dims.hidden, dims.heads, dims.head_dim, L.S
    hc, hs = _codes_and_scales(B * S, H, 21, -9.0, -6.0)
    wc, wsc = _codes_and_scales(3 * NH * D, H, 22, -16.0, -12.0)
    q = torch.empty((B, NH, S, D), dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    h3.h3_qkv_rope_e4m3(dl.dims, dl.handle, B, _dev_u8(hc), dev_f32(hs), _dev_u8(wc),
                        dev_f32(wsc), dev_bf16(w.q_norm), dev_bf16(w.k_norm), q, k, v)
    torch.cuda.synchronize()
    hv, wv = _values(hc, hs), _values(wc, wsc)
    for b in range(B):
        rq, rk, rv = O.qkv_project_values(hv[b * S:(b + 1) * S], L.pos, wv, w.q_norm, w.k_norm,
                                          dims)
        for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
            g = host_f64(got[b]).transpose(1, 0, 2)
            assert_close(g, ref, what=f"e4m3 {name} b={b}", storage_rounding=True)


@pytest.mark.parametrize("case", list(STEP_CASES))
def test_ffn_up_e4m3_step(case):
    dims, mk, B = STEP_CASES[case]
    L = mk()
    dl = DevLayout(dims, L)
    H, Fd, S = dims.hidden, dims.ffn, L.S
    hc, hs = _codes_and_scales(B * S, H, 23, -9.0, -6.0)
    wc, wsc = _codes_and_scales(2 * Fd, H, 24, -16.0, -12.0)
    g = torch.empty((B, S, Fd), dtype=torch.bfloat16, device="cuda")
    h3.h3_ffn_up_e4m3(dl.dims, dl.handle, B, _dev_u8(hc), dev_f32(hs), _dev_u8(wc), dev_f32(wsc),
                      g)
    torch.cuda.synchronize()
    got = host_f64(g)
    hv, wv = _values(hc, hs), _values(wc, wsc)
    for b in range(B):
        ref = O.ffn_gate_values(hv[b * S:(b + 1) * S], wv, Fd)
        assert_close(got[b], ref, what=f"e4m3 g b={b}", storage_rounding=True)


@pytest.mark.parametrize("case", list(STEP_CASES))
@pytest.mark.parametrize("which", ["out", "down"])
def test_residual_e4m3_steps(case, which):
    """h3_out_residual_e4m3 / h3_ffn_down_residual_e4m3 on the same random codes
    on both sides, the gated residual as in the bf16 steps."""
    dims, mk, B = STEP_CASES[case]
    L = mk()
    dl = DevLayout(dims, L)
    w = block_weights(dims, 53, 0)
    H, S = dims.hidden, L.S
    K = dims.attn_width if which == "out" else dims.ffn
    ac, asc = _codes_and_scales(B * S, K, 27, -8.0, -7.0)
    # uniform code bytes have rms value ~100: weight scales ~1 / (55 sqrt(K)) make
    # the update O(1), far above the bf16 rounding of the stored x
    hi = -float(np.log2(55.0 * np.sqrt(K)))
    wc, wsc = _codes_and_scales(H, K, 28, hi - 1.0, hi)
    xb = normal_bf16((B, S, H), [29, S], 1.0)
    tm = (np.random.default_rng([30, S]).standard_normal((L.n_t, 6, H))).astype(np.float32)
    x = dev_bf16(xb)
    fn = h3.h3_out_residual_e4m3 if which == "out" else h3.h3_ffn_down_residual_e4m3
    fn(dl.dims, dl.handle, B, _dev_u8(ac), dev_f32(asc), _dev_u8(wc), dev_f32(wsc),
       dev_f32(w.ada_table), dev_f32(tm), x)
    torch.cuda.synchronize()
    got = host_f64(x)
    m = O.row_modulation(L.tags, L.t_idx, w.ada_table, tm)
    av, wv = _values(ac, asc), _values(wc, wsc)
    valid = L.tags >= 0
    for b in range(B):
        x0 = O.bf16_to_f64(xb[b])
        a = av[b * S:(b + 1) * S]
        ref = (O.out_project_residual_values(x0, a, m[:, 2], wv) if which == "out"
               else O.ffn_down_residual_values(x0, a, m[:, 5], wv))
        assert_close(got[b, valid], ref[valid], what=f"e4m3 {which} x", storage_rounding=True)
        assert_close(got[b, valid] - x0[valid], ref[valid] - x0[valid], what=f"e4m3 {which} update",
                     mabs=np.inf)
        np.testing.assert_array_equal(host_bits(x)[b, ~valid], xb[b, ~valid])


def _check_codes_near_ties(got_bytes, got_scales, h, shift, scale, valid, tie_rel=2.0 ** -14,
                           err=2.0 ** -16):
    """Codes and scales of the valid rows against the oracle's quantization of h
    (float64, taken to fp32 as the device holds it). The device forms
    h = (x - mean) rstd (1 + scale) + shift in fp32 with its row statistics
    summed in fp32 over H / 32 terms per lane: its absolute error is bounded by
    err (2^-16, ~170 terms of 2^-24 each) times |1 + scale| (the mean's error,
    carried by rstd), |h - shift| (the rstd's relative error) and |shift|; this
    matters where the terms nearly cancel. tie_rel covers the scale's own
    relative error."""
    ref_vals, ref_s = O.quantize_rows_e4m3(h[valid])
    np.testing.assert_allclose(got_scales[valid], ref_s, rtol=2.0 ** -18, atol=0)
    got_vals = O.e4m3_decode(got_bytes[valid])
    assert not np.isnan(got_vals).any()
    diff = got_vals != ref_vals
    n = int(diff.sum())
    assert n <= max(8, 1e-3 * diff.size), f"{n} of {diff.size} codes differ"
    if n:
        t = (np.asarray(h[valid], np.float32) / ref_s[:, None]).astype(np.float64)[diff]
        a, r = got_vals[diff], ref_vals[diff]
        # adjacent grid values: rounding the midpoint's neighbourhood gives each
        mid = 0.5 * (a + r)
        hv, sv, cv = h[valid], shift[valid], scale[valid]
        abs_err = (err * (np.abs(1.0 + cv) + np.abs(hv - sv) + np.abs(sv)) / ref_s[:, None])[diff]
        far = np.abs(t - mid) > tie_rel * np.abs(mid) + abs_err
        assert not far.any(), (f"{int(far.sum())} of {n} differing codes are not near-ties: t "
                               f"{t[far][:4]}, codes {a[far][:4]} vs {r[far][:4]}, allowed "
                               f"{(tie_rel * np.abs(mid) + abs_err)[far][:4]}")
        lo, hi = np.minimum(a, r), np.maximum(a, r)
        assert np.all(O.e4m3_round(0.5 * (lo + mid)) == lo) and np.all(O.e4m3_round(0.5 * (hi + mid)) == hi)
    return n


@pytest.mark.parametrize("case", list(STEP_CASES))
@pytest.mark.parametrize("which", [0, 1])
def test_norm_modulate_e4m3_step(case, which):
    dims, mk, B = STEP_CASES[case]
    L = mk()
    dl = DevLayout(dims, L)
    w = block_weights(dims, 52, 0)
    H, S = dims.hidden, L.S
    xb = normal_bf16((B, S, H), [25, which, S], 1.5, 0.3)
    tm = (np.random.default_rng([26, which]).standard_normal((L.n_t, 6, H)) * 0.5
          ).astype(np.float32)
    codes = torch.empty((B * S, H), dtype=torch.uint8, device="cuda")
    scales = torch.empty(B * S, dtype=torch.float32, device="cuda")
    h3.h3_norm_modulate_e4m3(dl.dims, dl.handle, B, which, dev_bf16(xb), dev_f32(w.ada_table),
                             dev_f32(tm), codes, scales)
    torch.cuda.synchronize()
    cb = codes.cpu().numpy().reshape(B, S, H)
    sc = scales.cpu().numpy().reshape(B, S)
    m = O.row_modulation(L.tags, L.t_idx, w.ada_table, tm)
    c = 3 * which
    valid = L.tags >= 0
    for b in range(B):
        h = O.norm_modulate(O.bf16_to_f64(xb[b]), m[:, c], m[:, c + 1], dims.norm_eps)
        _check_codes_near_ties(cb[b], sc[b], h, m[:, c], m[:, c + 1], valid)
        assert np.all(cb[b, ~valid] == 0) and np.all(sc[b, ~valid] == 1.0)


class Spread:
    """How far the oracle's 8-bit block moves between its two storage readings
    (float64 intermediates, and bf16 where the device stores bf16): on x_out
    (rel-L2, max-abs) and on the update x_out - x_in of the valid rows (rel-L2)."""

    def __init__(self, ref_emulated, ref_float64, x0, valid):
        e, n = ref_emulated, ref_float64
        self.rel = rel_l2(n, e)
        self.max = float(np.max(np.abs(n - e))) if e.size else 0.0
        self.upd = rel_l2(n[valid] - x0[valid], e[valid] - x0[valid]) if valid.any() else 0.0


def assert_close_flips(got, ref, spread, what, storage_rounding=False):
    """The 8-bit block's bound (see the module docstring): rel-L2 and max-abs
    within the bar (1e-2, 5e-2) plus the oracle's own spread between its storage
    readings. (A flipped code moves a whole output row, so no per-element
    quantile is asked for.)"""
    r = rel_l2(got, ref)
    d = np.abs(got - ref)
    if storage_rounding:
        d = d - 2.0 ** -8 * np.abs(ref)
    m = float(d.max()) if d.size else 0.0
    rows = int((d.max(axis=-1) > MAX_ABS).sum()) if d.size else 0
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert r <= REL_L2 + spread.rel and m <= MAX_ABS + spread.max, (
        f"{what}: rel-L2 {r:.3e} (<= {REL_L2} + spread {spread.rel:.3e}), max-abs {m:.3e} "
        f"(<= {MAX_ABS} + spread {spread.max:.3e}); {rows} of {d.shape[0]} rows beyond {MAX_ABS}")


class E4m3Weights:
    def __init__(self, w, out_down=False):
        self.qkv = gpu_codes(w.w_qkv)
        self.w13 = gpu_codes(w.w13)
        extra = []
        if out_down:
            self.wo, self.w2 = gpu_codes(w.w_o), gpu_codes(w.w2)
            extra = [self.wo[0], self.wo[1], self.w2[0], self.w2[1]]
        self.c = h3.make_block_weights_e4m3(self.qkv[0], self.qkv[1], self.w13[0], self.w13[1],
                                            *extra)


def gpu_block_e4m3(dims, L, w, tmod, xb, B, out_down=False):
    dl = DevLayout(dims, L)
    dw, w8 = DevWeights(w), E4m3Weights(w, out_down)
    x = dev_bf16(xb)
    ws_b = h3.h3_workspace_size_e4m3(dl.dims, B, L.S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    h3.h3_block_forward_e4m3(dl.dims, dw.c, w8.c, dl.handle, tmod, x, B, ws, ws_b)
    torch.cuda.synchronize()
    assert h3.h3_layout_error(dl.handle) == h3.H3_OK
    return host_f64(x)


@pytest.mark.parametrize("out_down", [False, True])
def test_e4m3_block_tiny_workload(out_down):
    dims = TINY_DIMS
    L = config_layout(1)
    w = block_weights(dims, 1, 0)
    pw = prologue_weights(dims, 1)
    xb = activations(dims, 1, L.S)
    got = gpu_block_e4m3(dims, L, w, gpu_tmod(dims, L.timestep, pw), xb, 1, out_down)[0]
    x0 = O.bf16_to_f64(xb[0])
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim, dims.hidden)
    ref = O.block_forward_fp8(x0[None], w, L, tm, dims, emulate=True, out_down=out_down)[0]
    pad = L.tags < 0
    assert_close(got, ref, what="e4m3 block x_out")
    assert rel_l2(got[~pad] - x0[~pad], ref[~pad] - x0[~pad]) < 0.1
    np.testing.assert_array_equal(got[pad], x0[pad])


@pytest.mark.parametrize("out_down", [False, True])
@pytest.mark.parametrize("S,seed", [(256, 1), (333, 2), (97, 3)])
def test_e4m3_block_small_amplified(S, seed, out_down):
    dims = Dims(hidden=256, heads=2, head_dim=128, ffn=384, time_embed_dim=64, time_hidden=128)
    L = random_layout(S, seed, pad_runs=2, max_run=60)
    w = amplified_weights(dims, seed)
    tm = (np.random.default_rng([seed, 62]).standard_normal((L.n_t, 6, dims.hidden)) * 0.3
          ).astype(np.float32)
    B = 2
    xb = normal_bf16((B, S, dims.hidden), [seed, 63], 1.0)
    got = gpu_block_e4m3(dims, L, w, dev_f32(tm), xb, B, out_down)
    pad = L.tags < 0
    for b in range(B):
        x0 = O.bf16_to_f64(xb[b])
        ref = O.block_forward_fp8(x0[None], w, L, tm, dims, emulate=True, out_down=out_down)[0]
        sp = Spread(ref, O.block_forward_fp8(x0[None], w, L, tm, dims, out_down=out_down)[0],
                    x0, ~pad)
        assert_close_flips(got[b], ref, sp, what=f"e4m3 x_out b={b}", storage_rounding=True)
        assert_close(got[b, ~pad] - x0[~pad], ref[~pad] - x0[~pad], what="e4m3 update",
                     rel=REL_L2 + sp.upd, mabs=np.inf)
        np.testing.assert_array_equal(got[b, pad], x0[pad])
        # the 8-bit block is near the bf16 block: a few % of the update
        full = O.block_forward(x0[None], w, L, tm, dims)[0]
        assert rel_l2(got[b, ~pad] - x0[~pad], full[~pad] - x0[~pad]) < 0.1


@pytest.mark.parametrize("out_down", [False, True])
def test_e4m3_block_full_width(out_down):
    dims = FULL_DIMS
    segs = [("text", 0, 300), ("video", (2, 16, 16), 0, 2), ("pad", 90), ("audio", 0, 598)]
    L = make_layout(segs, seed=[19])
    assert L.S == 1500
    w = block_weights(dims, 9, 0)
    pw = prologue_weights(dims, 9)
    xb = activations(dims, 9, L.S)
    got = gpu_block_e4m3(dims, L, w, gpu_tmod(dims, L.timestep, pw), xb, 1, out_down)[0]
    x0 = O.bf16_to_f64(xb[0])
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim, dims.hidden)
    ref = O.block_forward_fp8(x0[None], w, L, tm, dims, emulate=True, out_down=out_down)[0]
    pad = L.tags < 0
    sp = Spread(ref, O.block_forward_fp8(x0[None], w, L, tm, dims, out_down=out_down)[0], x0,
                ~pad)
    assert_close_flips(got, ref, sp, what="full-width e4m3 x_out")
    assert_close(got[~pad] - x0[~pad], ref[~pad] - x0[~pad], what="full-width e4m3 update",
                 rel=REL_L2 + sp.upd, mabs=np.inf)
    np.testing.assert_array_equal(got[pad], x0[pad])


def _stack_refs(x0, ws_host, L, tm, dims, out_down):
    """The oracle's 8-bit blocks in sequence over an fp32 stream, rounded to bf16
    once at the end (as the stack scatters its rows back): the bf16-storage
    reading and the float64 one."""
    refs = []
    for emulate in (True, False):
        y = x0[None]
        for w in ws_host:
            y = O.block_forward_fp8(y, w, L, tm, dims, emulate=emulate, out_down=out_down,
                                    stream_f32=True)
        refs.append(O.round_bf16(y[0]) if emulate else y[0])
    return refs


def gpu_stack_e4m3(dims, L, ws_host, tmod, xb, out_down):
    dl = DevLayout(dims, L)
    dws = [DevWeights(w) for w in ws_host]
    w8s = [E4m3Weights(w, out_down) for w in ws_host]
    x = dev_bf16(xb)
    ws_b = h3.h3_workspace_size_e4m3(dl.dims, xb.shape[0], L.S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    h3.h3_stack_forward_e4m3(dl.dims, [w.c for w in dws], [w.c for w in w8s], dl.handle, tmod, x,
                             xb.shape[0], ws, ws_b)
    torch.cuda.synchronize()
    assert h3.h3_layout_error(dl.handle) == h3.H3_OK
    return host_f64(x)


@pytest.mark.parametrize("out_down", [False, True])
def test_e4m3_stack_small_amplified(out_down):
    """Three 8-bit blocks through h3_stack_forward_e4m3 (fp32 residual stream)
    against the oracle's 8-bit blocks in sequence, with the 8-bit block's budget."""
    dims = SMALL
    L = random_layout(256, 4, pad_runs=2, max_run=60)
    ws_host = [amplified_weights(dims, 40 + i) for i in range(3)]
    tm = (np.random.default_rng([4, 62]).standard_normal((L.n_t, 6, dims.hidden)) * 0.3
          ).astype(np.float32)
    xb = normal_bf16((1, L.S, dims.hidden), [4, 63], 1.0)
    got = gpu_stack_e4m3(dims, L, ws_host, dev_f32(tm), xb, out_down)[0]
    x0 = O.bf16_to_f64(xb[0])
    ref, ref64 = _stack_refs(x0, ws_host, L, tm, dims, out_down)
    pad = L.tags < 0
    sp = Spread(ref, ref64, x0, ~pad)
    assert_close_flips(got, ref, sp, what="e4m3 3-block stack x_out", storage_rounding=True)
    assert_close(got[~pad] - x0[~pad], ref[~pad] - x0[~pad], what="e4m3 stack update",
                 rel=REL_L2 + sp.upd, mabs=np.inf)
    np.testing.assert_array_equal(got[pad], x0[pad])


def test_e4m3_stack_full_width_two_blocks():
    dims = FULL_DIMS
    segs = [("text", 0, 300), ("video", (2, 16, 16), 0, 2), ("pad", 90), ("audio", 0, 598)]
    L = make_layout(segs, seed=[19])
    ws_host = [block_weights(dims, 9, i) for i in range(2)]
    pw = prologue_weights(dims, 9)
    xb = activations(dims, 9, L.S)
    got = gpu_stack_e4m3(dims, L, ws_host, gpu_tmod(dims, L.timestep, pw), xb, True)[0]
    x0 = O.bf16_to_f64(xb[0])
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim, dims.hidden)
    ref, ref64 = _stack_refs(x0, ws_host, L, tm, dims, True)
    pad = L.tags < 0
    sp = Spread(ref, ref64, x0, ~pad)
    assert_close_flips(got, ref, sp, what="full-width e4m3 2-block stack x_out",
                       storage_rounding=True)
    assert_close(got[~pad] - x0[~pad], ref[~pad] - x0[~pad], what="full-width e4m3 stack update",
                 rel=REL_L2 + sp.upd, mabs=np.inf)
    np.testing.assert_array_equal(got[pad], x0[pad])
