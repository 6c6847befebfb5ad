"""The 8-bit (e4m3) QKV and W1 || W3 GEMM inputs on the GPU against the oracle.

Source: "MiniMax H3 Inference Engine voor Mac computers", sections "Profiling
en diagnostische pads" and "Sampler en DiT controls" (8-bit MLP and QKV
projections, one activation scale per row). The oracle quantizes at the same
points (oracle.h3_oracle.block_forward_fp8), so the GPU block is held to the
same tolerance as the bf16 block against it; the weight codes and scales, whose
inputs are exact on both sides, are compared bit for bit.

An e4m3 code is an integer decided by floating point, and one code step is 6-12 %
of a value: the reference must decide the codes of h2 from the norm2 input the
device holds, x1 stored in bf16. The oracle's 8-bit block is therefore compared
in its bf16-storage emulation (bf16 where the device stores bf16; h and h2 go
from fp32 straight to codes on both sides). Against the float64 reference
without that emulation the norm2 input differs by bf16 rounding, which moves a
few % of the h2 codes by one step: ~1-2 % differences in x_out.
"""

import numpy as np
import pytest
import torch

from audio_generation_b200 import h3
from oracle import h3_oracle as O
from tests.h3_testlib import (DevLayout, DevWeights, assert_close, dev_bf16, dev_f32, host_f64,
                              rel_l2)
from tests.test_gpu_block import amplified_weights, gpu_tmod
from workloads import (FULL_DIMS, TINY_DIMS, Dims, activations, block_weights, config_layout,
                       f32_to_bf16_bits, make_layout, normal_bf16, prologue_weights,
                       random_layout)

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


class E4m3Weights:
    def __init__(self, w):
        self.qkv = gpu_codes(w.w_qkv)
        self.w13 = gpu_codes(w.w13)
        self.c = h3.make_block_weights_e4m3(self.qkv[0], self.qkv[1], self.w13[0], self.w13[1])


def gpu_block_e4m3(dims, L, w, tmod, xb, B):
    dl = DevLayout(dims, L)
    dw, w8 = DevWeights(w), E4m3Weights(w)
    x = dev_bf16(xb)
    ws_b = h3.h3_workspace_size_e4m3(dl.dims, B, L.S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    h3.h3_block_forward_e4m3(dl.dims, dw.c, w8.c, dl.handle, tmod, x, B, ws, ws_b)
    torch.cuda.synchronize()
    assert h3.h3_layout_error(dl.handle) == h3.H3_OK
    return host_f64(x)


def test_e4m3_block_tiny_workload():
    dims = TINY_DIMS
    L = config_layout(1)
    w = block_weights(dims, 1, 0)
    pw = prologue_weights(dims, 1)
    xb = activations(dims, 1, L.S)
    got = gpu_block_e4m3(dims, L, w, gpu_tmod(dims, L.timestep, pw), xb, 1)[0]
    x0 = O.bf16_to_f64(xb[0])
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim, dims.hidden)
    ref = O.block_forward_fp8(x0[None], w, L, tm, dims, emulate=True)[0]
    pad = L.tags < 0
    assert_close(got, ref, what="e4m3 block x_out")
    assert rel_l2(got[~pad] - x0[~pad], ref[~pad] - x0[~pad]) < 0.1
    np.testing.assert_array_equal(got[pad], x0[pad])


@pytest.mark.parametrize("S,seed", [(256, 1), (333, 2), (97, 3)])
def test_e4m3_block_small_amplified(S, seed):
    dims = Dims(hidden=256, heads=2, head_dim=128, ffn=384, time_embed_dim=64, time_hidden=128)
    L = random_layout(S, seed, pad_runs=2, max_run=60)
    w = amplified_weights(dims, seed)
    tm = (np.random.default_rng([seed, 62]).standard_normal((L.n_t, 6, dims.hidden)) * 0.3
          ).astype(np.float32)
    B = 2
    xb = normal_bf16((B, S, dims.hidden), [seed, 63], 1.0)
    got = gpu_block_e4m3(dims, L, w, dev_f32(tm), xb, B)
    pad = L.tags < 0
    for b in range(B):
        x0 = O.bf16_to_f64(xb[b])
        ref = O.block_forward_fp8(x0[None], w, L, tm, dims, emulate=True)[0]
        assert_close(got[b], ref, what=f"e4m3 x_out b={b}", storage_rounding=True)
        assert_close(got[b, ~pad] - x0[~pad], ref[~pad] - x0[~pad], what="e4m3 update",
                     mabs=np.inf)
        np.testing.assert_array_equal(got[b, pad], x0[pad])
        # the 8-bit block is near the bf16 block: a few % of the update
        full = O.block_forward(x0[None], w, L, tm, dims)[0]
        assert rel_l2(got[b, ~pad] - x0[~pad], full[~pad] - x0[~pad]) < 0.1


def test_e4m3_block_full_width():
    dims = FULL_DIMS
    segs = [("text", 0, 300), ("video", (2, 16, 16), 0, 2), ("pad", 90), ("audio", 0, 598)]
    L = make_layout(segs, seed=[19])
    assert L.S == 1500
    w = block_weights(dims, 9, 0)
    pw = prologue_weights(dims, 9)
    xb = activations(dims, 9, L.S)
    got = gpu_block_e4m3(dims, L, w, gpu_tmod(dims, L.timestep, pw), xb, 1)[0]
    x0 = O.bf16_to_f64(xb[0])
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim, dims.hidden)
    ref = O.block_forward_fp8(x0[None], w, L, tm, dims, emulate=True)[0]
    pad = L.tags < 0
    assert_close(got, ref, what="full-width e4m3 x_out")
    assert_close(got[~pad] - x0[~pad], ref[~pad] - x0[~pad], what="full-width e4m3 update",
                 mabs=np.inf)
    np.testing.assert_array_equal(got[pad], x0[pad])
