"""CPU oracle for the MiniMax-H3 transformer block forward — TEST INFRASTRUCTURE.

Only the tests, the package's ``smoke()`` check and the benchmark's CPU
baseline may import this module. It is a plain, slow, float64 NumPy
restatement of what the block computes, written to be checked against the
pages by eye. It shares nothing with the CUDA path.

Sources (titles and sections of the pages this follows):

* [MX] "MiniMaxH3Transformer3DModel" (diffusers v0.43.0 docs): the overview
  (one packed 1-D sequence, full self-attention, per-row modality tag selects
  the AdaLN modulation; padding rows, tag -1, form their own attention
  document under a boolean mask), the constructor parameters (56 heads of
  128, hidden 5376, ffn 14336, freq_dim 256, time_embed_dim 2688 = input of
  every AdaLN projection, rope_freq_dim 16 shared by the (t, h, w) axes with
  2*3*16 channels rotated, rope_theta 1e4, norm_eps, qk_norm_eps) and the
  ``forward`` arguments (timestep values, per-row timestep indices, tags,
  positions, the three index tensors).
* [ME] "MiniMax H3 Inference Engine voor Mac computers", sections
  "Exacte DiT fusions" (gated attention residual followed by the MLP's AdaLN,
  bf16 residual stream), "Checkpoint layout en media pipeline" (QKV rows
  interleaved per attention head; fused QK-norm + RoPE), "Profiling en
  diagnostische pads" (fc1 -> SwiGLU -> fc2).

Readings where the pages leave a step open (each also listed in the design
notes): LayerNorm without affine for the pre-norms; modulate as
norm * (1 + scale) + shift with chunk order (shift1, scale1, gate1, shift2,
scale2, gate2); per-row modulation = ada_table[tag] + tmod[t_idx] where
tmod = W_proj . SiLU(TimeMLP(sinusoid(t))) is shared by all blocks; QK-norm is
RMSNorm over a head's 128 channels with learned [128] weights; RoPE rotates
channel pairs (32a + j, 32a + j + 16), a = t, h, w, with
inv_freq[j] = theta^(-j/16); attention scale 1/sqrt(128); no biases; padding
rows (tag -1) attend only padding rows and leave the block unchanged.

Parity pins for every function here are in tests/test_oracle_pins.py.
"""

from __future__ import annotations

import math
from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

F = np.float64
TAG_PAD = -1
TILE = 128  # row-tile height used by the tile-class table of the layout step


# --------------------------------------------------------------------------
# Storage helpers
# --------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(F)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), through float32.

    Used only by the optional bf16-storage emulation, which mimics a device
    that holds fp32 values and stores them as bf16.
    """
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.astype(np.uint32).view(np.float32).astype(F)


def _store(a: np.ndarray, emulate: bool) -> np.ndarray:
    return round_bf16(a) if emulate else a


# --------------------------------------------------------------------------
# a2: timestep embedding and the shared AdaLN projection  [MX: freq_dim,
#     time_embed_hidden_dim, time_embed_dim; timesteps unscaled in [0, 1]]
# --------------------------------------------------------------------------

def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def timestep_sinusoid(t: np.ndarray, freq_dim: int) -> np.ndarray:
    """[n_t] -> [n_t, freq_dim]: [cos(t f_i), sin(t f_i)], f_i = 10^4^(-i/(freq_dim/2))."""
    half = freq_dim // 2
    i = np.arange(half, dtype=F)
    f = np.exp(-math.log(10000.0) * i / half)
    arg = np.asarray(t, dtype=F)[:, None] * f[None, :]
    return np.concatenate([np.cos(arg), np.sin(arg)], axis=1)


def timestep_modulation(t: np.ndarray, w_t1: np.ndarray, w_t2: np.ndarray,
                        w_proj: np.ndarray, freq_dim: int, hidden: int) -> np.ndarray:
    """tmod[n_t, 6, H] = W_proj . SiLU(W_t2 . SiLU(W_t1 . sinusoid(t))).

    Given only the first c*H rows of W_proj, returns the first c chunks [n_t, c, H].
    """
    s = timestep_sinusoid(t, freq_dim)
    temb = silu(s @ np.asarray(w_t1, F).T) @ np.asarray(w_t2, F).T
    tmod = silu(temb) @ np.asarray(w_proj, F).T
    return tmod.reshape(tmod.shape[0], -1, hidden)


# --------------------------------------------------------------------------
# a3 / a7: norm + AdaLN modulate  [MX: norm_eps; per-row tag selects AdaLN]
# --------------------------------------------------------------------------

def row_modulation(tags: np.ndarray, t_idx: np.ndarray, ada_table: np.ndarray,
                   tmod: np.ndarray) -> np.ndarray:
    """[n] rows -> [n, 6, H]: ada_table[tag] + tmod[t_idx]; zero for padding rows."""
    tags = np.asarray(tags)
    table = np.asarray(ada_table, F)
    m = np.zeros((tags.shape[0],) + table.shape[1:], F)
    v = tags >= 0
    m[v] = table[tags[v]] + np.asarray(tmod, F)[np.asarray(t_idx)[v]]
    return m


def layer_norm(x: np.ndarray, eps: float) -> np.ndarray:
    """(x - mean) / sqrt(var + eps) over the last axis, biased variance, no affine."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def norm_modulate(x: np.ndarray, shift: np.ndarray, scale: np.ndarray,
                  eps: float) -> np.ndarray:
    return layer_norm(x, eps) * (1.0 + scale) + shift


# --------------------------------------------------------------------------
# a4: QKV projection, per-head QK-norm, 3-axis RoPE
#     [MX: num_attention_heads * attention_head_dim > hidden_size;
#      qk_norm_eps; rope_freq_dim, rope_theta]  [ME: QKV rows per head]
# --------------------------------------------------------------------------

def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w over the last axis."""
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * w


def rope_inv_freq(rope_freq_dim: int, theta: float) -> np.ndarray:
    j = np.arange(rope_freq_dim, dtype=F)
    return theta ** (-j / rope_freq_dim)


def rope_apply(x: np.ndarray, pos: np.ndarray, inv_freq: np.ndarray) -> np.ndarray:
    """Rotate x[..., n, D] (n rows, any leading head axis after rows) by positions.

    x has shape [n, NH, D]; pos [n, 3]. For axis a in (t, h, w) and j < nf,
    the pair (c0, c1) = (2 nf a + j, 2 nf a + j + nf) is rotated by
    angle pos[r, a] * inv_freq[j]. Channels >= 6 nf are left unchanged.
    """
    nf = inv_freq.shape[0]
    out = np.array(x, dtype=F, copy=True)
    for a in range(3):
        ang = np.asarray(pos, F)[:, a:a + 1] * inv_freq[None, :]  # [n, nf]
        c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
        lo = 2 * nf * a
        x0 = x[:, :, lo:lo + nf]
        x1 = x[:, :, lo + nf:lo + 2 * nf]
        out[:, :, lo:lo + nf] = x0 * c - x1 * s
        out[:, :, lo + nf:lo + 2 * nf] = x0 * s + x1 * c
    return out


def split_qkv_weight(w_qkv: np.ndarray, heads: int, head_dim: int) -> Tuple[np.ndarray, ...]:
    """Head-interleaved [3 NH D, H] -> Wq, Wk, Wv each [NH D, H]."""
    w = np.asarray(w_qkv).reshape(heads, 3, head_dim, -1)
    return (w[:, 0].reshape(heads * head_dim, -1), w[:, 1].reshape(heads * head_dim, -1),
            w[:, 2].reshape(heads * head_dim, -1))


def split_w13(w13: np.ndarray, ffn: int) -> Tuple[np.ndarray, np.ndarray]:
    """Block-interleaved [2F, H] (128-row blocks W1_j, W3_j) -> W1, W3 each [F, H]."""
    w = np.asarray(w13).reshape(ffn // 128, 2, 128, -1)
    return w[:, 0].reshape(ffn, -1), w[:, 1].reshape(ffn, -1)


def qkv_project(h: np.ndarray, pos: np.ndarray, w_qkv: np.ndarray, q_norm: np.ndarray,
                k_norm: np.ndarray, dims, emulate: bool = False,
                need_q: bool = True) -> Tuple[Optional[np.ndarray], np.ndarray, np.ndarray]:
    """h [n, H] -> q, k, v [n, NH, D] after QK-norm and RoPE (q, k only); w_qkv
    as bf16 bits."""
    return qkv_project_values(h, pos, bf16_to_f64(w_qkv), q_norm, k_norm, dims, emulate, need_q)


def qkv_project_values(h: np.ndarray, pos: np.ndarray, w_qkv: np.ndarray, q_norm: np.ndarray,
                       k_norm: np.ndarray, dims, emulate: bool = False,
                       need_q: bool = True) -> Tuple[Optional[np.ndarray], np.ndarray, np.ndarray]:
    """qkv_project with the weight [3 NH D, H] given as values."""
    NH, D = dims.heads, dims.head_dim
    wq, wk, wv = split_qkv_weight(np.asarray(w_qkv, F), NH, D)
    inv = rope_inv_freq(dims.rope_freq_dim, dims.rope_theta)
    qn, kn = bf16_to_f64(q_norm), bf16_to_f64(k_norm)
    n = h.shape[0]
    k = (h @ wk.T).reshape(n, NH, D)
    v = (h @ wv.T).reshape(n, NH, D)
    k = rope_apply(rms_norm(k, kn, dims.qk_norm_eps), pos, inv)
    q = None
    if need_q:
        q = (h @ wq.T).reshape(n, NH, D)
        q = _store(rope_apply(rms_norm(q, qn, dims.qk_norm_eps), pos, inv), emulate)
    return q, _store(k, emulate), _store(v, emulate)


# --------------------------------------------------------------------------
# a5: bidirectional attention with the padding document
#     [MX: padding rows stay in their own attention document]
# --------------------------------------------------------------------------

def attention(q: np.ndarray, doc_q: np.ndarray, k: np.ndarray, v: np.ndarray,
              doc_k: np.ndarray, emulate: bool = False) -> np.ndarray:
    """q [n, NH, D], k/v [S, NH, D]; keys visible where doc_k == doc_q.

    Returns o [n, NH * D] = concat over heads of softmax(q k^T / sqrt(D)) v.
    """
    n, NH, D = q.shape
    scale = 1.0 / math.sqrt(D)
    o = np.empty((n, NH, D), F)
    same = np.asarray(doc_q)[:, None] == np.asarray(doc_k)[None, :]
    for hd in range(NH):
        s = (q[:, hd, :] @ k[:, hd, :].T) * scale
        s = np.where(same, s, -np.inf)
        mx = s.max(axis=1, keepdims=True)
        p = np.exp(s - mx)
        l = p.sum(axis=1, keepdims=True)
        p = _store(p, emulate)
        o[:, hd, :] = (p @ v[:, hd, :]) / l
    return _store(o.reshape(n, NH * D), emulate)


# --------------------------------------------------------------------------
# a6 .. a9: output projection, FFN, gated residuals  [ME: "Exacte DiT fusions"]
# --------------------------------------------------------------------------

def out_project_residual(x: np.ndarray, o: np.ndarray, gate: np.ndarray, w_o: np.ndarray,
                         emulate: bool = False) -> np.ndarray:
    """x1 = x + gate * (o W_o^T); w_o as bf16 bits."""
    return out_project_residual_values(x, o, gate, bf16_to_f64(w_o), emulate)


def out_project_residual_values(x: np.ndarray, o: np.ndarray, gate: np.ndarray, w_o: np.ndarray,
                                emulate: bool = False) -> np.ndarray:
    """out_project_residual with W_o [H, NH D] given as values."""
    return _store(x + gate * (o @ np.asarray(w_o, F).T), emulate)


def ffn_gate(h2: np.ndarray, w13: np.ndarray, ffn: int, emulate: bool = False) -> np.ndarray:
    """g = SiLU(h2 W1^T) * (h2 W3^T); w13 as bf16 bits."""
    return ffn_gate_values(h2, bf16_to_f64(w13), ffn, emulate)


def ffn_gate_values(h2: np.ndarray, w13: np.ndarray, ffn: int, emulate: bool = False) -> np.ndarray:
    """ffn_gate with W1 || W3 [2F, H] given as values."""
    w1, w3 = split_w13(np.asarray(w13, F), ffn)
    return _store(silu(h2 @ w1.T) * (h2 @ w3.T), emulate)


def ffn_down_residual(x1: np.ndarray, g: np.ndarray, gate: np.ndarray, w2: np.ndarray,
                      emulate: bool = False) -> np.ndarray:
    """x2 = x1 + gate * (g W2^T); w2 as bf16 bits."""
    return ffn_down_residual_values(x1, g, gate, bf16_to_f64(w2), emulate)


def ffn_down_residual_values(x1: np.ndarray, g: np.ndarray, gate: np.ndarray, w2: np.ndarray,
                             emulate: bool = False) -> np.ndarray:
    """ffn_down_residual with W2 [H, F] given as values."""
    return _store(x1 + gate * (g @ np.asarray(w2, F).T), emulate)


# --------------------------------------------------------------------------
# The block and the stack
# --------------------------------------------------------------------------

def _pre_attention(x, m, pos, w, dims, emulate, need_q=True):
    h = _store(norm_modulate(x, m[:, 0], m[:, 1], dims.norm_eps), emulate)
    return qkv_project(h, pos, w.w_qkv, w.q_norm, w.k_norm, dims, emulate, need_q)


def _stream(a: np.ndarray, emulate: bool, stream_f32: bool) -> np.ndarray:
    """Storage of the residual stream x1 / x2 under the emulation: bf16, or fp32
    where the stream is held in fp32 (the stack's residual stream)."""
    if emulate and stream_f32:
        return np.asarray(a, np.float32).astype(F)
    return _store(a, emulate)


def _post_attention(x, o, m, w, dims, emulate, stream_f32=False):
    x1 = _stream(out_project_residual(x, o, m[:, 2], w.w_o), emulate, stream_f32)
    h2 = _store(norm_modulate(x1, m[:, 3], m[:, 4], dims.norm_eps), emulate)
    g = ffn_gate(h2, w.w13, dims.ffn, emulate)
    return _stream(ffn_down_residual(x1, g, m[:, 5], w.w2), emulate, stream_f32)


def block_forward(x: np.ndarray, w, layout, tmod: np.ndarray, dims,
                  emulate: bool = False, stream_f32: bool = False) -> np.ndarray:
    """One block over the packed sequence. x [B, S, H] (values) -> [B, S, H] float64.

    Padding rows (tag -1) are returned unchanged. ``emulate`` rounds to bf16 at
    the device's storage points; with ``stream_f32`` the residual stream (x1 and
    the output) is held in fp32 instead, as a stack of blocks holds it.
    """
    x = np.asarray(x, F)
    tags = np.asarray(layout.tags)
    if tags.shape[0] == 0:
        return x.copy()
    pad = tags < 0
    m = row_modulation(tags, layout.t_idx, w.ada_table, tmod)
    out = np.empty_like(x)
    for b in range(x.shape[0]):
        q, k, v = _pre_attention(x[b], m, layout.pos, w, dims, emulate)
        o = attention(q, pad, k, v, pad, emulate)
        y = _post_attention(x[b], o, m, w, dims, emulate, stream_f32)
        out[b] = np.where(pad[:, None], x[b], y)
    return out


def key_value_rows(x: np.ndarray, w, layout, tmod_rows: Callable, dims,
                   chunk: int = 2048) -> Tuple[np.ndarray, np.ndarray]:
    """k, v [S, NH, D] of every row of one sequence (B = 1), in row chunks (each
    row's k and v depend on that row alone). ``tmod_rows(t_idx, n_chunks)``
    returns the first ``n_chunks`` modulation chunks of tmod for those timestep
    indices, [n, n_chunks, H]; this pass asks only for (shift1, scale1), so a
    caller with one timestep per row never forms the whole tmod."""
    x = np.asarray(x, F)
    S = x.shape[0]
    tags = np.asarray(layout.tags)
    NH, D = dims.heads, dims.head_dim
    K = np.empty((S, NH, D), F)
    V = np.empty((S, NH, D), F)
    table = np.asarray(w.ada_table, F)
    t_idx = np.asarray(layout.t_idx)
    for r0 in range(0, S, chunk):
        r1 = min(S, r0 + chunk)
        tg = tags[r0:r1]
        m = np.zeros((r1 - r0, 2, dims.hidden), F)
        vv = tg >= 0
        if vv.any():
            m[vv] = table[tg[vv], :2] + tmod_rows(t_idx[r0:r1][vv], 2)
        _, K[r0:r1], V[r0:r1] = _pre_attention(x[r0:r1], m, layout.pos[r0:r1], w, dims,
                                               False, need_q=False)
    return K, V


def query_rows(x: np.ndarray, w, layout, tmod_rows: Callable, dims, rows: np.ndarray,
               K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """The block's output at the query rows ``rows`` (B = 1), given k and v of
    every row (from ``key_value_rows``). The rows' own q, k and v are formed
    here from their inputs, as in the block."""
    x = np.asarray(x, F)
    tags = np.asarray(layout.tags)
    pad = tags < 0
    table = np.asarray(w.ada_table, F)
    t_idx = np.asarray(layout.t_idx)
    rows = np.asarray(rows)
    tg = tags[rows]
    m = np.zeros((rows.shape[0], 6, dims.hidden), F)
    vv = tg >= 0
    if vv.any():
        m[vv] = table[tg[vv]] + tmod_rows(t_idx[rows][vv], 6)
    q, _, _ = _pre_attention(x[rows], m, layout.pos[rows], w, dims, False)
    o = attention(q, pad[rows], K, V, pad)
    y = _post_attention(x[rows], o, m, w, dims, False)
    return np.where(pad[rows][:, None], x[rows], y)


def block_forward_rows(x: np.ndarray, w, layout, tmod_rows: Callable, dims, rows: np.ndarray,
                       chunk: int = 2048) -> np.ndarray:
    """The same block evaluated only at the query rows ``rows`` (B = 1).

    Keys and values are needed for every row, so they are formed for all rows
    first (``key_value_rows``), then the block runs at the query rows
    (``query_rows``).
    """
    K, V = key_value_rows(x, w, layout, tmod_rows, dims, chunk)
    return query_rows(x, w, layout, tmod_rows, dims, rows, K, V)


def stack_forward(x: np.ndarray, weights_for_block: Callable[[int], object], n_blocks: int,
                  layout, tmod: np.ndarray, dims, emulate: bool = False) -> np.ndarray:
    """``n_blocks`` blocks in sequence, sharing one tmod (computed once per forward)."""
    y = np.asarray(x, F)
    for i in range(n_blocks):
        y = block_forward(y, weights_for_block(i), layout, tmod, dims, emulate)
    return y


# --------------------------------------------------------------------------
# The denoiser around the stack: input projections, text refiner, norm_out and
# the two output heads  [MX: constructor parameters in_channels,
# audio_in_channels, patch_size, text_dim, num_refiner_layers, final_norm_eps;
# the mixed-precision note (patch projections, timestep MLP and output heads
# in float32); `forward` returns the video and audio velocities in the row
# order of video_indices and audio_indices]  [ME: "Exacte DiT fusions": final
# audio / video AdaLN; "Sampler en DiT controls": timestep-aware output head]
#
# Readings where the pages leave the structure open: no biases; the text
# projection belongs to the bf16 stack (it is not among the float32 modules);
# each refiner block is a block of the stack's structure with its own weights,
# run over the text rows alone as their own sequence and modulated like the
# stack (table row of the text tag + the row's timestep); the refiner output is
# a LayerNorm without affine (eps = final_norm_eps); norm_out is the same
# LayerNorm followed by a per-modality AdaLN (shift, scale) whose rows are
# out_table[modality] + W_out . SiLU(temb); the heads are float32 linears.
# --------------------------------------------------------------------------

def timestep_embedding(t: np.ndarray, w_t1: np.ndarray, w_t2: np.ndarray,
                       freq_dim: int) -> np.ndarray:
    """temb[n_t, E] = W_t2 . SiLU(W_t1 . sinusoid(t)): the timestep MLP."""
    s = timestep_sinusoid(t, freq_dim)
    return silu(s @ np.asarray(w_t1, F).T) @ np.asarray(w_t2, F).T


def output_modulation(t: np.ndarray, w_t1: np.ndarray, w_t2: np.ndarray, w_out: np.ndarray,
                      freq_dim: int, hidden: int) -> np.ndarray:
    """tmod_out[n_t, 2, H] = W_out . SiLU(temb): the (shift, scale) of norm_out."""
    temb = timestep_embedding(t, w_t1, w_t2, freq_dim)
    return (silu(temb) @ np.asarray(w_out, F).T).reshape(len(t), 2, hidden)


def patch_project(latents: np.ndarray, w: np.ndarray) -> np.ndarray:
    """[n, C] latent rows -> [n, H] = rows . W^T (float32 module, no bias)."""
    return np.asarray(latents, F) @ np.asarray(w, F).T


def text_project(enc_bits: np.ndarray, w_text_bits: np.ndarray) -> np.ndarray:
    """[n, text_dim] bf16 text condition -> [n, H] with the bf16 [H, text_dim] weight."""
    return bf16_to_f64(enc_bits) @ bf16_to_f64(w_text_bits).T


def text_only_layout(layout):
    """The text rows of a packed layout as a sequence of their own (index
    order of text_idx): their positions and timestep indices, tag 1."""
    from types import SimpleNamespace
    ti = np.asarray(layout.text_idx)
    n = ti.shape[0]
    return SimpleNamespace(tags=np.full(n, 1, np.int32), pos=np.asarray(layout.pos)[ti],
                           t_idx=np.asarray(layout.t_idx)[ti], timestep=layout.timestep,
                           text_idx=np.arange(n), video_idx=np.zeros(0, np.int32),
                           audio_idx=np.zeros(0, np.int32), S=n)


def refine_text(xt: np.ndarray, refiner: Sequence, layout, tmod: np.ndarray, dims,
                final_eps: float) -> np.ndarray:
    """The refiner blocks over the projected text rows ([n_text, H], text_idx
    order) as their own sequence, then LayerNorm (no affine, final_norm_eps)."""
    lt = text_only_layout(layout)
    y = np.asarray(xt, F)[None]
    for w in refiner:
        y = block_forward(y, w, lt, tmod, dims)
    return layer_norm(y[0], final_eps)


def output_head(x_rows: np.ndarray, shift: np.ndarray, scale: np.ndarray, w_head: np.ndarray,
                final_eps: float) -> np.ndarray:
    """norm_out then the float32 head: (LN(x) (1 + scale) + shift) . W_head^T."""
    return norm_modulate(np.asarray(x_rows, F), shift, scale, final_eps) @ np.asarray(w_head, F).T


def denoiser_forward(video: np.ndarray, audio: np.ndarray, text: np.ndarray, dw,
                     blocks: Callable[[int], object], n_blocks: int, layout, dims,
                     final_eps: float, core_residual: Optional[np.ndarray] = None,
                     reuse: bool = False) -> Tuple[np.ndarray, np.ndarray]:
    """One transformer forward for one batch element: video [n_video, C_v] and
    audio [n_audio, C_a] latent rows, text [n_text, text_dim] bf16 bits, each in
    the order of its index tensor -> (video velocity [n_video, C_v], audio
    velocity [n_audio, C_a]) in the same orders.

    ``dw`` holds w_patch_video, w_patch_audio, w_text, refiner (block weights),
    w_t1, w_t2, w_proj, w_out, out_table ([2, 2, H]: video, audio x shift,
    scale), w_head_video, w_head_audio.

    Core residual reuse ([ME] "Sampler en DiT controls": the previous full
    transformer residual is held while the patch projections and the
    timestep-aware head are refreshed; reading: the core is the refiner and the
    block stack, its residual the stack's output minus the stack's input, [S, H];
    the text rows carry no output, so only video and audio rows use it): with
    ``core_residual`` given and ``reuse`` False the forward also stores that
    residual in it; with ``reuse`` True the core does not run and the stream is
    the fresh projections plus the stored residual.
    """
    H = dims.hidden
    t = layout.timestep
    tmod = timestep_modulation(t, dw.w_t1, dw.w_t2, dw.w_proj, dims.freq_dim, H)
    tmo = output_modulation(t, dw.w_t1, dw.w_t2, dw.w_out, dims.freq_dim, H)
    x = np.zeros((layout.S, H), F)
    vi, ai, ti = (np.asarray(a) for a in (layout.video_idx, layout.audio_idx, layout.text_idx))
    x[vi] = patch_project(video, dw.w_patch_video)
    x[ai] = patch_project(audio, dw.w_patch_audio)
    if reuse:
        x = x + core_residual
    else:
        if ti.shape[0]:
            x[ti] = refine_text(text_project(text, dw.w_text), dw.refiner, layout, tmod, dims,
                                final_eps)
        x_in = x.copy()
        x = stack_forward(x[None], blocks, n_blocks, layout, tmod, dims)[0]
        if core_residual is not None:
            core_residual[...] = x - x_in
    t_idx = np.asarray(layout.t_idx)
    out = []
    for idx, m, w_head in ((vi, 0, dw.w_head_video), (ai, 1, dw.w_head_audio)):
        mod = np.asarray(dw.out_table, F)[m][None] + tmo[t_idx[idx]]  # [n, 2, H]
        out.append(output_head(x[idx], mod[:, 0], mod[:, 1], w_head, final_eps))
    return out[0], out[1]


# --------------------------------------------------------------------------
# 8-bit GEMM inputs for the QKV and W1 || W3 projections  [ME: "Profiling en
# diagnostische pads" and "Sampler en DiT controls": an 8-bit MLP and 8-bit QKV
# projections, with one activation scale per row]
#
# Reading (B200 form): the e4m3 format (1 sign, 4 exponent bits of bias 7, 3
# mantissa bits, largest finite value 448, no infinities) for both operands;
# one scale per activation row (that row's largest |h| / 448) and one per
# weight row (output channel); the product of the two scales is applied to the
# fp32 dot product of the codes. The scale and the division are float32, as on
# the device, so that both sides round the same values to the same codes.
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value (ties to even), saturating at +-448: normal numbers
    2^(e-7) (1 + m/8), e = 1..15 (e = 15 only up to m = 6), subnormals
    2^-6 m/8; the grid spacing of a value in [2^k, 2^(k+1)) is 2^(k-3), below
    2^-6 it is 2^-9."""
    a = np.abs(np.asarray(x, F))
    k = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    step = 2.0 ** (np.maximum(k, -6.0) - 3.0)
    q = a / step
    r = np.floor(q)
    frac = q - r
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(r, 2) == 1))
    v = (r + up) * step
    v = np.minimum(v, E4M3_MAX)
    return np.where(np.asarray(x, F) < 0, -v, v)


def row_scales_f32(a: np.ndarray) -> np.ndarray:
    """Per-row scale max|a| / 448 in float32 (1 for an all-zero row)."""
    m = np.max(np.abs(np.asarray(a, np.float32)), axis=-1)
    s = (m / np.float32(E4M3_MAX)).astype(np.float32)
    return np.where(s > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows_e4m3(a: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """(codes as their e4m3 values, float32 row scales): a ~= codes * scale."""
    a32 = np.asarray(a, np.float32)
    s = row_scales_f32(a32)
    return e4m3_round((a32 / s[:, None]).astype(np.float32)), s


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Values of e4m3 code bytes: bit 7 the sign, bits 6-3 the exponent field e
    (bias 7), bits 2-0 the mantissa m; e = 0 gives 2^-6 m/8, otherwise
    2^(e-7) (1 + m/8); e = 15 with m = 7 is NaN (no infinities)."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(F)
    mag = np.where(e == 0, 2.0 ** -6 * m / 8.0, 2.0 ** (e.astype(F) - 7.0) * (1.0 + m / 8.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    return np.asarray(codes, F) * np.asarray(scales, F)[:, None]


def block_forward_fp8(x: np.ndarray, w, layout, tmod: np.ndarray, dims,
                      emulate: bool = False, out_down: bool = False,
                      stream_f32: bool = False) -> np.ndarray:
    """The block with its QKV and W1 || W3 GEMMs on e4m3 inputs: the norm outputs
    h and h2 quantized per row (their values held in float32, as the device
    holds them) and the bf16 weights per output channel; everything else as in
    block_forward. (B = 1 or more; padding rows unchanged.) With ``out_down``
    the O and W2 GEMMs take e4m3 inputs too: o and g quantized per row from
    their values as stored, W_o and W2 per output channel.

    ``emulate`` rounds to bf16 where the device stores bf16 in this block (q, k, v
    after RoPE, P, o, x1, g, x2; h and h2 go from fp32 straight to codes). A
    code is an integer that floating point decides: compared with the device,
    the reference must take that decision from the values the device holds, so
    the norm2 input x1 has to be the bf16 value the device stored. With
    ``stream_f32`` (and ``emulate``) x1 and the output are held in fp32 instead,
    as a stack's residual stream holds them."""
    import copy
    wq = copy.copy(w)
    for name in ("w_qkv", "w13") + (("w_o", "w2") if out_down else ()):
        wf = bf16_to_f64(getattr(w, name)).astype(np.float32)
        codes, sc = quantize_rows_e4m3(wf)
        setattr(wq, name, dequantize_rows(codes, sc))
    x = np.asarray(x, F)
    tags = np.asarray(layout.tags)
    if tags.shape[0] == 0:
        return x.copy()
    pad = tags < 0
    m = row_modulation(tags, layout.t_idx, w.ada_table, tmod)
    out = np.empty_like(x)
    for b in range(x.shape[0]):
        h = norm_modulate(x[b], m[:, 0], m[:, 1], dims.norm_eps)
        hq = dequantize_rows(*quantize_rows_e4m3(h))
        q, k, v = qkv_project_values(hq, layout.pos, wq.w_qkv, w.q_norm, w.k_norm, dims, emulate)
        o = attention(q, pad, k, v, pad, emulate)
        if out_down:
            x1 = out_project_residual_values(x[b], dequantize_rows(*quantize_rows_e4m3(o)),
                                             m[:, 2], wq.w_o)
        else:
            x1 = out_project_residual(x[b], o, m[:, 2], w.w_o)
        x1 = _stream(x1, emulate, stream_f32)
        h2 = norm_modulate(x1, m[:, 3], m[:, 4], dims.norm_eps)
        h2q = dequantize_rows(*quantize_rows_e4m3(h2))
        g = ffn_gate_values(h2q, wq.w13, dims.ffn, emulate)
        if out_down:
            y = ffn_down_residual_values(x1, dequantize_rows(*quantize_rows_e4m3(g)), m[:, 5],
                                         wq.w2)
        else:
            y = ffn_down_residual(x1, g, m[:, 5], w.w2)
        y = _stream(y, emulate, stream_f32)
        out[b] = np.where(pad[:, None], x[b], y)
    return out


# --------------------------------------------------------------------------
# Token reduction in the middle blocks  [ME: "Token-reduction internals": after
# block 3 adjacent horizontal target-video tokens are paired, text, audio and
# reference tokens stay exact; the full-resolution state is kept as a bypass
# and restored before a later block (40, then 30)]
#
# Readings where the page leaves the steps open: a pair is two packed rows r,
# r + 1 that are both target-video rows with the same t_idx, the same t and h
# coordinates and w coordinates 2k and 2k + 1; the merged row is the mean of the
# pair's rows, at the mean of their positions, in the place of the first; at
# the restore point each row of a pair receives the pair's update (the merged
# row's change since the merge), added to the bypass; unpaired rows map one to
# one. Blocks [r0, r1) run on the reduced sequence.
# --------------------------------------------------------------------------

def reduction_pairs(layout, target: np.ndarray) -> np.ndarray:
    """Packed rows that head a pair (their partner is the next row)."""
    tags = np.asarray(layout.tags)
    pos = np.asarray(layout.pos, F)
    ti = np.asarray(layout.t_idx)
    tg = np.asarray(target, bool) & (tags == 0)
    S = tags.shape[0]
    heads = []
    r = 0
    while r + 1 < S:
        w = pos[r, 2]
        if (tg[r] and tg[r + 1] and ti[r] == ti[r + 1] and pos[r, 0] == pos[r + 1, 0]
                and pos[r, 1] == pos[r + 1, 1] and w % 2 == 0 and pos[r + 1, 2] == w + 1):
            heads.append(r)
            r += 2
        else:
            r += 1
    return np.asarray(heads, np.int64)


def reduced_layout(layout, heads: np.ndarray):
    """The sequence with each pair replaced by one row at the first row's place:
    the pair's tag and timestep index and the mean of the two positions.
    Returns (layout, rows) with rows[j] = (first packed row, second or -1)."""
    from types import SimpleNamespace
    S = len(layout.tags)
    tail = np.zeros(S, bool)
    tail[np.asarray(heads, np.int64) + 1] = True
    is_head = np.zeros(S, bool)
    is_head[np.asarray(heads, np.int64)] = True
    keep = np.nonzero(~tail)[0]
    rows = np.stack([keep, np.where(is_head[keep], keep + 1, -1)], 1)
    pos = np.asarray(layout.pos, F)[keep].copy()
    h = is_head[keep]
    pos[h] = 0.5 * (pos[h] + np.asarray(layout.pos, F)[keep[h] + 1])
    tags = np.asarray(layout.tags)[keep]
    return SimpleNamespace(tags=tags, pos=pos, t_idx=np.asarray(layout.t_idx)[keep],
                           timestep=layout.timestep, S=len(keep),
                           video_idx=np.nonzero(tags == 0)[0], audio_idx=np.nonzero(tags == 2)[0],
                           text_idx=np.nonzero(tags == 1)[0]), rows


def merge_rows(x: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """x [S, H] -> [len(rows), H]: a pair's rows averaged, other rows copied."""
    a, b = rows[:, 0], rows[:, 1]
    out = np.array(x[a], F, copy=True)
    p = b >= 0
    out[p] = 0.5 * (x[a[p]] + x[b[p]])
    return out


def restore_rows(bypass: np.ndarray, x_red: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """The full-resolution state: the bypass plus, for every row, the change of
    its reduced row since the merge (both rows of a pair get the same change)."""
    d = x_red - merge_rows(bypass, rows)
    out = np.array(bypass, F, copy=True)
    out[rows[:, 0]] += d
    p = rows[:, 1] >= 0
    out[rows[p, 1]] += d[p]
    return out


def stack_forward_reduced(x: np.ndarray, weights_for_block: Callable[[int], object],
                          n_blocks: int, layout, tmod: np.ndarray, dims, target: np.ndarray,
                          r0: int, r1: int) -> np.ndarray:
    """The stack with blocks [r0, r1) on the token-reduced sequence (B = 1)."""
    y = np.asarray(x, F)
    heads = reduction_pairs(layout, target)
    red, rows = reduced_layout(layout, heads)
    for i in range(min(r0, n_blocks)):
        y = block_forward(y, weights_for_block(i), layout, tmod, dims)
    if r0 < min(r1, n_blocks):
        bypass = y[0]
        z = merge_rows(bypass, rows)[None]
        for i in range(r0, min(r1, n_blocks)):
            z = block_forward(z, weights_for_block(i), red, tmod, dims)
        y = restore_rows(bypass, z[0], rows)[None]
    for i in range(max(r1, r0), n_blocks):
        y = block_forward(y, weights_for_block(i), layout, tmod, dims)
    return y


# --------------------------------------------------------------------------
# a0 / a1: layout validation, tile classes, compaction, pack / unpack
#          [MX: forward arguments; caller builds the packing]
# --------------------------------------------------------------------------

LAYOUT_OK = 0
LAYOUT_BAD = -4


def layout_check(layout, n_t: Optional[int] = None) -> int:
    """0 if the layout is consistent, else -4.

    Tags in {-1, 0, 1, 2}; every t_idx in [0, n_t); positions finite; each
    index tensor in range, free of duplicates, pointing only at rows of its
    modality, and as long as the number of such rows.
    """
    tags = np.asarray(layout.tags)
    S = tags.shape[0]
    nt = layout.timestep.shape[0] if n_t is None else n_t
    if np.any((tags < -1) | (tags > 2)):
        return LAYOUT_BAD
    ti = np.asarray(layout.t_idx)
    if ti.shape[0] != S or np.any((ti < 0) | (ti >= nt)):
        return LAYOUT_BAD
    if not np.all(np.isfinite(np.asarray(layout.pos))):
        return LAYOUT_BAD
    for idx, tag in ((layout.video_idx, 0), (layout.text_idx, 1), (layout.audio_idx, 2)):
        idx = np.asarray(idx, np.int64)
        if np.any((idx < 0) | (idx >= S)):
            return LAYOUT_BAD
        if np.unique(idx).shape[0] != idx.shape[0]:
            return LAYOUT_BAD
        if np.any(tags[idx] != tag):
            return LAYOUT_BAD
        if idx.shape[0] != int(np.count_nonzero(tags == tag)):
            return LAYOUT_BAD
    return LAYOUT_OK


def tile_classes(tags: np.ndarray, tile: int = TILE) -> np.ndarray:
    """Per row tile: 0 all rows valid, 1 all rows padding, 2 mixed."""
    tags = np.asarray(tags)
    S = tags.shape[0]
    n = (S + tile - 1) // tile
    out = np.zeros(n, np.uint8)
    for i in range(n):
        seg = tags[i * tile:min(S, (i + 1) * tile)]
        npad = int(np.count_nonzero(seg < 0))
        out[i] = 0 if npad == 0 else (1 if npad == seg.shape[0] else 2)
    return out


def compaction_perm(tags: np.ndarray) -> np.ndarray:
    """Row order with valid rows first then padding rows, each in packed order."""
    tags = np.asarray(tags)
    return np.concatenate([np.nonzero(tags >= 0)[0], np.nonzero(tags < 0)[0]]).astype(np.int32)


def pack_rows(layout, video: np.ndarray, audio: np.ndarray, text: np.ndarray,
              H: int) -> np.ndarray:
    """Scatter per-modality rows [B, N_m, H] into the packed [B, S, H]; padding rows 0."""
    B = max(a.shape[0] for a in (video, audio, text))
    out = np.zeros((B, layout.S, H), dtype=video.dtype)
    for src, idx in ((video, layout.video_idx), (audio, layout.audio_idx),
                     (text, layout.text_idx)):
        for i, r in enumerate(np.asarray(idx)):
            out[:, r] = src[:, i]
    return out


def unpack_rows(layout, x: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gather packed rows back to per-modality [B, N_m, H], in index order."""
    return tuple(np.stack([x[:, r] for r in np.asarray(idx)], axis=1)
                 if len(idx) else np.zeros((x.shape[0], 0, x.shape[2]), x.dtype)
                 for idx in (layout.video_idx, layout.audio_idx, layout.text_idx))
