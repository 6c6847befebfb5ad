"""Seeded synthetic inputs shaped like the MiniMax-H3 packed-sequence workloads.

Source: "MiniMaxH3Transformer3DModel" (diffusers v0.43.0 docs), constructor
parameters and `forward` arguments: the packed 1-D sequence carries per-row
modality tags (0 video, 1 text, 2 audio; -1 padding rows), (t, h, w) rotary
positions, per-row timestep indices into the distinct `timestep` values, and
three index tensors that place the video, audio and text rows.

Everything here is input preparation: random draws, rounding of those draws to
bf16 storage, and row bookkeeping. No step of the block's computation lives in
this file. Random streams are NumPy PCG64 generators seeded with
``[config, tensor_key, block, chunk]``; large tensors are drawn in fixed
chunks of rows so the values do not depend on the number of worker threads.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

TAG_VIDEO = 0
TAG_TEXT = 1
TAG_AUDIO = 2
TAG_PAD = -1

CONFIG_NAMES = {
    1: "tiny single block, S=256 with 16 padding rows",
    2: "full-width single block, S=8192, no padding",
    3: "full-width single block, S=16384 with 512 padding rows in 4 runs",
    4: "full-width single block, S=32768, no padding",
    5: "full-width 50-block stack, S=16384 (config-3 layout), 2 timesteps",
}


@dataclasses.dataclass(frozen=True)
class Dims:
    """Block dimensions (constructor parameters of the transformer)."""

    hidden: int
    heads: int
    head_dim: int
    ffn: int
    time_embed_dim: int
    time_hidden: int
    freq_dim: int = 256
    rope_freq_dim: int = 16
    rope_theta: float = 10000.0
    norm_eps: float = 1e-5
    qk_norm_eps: float = 1e-5
    n_modalities: int = 3
    # the denoiser around the stack
    in_channels: int = 24
    patch_size: Tuple[int, int, int] = (1, 2, 2)
    audio_in_channels: int = 32
    text_dim: int = 5120
    num_refiner_layers: int = 2
    final_norm_eps: float = 1e-5

    @property
    def attn_width(self) -> int:
        return self.heads * self.head_dim

    @property
    def video_channels(self) -> int:
        """Channels of one patched video latent row: in_channels * prod(patch_size)."""
        return self.in_channels * int(np.prod(self.patch_size))


# Default constructor values of MiniMaxH3Transformer3DModel.
FULL_DIMS = Dims(hidden=5376, heads=56, head_dim=128, ffn=14336,
                 time_embed_dim=2688, time_hidden=5376)
# The small single-block case: hidden 512, 6 heads of 128 (768 > 512),
# ffn 1408, time_embed_dim 256; the timestep MLP's hidden width equals the
# hidden size, as it does at full width.
TINY_DIMS = Dims(hidden=512, heads=6, head_dim=128, ffn=1408,
                 time_embed_dim=256, time_hidden=512, text_dim=384)


@dataclasses.dataclass
class Layout:
    """One packed layout shared by every batch element."""

    tags: np.ndarray        # [S] int32
    pos: np.ndarray         # [S, 3] float32 (t, h, w)
    t_idx: np.ndarray       # [S] int32, index into `timestep`
    timestep: np.ndarray    # [n_t] float32 in [0, 1]
    video_idx: np.ndarray   # [N_v] int32
    audio_idx: np.ndarray   # [N_a] int32
    text_idx: np.ndarray    # [N_t] int32

    @property
    def S(self) -> int:
        return int(self.tags.shape[0])

    @property
    def n_t(self) -> int:
        return int(self.timestep.shape[0])

    @property
    def n_valid(self) -> int:
        return int(np.count_nonzero(self.tags >= 0))


@dataclasses.dataclass
class BlockWeights:
    """One block's parameters; matrices as bf16 bit patterns (uint16), [out, in]."""

    w_qkv: np.ndarray      # [3*NH*D, H]; row n*3D + {0, D, 2D} + d = q/k/v of head n
    q_norm: np.ndarray     # [D]
    k_norm: np.ndarray     # [D]
    w_o: np.ndarray        # [H, NH*D]
    w13: np.ndarray        # [2F, H]; rows [256j, 256j+128) = W1 rows [128j, 128j+128),
                           #          rows [256j+128, 256j+256) = W3 rows [128j, 128j+128)
    w2: np.ndarray         # [H, F]
    ada_table: np.ndarray  # [n_mod, 6, H] float32


@dataclasses.dataclass
class PrologueWeights:
    """fp32 timestep-MLP and shared AdaLN projection weights, [out, in]."""

    w_t1: np.ndarray   # [time_hidden, freq_dim]
    w_t2: np.ndarray   # [time_embed_dim, time_hidden]
    w_proj: np.ndarray  # [6*H, time_embed_dim]


# --------------------------------------------------------------------------
# bf16 storage of random draws (round to nearest even on the fp32 bits)
# --------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


_CHUNK = 1 << 22  # elements per independently seeded chunk


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _normal_chunks(shape: Tuple[int, ...], seed: Sequence[int], std: float, mean: float,
                   to_bf16: bool) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16 if to_bf16 else np.float32)
    n_chunks = (n + _CHUNK - 1) // _CHUNK

    def fill(i: int) -> None:
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        g = np.random.default_rng(list(seed) + [i])
        v = g.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        if mean != 0.0:
            v += np.float32(mean)
        out[lo:hi] = f32_to_bf16_bits(v) if to_bf16 else v

    if n_chunks <= 1:
        for i in range(n_chunks):
            fill(i)
    else:
        with ThreadPoolExecutor(max_workers=min(_threads(), n_chunks)) as ex:
            list(ex.map(fill, range(n_chunks)))
    return out.reshape(shape)


def _normal_f32(shape: Tuple[int, ...], seed: Sequence[int], std: float,
                mean: float = 0.0) -> np.ndarray:
    return _normal_chunks(shape, seed, std, mean, False)


def normal_bf16(shape: Tuple[int, ...], seed: Sequence[int], std: float = 1.0,
                mean: float = 0.0) -> np.ndarray:
    """N(mean, std^2) draws rounded to bf16; returns uint16 bit patterns."""
    return _normal_chunks(tuple(shape), seed, std, mean, True)


def normal_f32(shape: Tuple[int, ...], seed: Sequence[int], std: float = 1.0) -> np.ndarray:
    return _normal_f32(tuple(shape), seed, std)


def uniform_f32(shape: Tuple[int, ...], seed: Sequence[int]) -> np.ndarray:
    g = np.random.default_rng(list(seed))
    return g.random(shape, dtype=np.float32)


def random_code_bytes(shape: Tuple[int, ...], seed: Sequence[int]) -> np.ndarray:
    """Uniform random bytes, excluding 0x7F and 0xFF (the two NaN codes of the
    8-bit e4m3 format): operands for the 8-bit GEMM steps."""
    g = np.random.default_rng(list(seed))
    b = g.integers(0, 254, size=shape, dtype=np.int64)  # 254 values, then skip 0x7F
    b = np.where(b >= 0x7F, b + 1, b)
    return b.astype(np.uint8)


def random_scales(n: int, seed: Sequence[int], lo: float = -12.0, hi: float = -6.0) -> np.ndarray:
    """n positive float32 scales 2^u, u uniform in [lo, hi)."""
    g = np.random.default_rng(list(seed))
    return np.exp2(g.uniform(lo, hi, size=n)).astype(np.float32)


# --------------------------------------------------------------------------
# Packed layouts
# --------------------------------------------------------------------------

def make_layout(segments: List[Tuple], timesteps: str = "per_row",
                seed: Sequence[int] = (0,), t_values: Optional[np.ndarray] = None,
                t_idx: Optional[np.ndarray] = None) -> Layout:
    """Build a packed layout from segments in row order.

    Segments:
      ("text", i0, i1)            text rows i0..i1-1, position (i, 0, 0)
      ("video", grid, f0, f1)     video frames f0..f1-1 of grid (T, Hh, Ww),
                                  row-major (t, h, w), position (t, h, w)
      ("audio", j0, j1)           audio rows j0..j1-1, position (j, 0, 0)
      ("pad", n)                  n padding rows, position (0, 0, 0)

    ``timesteps == "per_row"`` gives every row its own t ~ U[0, 1]
    (n_t = S, t_idx = arange(S)); otherwise pass ``t_values`` and ``t_idx``.
    """
    tags: List[np.ndarray] = []
    pos: List[np.ndarray] = []
    for seg in segments:
        kind = seg[0]
        if kind == "text":
            i = np.arange(seg[1], seg[2], dtype=np.float32)
            tags.append(np.full(i.shape[0], TAG_TEXT, np.int32))
            pos.append(np.stack([i, np.zeros_like(i), np.zeros_like(i)], 1))
        elif kind == "audio":
            j = np.arange(seg[1], seg[2], dtype=np.float32)
            tags.append(np.full(j.shape[0], TAG_AUDIO, np.int32))
            pos.append(np.stack([j, np.zeros_like(j), np.zeros_like(j)], 1))
        elif kind == "video":
            (T, Hh, Ww), f0, f1 = seg[1], seg[2], seg[3]
            tt, hh, ww = np.meshgrid(np.arange(f0, f1), np.arange(Hh), np.arange(Ww),
                                     indexing="ij")
            p = np.stack([tt.ravel(), hh.ravel(), ww.ravel()], 1).astype(np.float32)
            tags.append(np.full(p.shape[0], TAG_VIDEO, np.int32))
            pos.append(p)
        elif kind == "pad":
            tags.append(np.full(seg[1], TAG_PAD, np.int32))
            pos.append(np.zeros((seg[1], 3), np.float32))
        else:
            raise ValueError(kind)
    tag_arr = np.concatenate(tags) if tags else np.zeros(0, np.int32)
    pos_arr = np.concatenate(pos) if pos else np.zeros((0, 3), np.float32)
    S = tag_arr.shape[0]
    if timesteps == "per_row":
        t_values = uniform_f32((S,), list(seed) + [2])
        t_idx = np.arange(S, dtype=np.int32)
    else:
        assert t_values is not None and t_idx is not None
    return Layout(
        tags=tag_arr.astype(np.int32),
        pos=np.ascontiguousarray(pos_arr, dtype=np.float32),
        t_idx=np.ascontiguousarray(t_idx, dtype=np.int32),
        timestep=np.ascontiguousarray(t_values, dtype=np.float32),
        video_idx=np.nonzero(tag_arr == TAG_VIDEO)[0].astype(np.int32),
        audio_idx=np.nonzero(tag_arr == TAG_AUDIO)[0].astype(np.int32),
        text_idx=np.nonzero(tag_arr == TAG_TEXT)[0].astype(np.int32),
    )


def config_dims(cfg: int) -> Dims:
    return TINY_DIMS if cfg == 1 else FULL_DIMS


def _config3_segments() -> List[Tuple]:
    g = (12, 32, 32)
    return [("text", 0, 960), ("pad", 128), ("text", 960, 1024),
            ("video", g, 0, 6), ("pad", 128), ("video", g, 6, 12),
            ("audio", 0, 1280), ("pad", 128), ("audio", 1280, 2560), ("pad", 128)]


def config_layout(cfg: int) -> Layout:
    """The packed layouts of the five workloads (row order as listed)."""
    seed = [cfg]
    if cfg == 1:
        segs = [("text", 0, 48), ("video", (4, 4, 8), 0, 4), ("pad", 8),
                ("audio", 0, 64), ("pad", 8)]
        return make_layout(segs, seed=seed)
    if cfg == 2:
        segs = [("text", 0, 512), ("video", (6, 32, 32), 0, 6), ("audio", 0, 1536)]
        return make_layout(segs, seed=seed)
    if cfg == 3:
        return make_layout(_config3_segments(), seed=seed)
    if cfg == 4:
        segs = [("text", 0, 512), ("video", (30, 32, 32), 0, 30), ("audio", 0, 1536)]
        return make_layout(segs, seed=seed)
    if cfg == 5:
        base = make_layout(_config3_segments(), seed=seed)
        # Two distinct timesteps: conditioning rows (text and the first video
        # frame) at t = 0, target rows (other video frames, audio) at t ~ U[0,1].
        u = uniform_f32((1,), [cfg, 2])
        t_values = np.array([0.0, float(u[0])], np.float32)
        cond = (base.tags == TAG_TEXT) | ((base.tags == TAG_VIDEO) & (base.pos[:, 0] == 0))
        tgt = ((base.tags == TAG_VIDEO) & (base.pos[:, 0] > 0)) | (base.tags == TAG_AUDIO)
        t_idx = np.zeros(base.S, np.int32)
        t_idx[tgt] = 1
        t_idx[cond] = 0
        base.timestep = t_values
        base.t_idx = t_idx
        return base
    raise ValueError(cfg)


def random_layout(S: int, seed: int, pad_runs: int = 2, max_run: int = 40,
                  n_t: Optional[int] = None) -> Layout:
    """A random packed layout for property and edge-case tests.

    Modalities are drawn per row; ``pad_runs`` runs of padding rows of random
    length (<= max_run) are placed at random offsets. Positions are random
    small integers (stored as fp32); ``n_t`` distinct timesteps (default S).
    """
    g = np.random.default_rng([9999, seed, S])
    tags = g.integers(0, 3, size=S).astype(np.int32)
    for _ in range(pad_runs):
        if S == 0:
            break
        ln = int(g.integers(1, max(2, min(max_run, S) + 1)))
        st = int(g.integers(0, max(1, S - ln + 1)))
        tags[st:st + ln] = TAG_PAD
    pos = g.integers(0, 50, size=(S, 3)).astype(np.float32)
    pos[tags == TAG_PAD] = 0.0
    nt = S if n_t is None else n_t
    t_values = g.random(max(nt, 1), dtype=np.float32)[:nt] if nt > 0 else np.zeros(0, np.float32)
    t_idx = (np.arange(S) if n_t is None else g.integers(0, max(nt, 1), size=S)).astype(np.int32)
    return Layout(
        tags=tags, pos=pos, t_idx=t_idx, timestep=t_values,
        video_idx=np.nonzero(tags == TAG_VIDEO)[0].astype(np.int32),
        audio_idx=np.nonzero(tags == TAG_AUDIO)[0].astype(np.int32),
        text_idx=np.nonzero(tags == TAG_TEXT)[0].astype(np.int32),
    )


# --------------------------------------------------------------------------
# Parameters and activations
# --------------------------------------------------------------------------

_KEYS: Dict[str, int] = {
    "x": 1, "w_qkv": 10, "q_norm": 11, "k_norm": 12, "w_o": 13, "w13": 14,
    "w2": 15, "ada_table": 16, "w_t1": 20, "w_t2": 21, "w_proj": 22,
    "video": 30, "audio": 31, "text": 32, "w_patch_video": 40, "w_patch_audio": 41,
    "w_text": 42, "w_out": 43, "out_table": 44, "w_head_video": 45, "w_head_audio": 46,
}
REFINER_BLOCK0 = 1000  # block index of the first refiner block's random streams

WEIGHT_STD = 0.02


def block_weights(dims: Dims, cfg: int, block: int = 0) -> BlockWeights:
    """Random-init block parameters: matrices ~N(0, 0.02^2) in bf16, QK-norm
    weights 1 + N(0, 0.02^2) in bf16, AdaLN table ~N(0, 0.02^2) in fp32."""
    H, A, D, F = dims.hidden, dims.attn_width, dims.head_dim, dims.ffn

    def s(name: str) -> List[int]:
        return [cfg, _KEYS[name], block]

    return BlockWeights(
        w_qkv=normal_bf16((3 * A, H), s("w_qkv"), WEIGHT_STD),
        q_norm=normal_bf16((D,), s("q_norm"), WEIGHT_STD, 1.0),
        k_norm=normal_bf16((D,), s("k_norm"), WEIGHT_STD, 1.0),
        w_o=normal_bf16((H, A), s("w_o"), WEIGHT_STD),
        w13=normal_bf16((2 * F, H), s("w13"), WEIGHT_STD),
        w2=normal_bf16((H, F), s("w2"), WEIGHT_STD),
        ada_table=normal_f32((dims.n_modalities, 6, H), s("ada_table"), WEIGHT_STD),
    )


def prologue_weights(dims: Dims, cfg: int) -> PrologueWeights:
    def s(name: str) -> List[int]:
        return [cfg, _KEYS[name], 0]

    return PrologueWeights(
        w_t1=normal_f32((dims.time_hidden, dims.freq_dim), s("w_t1"), WEIGHT_STD),
        w_t2=normal_f32((dims.time_embed_dim, dims.time_hidden), s("w_t2"), WEIGHT_STD),
        w_proj=normal_f32((6 * dims.hidden, dims.time_embed_dim), s("w_proj"), WEIGHT_STD),
    )


def activations(dims: Dims, cfg: int, S: int, B: int = 1, key: int = 0) -> np.ndarray:
    """Packed hidden stream x ~ N(0, 1), bf16 bits, [B, S, H]."""
    return normal_bf16((B, S, dims.hidden), [cfg, _KEYS["x"], key], 1.0)


# --------------------------------------------------------------------------
# The denoiser around the stack
# --------------------------------------------------------------------------

@dataclasses.dataclass
class DenoiserWeights:
    """Parameters outside the block stack, [out, in]: float32 patch projections,
    timestep MLP, output modulation and heads; bf16 text projection; the refiner
    blocks (BlockWeights)."""

    w_patch_video: np.ndarray  # [H, C_v] f32
    w_patch_audio: np.ndarray  # [H, C_a] f32
    w_text: np.ndarray         # [H, text_dim] bf16 bits
    refiner: List[BlockWeights]
    w_t1: np.ndarray           # [time_hidden, freq_dim] f32
    w_t2: np.ndarray           # [time_embed_dim, time_hidden] f32
    w_proj: np.ndarray         # [6H, time_embed_dim] f32
    w_out: np.ndarray          # [2H, time_embed_dim] f32: norm_out's (shift, scale)
    out_table: np.ndarray      # [2, 2, H] f32: (video, audio) x (shift, scale)
    w_head_video: np.ndarray   # [C_v, H] f32
    w_head_audio: np.ndarray   # [C_a, H] f32


def denoiser_weights(dims: Dims, cfg: int) -> DenoiserWeights:
    """Random-init parameters outside the stack: matrices ~N(0, 0.02^2) (float32,
    or bf16 for the text projection), the output AdaLN table ~N(0, 0.02^2)."""
    H, E = dims.hidden, dims.time_embed_dim

    def s(name: str) -> List[int]:
        return [cfg, _KEYS[name], 0]

    pw = prologue_weights(dims, cfg)
    return DenoiserWeights(
        w_patch_video=normal_f32((H, dims.video_channels), s("w_patch_video"), WEIGHT_STD),
        w_patch_audio=normal_f32((H, dims.audio_in_channels), s("w_patch_audio"), WEIGHT_STD),
        w_text=normal_bf16((H, dims.text_dim), s("w_text"), WEIGHT_STD),
        refiner=[block_weights(dims, cfg, REFINER_BLOCK0 + i)
                 for i in range(dims.num_refiner_layers)],
        w_t1=pw.w_t1, w_t2=pw.w_t2, w_proj=pw.w_proj,
        w_out=normal_f32((2 * H, E), s("w_out"), WEIGHT_STD),
        out_table=normal_f32((2, 2, H), s("out_table"), WEIGHT_STD),
        w_head_video=normal_f32((dims.video_channels, H), s("w_head_video"), WEIGHT_STD),
        w_head_audio=normal_f32((dims.audio_in_channels, H), s("w_head_audio"), WEIGHT_STD),
    )


def denoiser_inputs(dims: Dims, cfg: int, layout: Layout, B: int = 1):
    """Latent rows of one forward, each in the order of its index tensor:
    video [B, n_video, C_v] and audio [B, n_audio, C_a] float32 ~N(0, 1), text
    condition [B, n_text, text_dim] bf16 ~N(0, 1)."""
    nv, na, nt = (int(np.asarray(a).shape[0]) for a in
                  (layout.video_idx, layout.audio_idx, layout.text_idx))
    return (normal_f32((B, nv, dims.video_channels), [cfg, _KEYS["video"], 0], 1.0),
            normal_f32((B, na, dims.audio_in_channels), [cfg, _KEYS["audio"], 0], 1.0),
            normal_bf16((B, nt, dims.text_dim), [cfg, _KEYS["text"], 0], 1.0))
