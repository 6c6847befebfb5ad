"""ctypes binding of the C ABI in include/h3.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
computation of its own: it turns tensors into device pointers, checks the
returned status and raises ``H3Error`` on failure. Device memory, streams and
tensors come from PyTorch; all of the block's arithmetic runs in libh3.so.

The library must be built (``python -m audio_generation_b200.build``); there is
no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libh3.so")

H3_OK = 0
H3_ERR_ARG = -1
H3_ERR_SHAPE = -2
H3_ERR_ALIGN = -3
H3_ERR_LAYOUT = -4
H3_ERR_WORKSPACE = -5
H3_ERR_CUDA = -6
H3_ERR_TIMEOUT = -7


class H3Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {h3_status_string(status)} ({status})")


class h3_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "hidden", "heads", "head_dim", "ffn", "time_embed_dim", "time_hidden", "freq_dim",
        "rope_freq_dim", "n_modalities")] + [
        ("rope_theta", ctypes.c_float), ("norm_eps", ctypes.c_float),
        ("qk_norm_eps", ctypes.c_float)]


class h3_layout_desc(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int), ("n_t", ctypes.c_int), ("n_video", ctypes.c_int),
                ("n_audio", ctypes.c_int), ("n_text", ctypes.c_int),
                ("pos", ctypes.c_void_p), ("tags", ctypes.c_void_p), ("t_idx", ctypes.c_void_p),
                ("video_idx", ctypes.c_void_p), ("audio_idx", ctypes.c_void_p),
                ("text_idx", ctypes.c_void_p)]


class h3_block_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_qkv", "q_norm", "k_norm", "w_o", "w13", "w2", "ada_table")]


class h3_io_dims(ctypes.Structure):
    _fields_ = [("video_channels", ctypes.c_int), ("audio_channels", ctypes.c_int),
                ("text_dim", ctypes.c_int), ("final_norm_eps", ctypes.c_float)]


class h3_io_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_patch_video", "w_patch_audio", "w_text", "w_t1", "w_t2", "w_proj", "w_out",
        "out_table", "w_head_video", "w_head_audio")]


class h3_block_weights_e4m3(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_qkv_codes", "w_qkv_scales", "w13_codes", "w13_scales", "w_o_codes", "w_o_scales",
        "w2_codes", "w2_scales")]


H3_MAX_RANKS = 8


class h3_ulysses_peers(ctypes.Structure):
    _fields_ = [("n_ranks", ctypes.c_int), ("rank", ctypes.c_int),
                ("q", ctypes.c_void_p * H3_MAX_RANKS), ("k", ctypes.c_void_p * H3_MAX_RANKS),
                ("v", ctypes.c_void_p * H3_MAX_RANKS), ("o", ctypes.c_void_p * H3_MAX_RANKS)]


_lib: Optional[ctypes.CDLL] = None

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGNATURES = {
    "h3_status_string": (ctypes.c_char_p, [_i]),
    "h3_abi_version": (_i, []),
    "h3_layout_prepare": (_i, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_layout_desc), _vp,
                               ctypes.POINTER(_vp)]),
    "h3_layout_destroy": (None, [_vp]),
    "h3_layout_error": (_i, [_vp]),
    "h3_layout_export": (_i, [_vp, _vp, _vp, _vp]),
    "h3_workspace_size": (_sz, [ctypes.POINTER(h3_dims), _i, _i]),
    "h3_pack_rows": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "h3_unpack_rows": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "h3_timestep_workspace_size": (_sz, [ctypes.POINTER(h3_dims), _i]),
    "h3_timestep_modulation": (_i, [ctypes.POINTER(h3_dims), _i, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _sz, _vp]),
    "h3_timestep_error": (_i, []),
    "h3_timestep_modulation_noalloc": (_i, [ctypes.POINTER(h3_dims), _i, _vp, _vp, _vp, _vp,
                                            _vp, _vp]),
    "h3_norm_modulate": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "h3_qkv_rope": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                         _vp]),
    "h3_attention": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp, _vp]),
    "h3_out_residual": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "h3_ffn_up": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp]),
    "h3_ffn_down_residual": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp, _vp,
                                  _vp]),
    "h3_block_forward": (_i, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_block_weights), _vp,
                              _vp, _vp, _i, _vp, _sz, _vp]),
    "h3_quantize_e4m3_rows": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "h3_qkv_rope_to_heads": (_i, [ctypes.POINTER(h3_dims), _vp, _vp, _vp, _vp, _vp,
                                  ctypes.POINTER(h3_ulysses_peers), _vp]),
    "h3_attention_to_rows": (_i, [ctypes.POINTER(h3_dims), _vp, _vp, _vp, _vp,
                                  ctypes.POINTER(h3_ulysses_peers), _vp]),
    "h3_norm_modulate_e4m3": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _i, _vp, _vp, _vp, _vp,
                                   _vp, _vp]),
    "h3_qkv_rope_e4m3": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp,
                              _vp, _vp, _vp, _vp]),
    "h3_ffn_up_e4m3": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "h3_out_residual_e4m3": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _vp, _vp]),
    "h3_ffn_down_residual_e4m3": (_i, [ctypes.POINTER(h3_dims), _vp, _i, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _vp, _vp]),
    "h3_workspace_size_e4m3": (_sz, [ctypes.POINTER(h3_dims), _i, _i]),
    "h3_stack_forward_e4m3": (_i, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_block_weights),
                                   ctypes.POINTER(h3_block_weights_e4m3), _i, _vp, _vp, _vp, _i,
                                   _vp, _sz, _vp]),
    "h3_block_forward_e4m3": (_i, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_block_weights),
                                   ctypes.POINTER(h3_block_weights_e4m3), _vp, _vp, _vp, _i, _vp,
                                   _sz, _vp]),
    "h3_layout_reduce": (_i, [ctypes.POINTER(h3_dims), _vp, _vp, _vp, ctypes.POINTER(_vp)]),
    "h3_stack_reduced_workspace_size": (_sz, [ctypes.POINTER(h3_dims), _vp, _vp, _i]),
    "h3_stack_forward_reduced": (_i, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_block_weights),
                                      _i, _vp, _vp, _i, _i, _vp, _vp, _i, _vp, _sz, _vp]),
    "h3_forward_workspace_size": (_sz, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_io_dims),
                                        _vp, _i]),
    "h3_forward": (_i, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_io_dims),
                        ctypes.POINTER(h3_io_weights), ctypes.POINTER(h3_block_weights), _i,
                        ctypes.POINTER(h3_block_weights), _i, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                        _vp, _vp, _i, _vp, _sz, _vp]),
    "h3_stack_forward": (_i, [ctypes.POINTER(h3_dims), ctypes.POINTER(h3_block_weights), _i, _vp,
                              _vp, _vp, _i, _vp, _sz, _vp]),
}


def lib() -> ctypes.CDLL:
    """Load libh3.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m audio_generation_b200.build` (no fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


# ---------------------------------------------------------------- marshalling helpers

def _ptr(t) -> Optional[int]:
    """Device (or host) address of a tensor / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check(status: int, where: str) -> None:
    if status != H3_OK:
        raise H3Error(status, where)


def make_dims(d) -> h3_dims:
    """h3_dims from any object with the constructor-parameter attributes."""
    return h3_dims(hidden=d.hidden, heads=d.heads, head_dim=d.head_dim, ffn=d.ffn,
                   time_embed_dim=d.time_embed_dim, time_hidden=d.time_hidden,
                   freq_dim=d.freq_dim, rope_freq_dim=d.rope_freq_dim,
                   n_modalities=getattr(d, "n_modalities", 3), rope_theta=d.rope_theta,
                   norm_eps=d.norm_eps, qk_norm_eps=d.qk_norm_eps)


def make_block_weights(w_qkv, q_norm, k_norm, w_o, w13, w2, ada_table) -> h3_block_weights:
    return h3_block_weights(*[_ptr(t) for t in (w_qkv, q_norm, k_norm, w_o, w13, w2, ada_table)])


# ---------------------------------------------------------------- entry points

def h3_status_string(status: int) -> str:
    return lib().h3_status_string(status).decode()


def h3_abi_version() -> int:
    return lib().h3_abi_version()


class Layout:
    """Owns an h3_layout_t; released by close() or garbage collection."""

    def __init__(self, handle: int, S: int):
        self.handle = handle
        self.S = S

    def close(self) -> None:
        if self.handle:
            lib().h3_layout_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def _as_param_(self):
        return self.handle


def h3_layout_prepare(dims: h3_dims, S: int, n_t: int, pos, tags, t_idx, video_idx, audio_idx,
                      text_idx, stream=None) -> Layout:
    desc = h3_layout_desc(S=S, n_t=n_t, n_video=_numel(video_idx), n_audio=_numel(audio_idx),
                          n_text=_numel(text_idx), pos=_ptr(pos), tags=_ptr(tags),
                          t_idx=_ptr(t_idx), video_idx=_ptr(video_idx),
                          audio_idx=_ptr(audio_idx), text_idx=_ptr(text_idx))
    out = ctypes.c_void_p()
    _check(lib().h3_layout_prepare(ctypes.byref(dims), ctypes.byref(desc), _stream(stream),
                                   ctypes.byref(out)), "h3_layout_prepare")
    return Layout(out.value, S)


def _numel(t) -> int:
    return 0 if t is None else int(t.numel())


def h3_layout_destroy(layout: Layout) -> None:
    layout.close()


def h3_layout_error(layout: Layout) -> int:
    return lib().h3_layout_error(layout.handle)


def h3_layout_export(layout: Layout, perm_host=None, tile_class_host=None) -> int:
    """Fill host numpy arrays (perm int32 [S], tile classes uint8); return n_valid."""
    nv = ctypes.c_int32(0)
    pp = perm_host.ctypes.data if perm_host is not None else None
    tp = tile_class_host.ctypes.data if tile_class_host is not None else None
    _check(lib().h3_layout_export(layout.handle, pp, tp, ctypes.addressof(nv)),
           "h3_layout_export")
    return int(nv.value)


def h3_workspace_size(dims: h3_dims, B: int, S: int) -> int:
    return int(lib().h3_workspace_size(ctypes.byref(dims), B, S))


def h3_pack_rows(layout: Layout, B: int, row_elems: int, video, audio, text, x_packed,
                 stream=None) -> None:
    _check(lib().h3_pack_rows(layout.handle, B, row_elems, _ptr(video), _ptr(audio), _ptr(text),
                              _ptr(x_packed), _stream(stream)), "h3_pack_rows")


def h3_unpack_rows(layout: Layout, B: int, row_elems: int, x_packed, video, audio, text,
                   stream=None) -> None:
    _check(lib().h3_unpack_rows(layout.handle, B, row_elems, _ptr(x_packed), _ptr(video),
                                _ptr(audio), _ptr(text), _stream(stream)), "h3_unpack_rows")


def h3_timestep_workspace_size(dims: h3_dims, n_t: int) -> int:
    return int(lib().h3_timestep_workspace_size(ctypes.byref(dims), n_t))


def h3_timestep_modulation(dims: h3_dims, n_t: int, t, w_t1, w_t2, w_proj, tmod, ws,
                           ws_bytes: int, stream=None) -> None:
    _check(lib().h3_timestep_modulation(ctypes.byref(dims), n_t, _ptr(t), _ptr(w_t1),
                                        _ptr(w_t2), _ptr(w_proj), _ptr(tmod), _ptr(ws),
                                        ws_bytes, _stream(stream)), "h3_timestep_modulation")


def h3_timestep_error() -> int:
    return lib().h3_timestep_error()


def h3_timestep_modulation_noalloc(dims: h3_dims, n_t: int, t, w_t1, w_t2, w_proj, tmod,
                                   stream=None) -> None:
    """h3_timestep_modulation with library-owned scratch (no allocation; see include/h3.h)."""
    _check(lib().h3_timestep_modulation_noalloc(ctypes.byref(dims), n_t, _ptr(t), _ptr(w_t1),
                                                _ptr(w_t2), _ptr(w_proj), _ptr(tmod),
                                                _stream(stream)),
           "h3_timestep_modulation_noalloc")


def h3_norm_modulate(dims: h3_dims, layout: Layout, B: int, which: int, x, ada_table, tmod, h,
                     stream=None) -> None:
    _check(lib().h3_norm_modulate(ctypes.byref(dims), layout.handle, B, which, _ptr(x),
                                  _ptr(ada_table), _ptr(tmod), _ptr(h), _stream(stream)),
           "h3_norm_modulate")


def h3_qkv_rope(dims: h3_dims, layout: Layout, B: int, h, w_qkv, q_norm, k_norm, q, k, v,
                stream=None) -> None:
    _check(lib().h3_qkv_rope(ctypes.byref(dims), layout.handle, B, _ptr(h), _ptr(w_qkv),
                             _ptr(q_norm), _ptr(k_norm), _ptr(q), _ptr(k), _ptr(v),
                             _stream(stream)), "h3_qkv_rope")


def h3_attention(dims: h3_dims, layout: Layout, B: int, q, k, v, o, stream=None) -> None:
    _check(lib().h3_attention(ctypes.byref(dims), layout.handle, B, _ptr(q), _ptr(k), _ptr(v),
                              _ptr(o), _stream(stream)), "h3_attention")


def h3_out_residual(dims: h3_dims, layout: Layout, B: int, o, w_o, ada_table, tmod, x,
                    stream=None) -> None:
    _check(lib().h3_out_residual(ctypes.byref(dims), layout.handle, B, _ptr(o), _ptr(w_o),
                                 _ptr(ada_table), _ptr(tmod), _ptr(x), _stream(stream)),
           "h3_out_residual")


def h3_ffn_up(dims: h3_dims, layout: Layout, B: int, h2, w13, g, stream=None) -> None:
    _check(lib().h3_ffn_up(ctypes.byref(dims), layout.handle, B, _ptr(h2), _ptr(w13), _ptr(g),
                           _stream(stream)), "h3_ffn_up")


def h3_ffn_down_residual(dims: h3_dims, layout: Layout, B: int, g, w2, ada_table, tmod, x,
                         stream=None) -> None:
    _check(lib().h3_ffn_down_residual(ctypes.byref(dims), layout.handle, B, _ptr(g), _ptr(w2),
                                      _ptr(ada_table), _ptr(tmod), _ptr(x), _stream(stream)),
           "h3_ffn_down_residual")


def h3_block_forward(dims: h3_dims, weights: h3_block_weights, layout: Layout, tmod, x, B: int,
                     ws, ws_bytes: int, stream=None) -> None:
    _check(lib().h3_block_forward(ctypes.byref(dims), ctypes.byref(weights), layout.handle,
                                  _ptr(tmod), _ptr(x), B, _ptr(ws), ws_bytes, _stream(stream)),
           "h3_block_forward")


def h3_stack_forward(dims: h3_dims, weights: Sequence[h3_block_weights], layout: Layout, tmod,
                     x, B: int, ws, ws_bytes: int, stream=None) -> None:
    arr = (h3_block_weights * max(1, len(weights)))(*weights)
    _check(lib().h3_stack_forward(ctypes.byref(dims), arr, len(weights), layout.handle,
                                  _ptr(tmod), _ptr(x), B, _ptr(ws), ws_bytes, _stream(stream)),
           "h3_stack_forward")


def make_io_dims(d) -> h3_io_dims:
    """h3_io_dims from any object with video_channels, audio_in_channels,
    text_dim and final_norm_eps attributes."""
    return h3_io_dims(video_channels=d.video_channels, audio_channels=d.audio_in_channels,
                      text_dim=d.text_dim, final_norm_eps=d.final_norm_eps)


def make_io_weights(w_patch_video, w_patch_audio, w_text, w_t1, w_t2, w_proj, w_out, out_table,
                    w_head_video, w_head_audio) -> h3_io_weights:
    return h3_io_weights(*[_ptr(t) for t in (w_patch_video, w_patch_audio, w_text, w_t1, w_t2,
                                             w_proj, w_out, out_table, w_head_video,
                                             w_head_audio)])


def h3_forward_workspace_size(dims: h3_dims, io: h3_io_dims, layout: Layout, B: int) -> int:
    return lib().h3_forward_workspace_size(ctypes.byref(dims), ctypes.byref(io), layout.handle, B)


H3_CORE_RUN, H3_CORE_STORE, H3_CORE_REUSE = 0, 1, 2


def h3_forward(dims: h3_dims, io: h3_io_dims, io_weights: h3_io_weights,
               refiner: Sequence[h3_block_weights], blocks: Sequence[h3_block_weights],
               layout: Layout, timestep, B: int, video, audio, text, video_out, audio_out, ws,
               ws_bytes: int, stream=None, core_residual=None, core_mode: int = 0) -> None:
    ref = (h3_block_weights * max(1, len(refiner)))(*refiner)
    blk = (h3_block_weights * max(1, len(blocks)))(*blocks)
    _check(lib().h3_forward(ctypes.byref(dims), ctypes.byref(io), ctypes.byref(io_weights), ref,
                            len(refiner), blk, len(blocks), layout.handle, _ptr(timestep), B,
                            _ptr(video), _ptr(audio), _ptr(text), _ptr(video_out),
                            _ptr(audio_out), _ptr(core_residual), core_mode, _ptr(ws), ws_bytes,
                            _stream(stream)),
           "h3_forward")


def h3_layout_reduce(dims: h3_dims, full: Layout, target, stream=None) -> Layout:
    out = ctypes.c_void_p()
    _check(lib().h3_layout_reduce(ctypes.byref(dims), full.handle, _ptr(target),
                                  _stream(stream), ctypes.byref(out)), "h3_layout_reduce")
    return Layout(out.value, -1)


def h3_stack_reduced_workspace_size(dims: h3_dims, full: Layout, reduced: Layout, B: int) -> int:
    return lib().h3_stack_reduced_workspace_size(ctypes.byref(dims), full.handle, reduced.handle, B)


def h3_stack_forward_reduced(dims: h3_dims, weights: Sequence[h3_block_weights], full: Layout,
                             reduced: Layout, r0: int, r1: int, tmod, x, B: int, ws, ws_bytes: int,
                             stream=None) -> None:
    arr = (h3_block_weights * max(1, len(weights)))(*weights)
    _check(lib().h3_stack_forward_reduced(ctypes.byref(dims), arr, len(weights), full.handle,
                                          reduced.handle, r0, r1, _ptr(tmod), _ptr(x), B, _ptr(ws),
                                          ws_bytes, _stream(stream)),
           "h3_stack_forward_reduced")


def h3_quantize_e4m3_rows(w, rows: int, K: int, codes, scales, stream=None) -> None:
    _check(lib().h3_quantize_e4m3_rows(_ptr(w), rows, K, _ptr(codes), _ptr(scales),
                                       _stream(stream)), "h3_quantize_e4m3_rows")


def make_peers(rank: int, q, k, v, o) -> h3_ulysses_peers:
    """The exchange destinations of one rank: q, k, v, o are per-rank lists of
    tensors or raw device addresses (ints), one entry per rank."""
    P = len(q)
    if not (len(k) == len(v) == len(o) == P) or not 1 <= P <= H3_MAX_RANKS:
        raise ValueError("one q, k, v and o destination per rank, at most %d ranks" % H3_MAX_RANKS)
    addr = lambda t: t if isinstance(t, int) else _ptr(t)
    p = h3_ulysses_peers()
    p.n_ranks, p.rank = P, rank
    for j in range(P):
        p.q[j], p.k[j], p.v[j], p.o[j] = addr(q[j]), addr(k[j]), addr(v[j]), addr(o[j])
    return p


def h3_qkv_rope_to_heads(dims: h3_dims, chunk: Layout, h, w_qkv, q_norm, k_norm,
                         peers: h3_ulysses_peers, stream=None) -> None:
    _check(lib().h3_qkv_rope_to_heads(ctypes.byref(dims), chunk.handle, _ptr(h), _ptr(w_qkv),
                                      _ptr(q_norm), _ptr(k_norm), ctypes.byref(peers),
                                      _stream(stream)), "h3_qkv_rope_to_heads")


def h3_attention_to_rows(dims: h3_dims, full: Layout, q, k, v, peers: h3_ulysses_peers,
                         stream=None) -> None:
    _check(lib().h3_attention_to_rows(ctypes.byref(dims), full.handle, _ptr(q), _ptr(k), _ptr(v),
                                      ctypes.byref(peers), _stream(stream)),
           "h3_attention_to_rows")


def h3_norm_modulate_e4m3(dims: h3_dims, layout: Layout, B: int, which: int, x, ada_table, tmod,
                          codes, scales, stream=None) -> None:
    _check(lib().h3_norm_modulate_e4m3(ctypes.byref(dims), layout.handle, B, which, _ptr(x),
                                       _ptr(ada_table), _ptr(tmod), _ptr(codes), _ptr(scales),
                                       _stream(stream)), "h3_norm_modulate_e4m3")


def h3_qkv_rope_e4m3(dims: h3_dims, layout: Layout, B: int, h_codes, h_scales, w_codes,
                     w_scales, q_norm, k_norm, q, k, v, stream=None) -> None:
    _check(lib().h3_qkv_rope_e4m3(ctypes.byref(dims), layout.handle, B, _ptr(h_codes),
                                  _ptr(h_scales), _ptr(w_codes), _ptr(w_scales), _ptr(q_norm),
                                  _ptr(k_norm), _ptr(q), _ptr(k), _ptr(v), _stream(stream)),
           "h3_qkv_rope_e4m3")


def h3_ffn_up_e4m3(dims: h3_dims, layout: Layout, B: int, h2_codes, h2_scales, w_codes, w_scales,
                   g, stream=None) -> None:
    _check(lib().h3_ffn_up_e4m3(ctypes.byref(dims), layout.handle, B, _ptr(h2_codes),
                                _ptr(h2_scales), _ptr(w_codes), _ptr(w_scales), _ptr(g),
                                _stream(stream)), "h3_ffn_up_e4m3")


def make_block_weights_e4m3(w_qkv_codes, w_qkv_scales, w13_codes, w13_scales, w_o_codes=None,
                            w_o_scales=None, w2_codes=None, w2_scales=None):
    return h3_block_weights_e4m3(*[_ptr(t) for t in (w_qkv_codes, w_qkv_scales, w13_codes,
                                                     w13_scales, w_o_codes, w_o_scales, w2_codes,
                                                     w2_scales)])


def h3_stack_forward_e4m3(dims: h3_dims, weights: Sequence[h3_block_weights],
                          w8: Sequence[h3_block_weights_e4m3], layout: Layout, tmod, x, B: int,
                          ws, ws_bytes: int, stream=None) -> None:
    if len(weights) != len(w8):
        raise ValueError("one set of 8-bit operands per block")
    n = len(weights)
    arr = (h3_block_weights * max(1, n))(*weights)
    arr8 = (h3_block_weights_e4m3 * max(1, n))(*w8)
    _check(lib().h3_stack_forward_e4m3(ctypes.byref(dims), arr, arr8, n, layout.handle, _ptr(tmod),
                                       _ptr(x), B, _ptr(ws), ws_bytes, _stream(stream)),
           "h3_stack_forward_e4m3")


def h3_out_residual_e4m3(dims: h3_dims, layout: Layout, B: int, o_codes, o_scales, w_codes,
                         w_scales, ada_table, tmod, x, stream=None) -> None:
    _check(lib().h3_out_residual_e4m3(ctypes.byref(dims), layout.handle, B, _ptr(o_codes),
                                      _ptr(o_scales), _ptr(w_codes), _ptr(w_scales),
                                      _ptr(ada_table), _ptr(tmod), _ptr(x), _stream(stream)),
           "h3_out_residual_e4m3")


def h3_ffn_down_residual_e4m3(dims: h3_dims, layout: Layout, B: int, g_codes, g_scales, w_codes,
                              w_scales, ada_table, tmod, x, stream=None) -> None:
    _check(lib().h3_ffn_down_residual_e4m3(ctypes.byref(dims), layout.handle, B, _ptr(g_codes),
                                           _ptr(g_scales), _ptr(w_codes), _ptr(w_scales),
                                           _ptr(ada_table), _ptr(tmod), _ptr(x), _stream(stream)),
           "h3_ffn_down_residual_e4m3")


def h3_workspace_size_e4m3(dims: h3_dims, B: int, S: int) -> int:
    return lib().h3_workspace_size_e4m3(ctypes.byref(dims), B, S)


def h3_block_forward_e4m3(dims: h3_dims, weights: h3_block_weights, w8: h3_block_weights_e4m3,
                          layout: Layout, tmod, x, B: int, ws, ws_bytes: int, stream=None) -> None:
    _check(lib().h3_block_forward_e4m3(ctypes.byref(dims), ctypes.byref(weights), ctypes.byref(w8),
                                       layout.handle, _ptr(tmod), _ptr(x), B, _ptr(ws), ws_bytes,
                                       _stream(stream)), "h3_block_forward_e4m3")
