"""CPU checks of the C-ABI library: it loads, exports every entry point the
header declares, and rejects bad arguments before touching the device."""

import ctypes
import os
import re
import subprocess
import sys

import pytest

from audio_generation_b200 import h3
from workloads import FULL_DIMS, TINY_DIMS, Dims

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    with open(os.path.join(ROOT, "include", "h3.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"^H3_API\s+[\w\s\*]+?\b(h3_\w+)\s*\(", src, re.M)))


def exported_symbols():
    out = subprocess.run(["nm", "-D", "--defined-only", h3.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    return {l.split()[-1] for l in out.splitlines() if " T " in l}


def test_library_exports_every_declared_entry_point():
    decl = header_functions()
    assert len(decl) >= 19
    exp = exported_symbols()
    missing = [n for n in decl if n not in exp]
    assert not missing, missing
    # and the binding wires every one of them
    assert set(decl) <= set(h3._SIGNATURES)


def test_only_declared_entry_points_are_exported():
    exp = {s for s in exported_symbols() if s.startswith("h3_")}
    assert exp == set(header_functions())


def test_status_strings_and_version():
    assert h3.h3_abi_version() >= 1
    for code, word in [(0, "ok"), (-1, "argument"), (-2, "shape"), (-3, "aligned"),
                       (-4, "layout"), (-5, "workspace"), (-6, "CUDA"), (-7, "timed out")]:
        assert word in h3.h3_status_string(code)
    assert "unknown" in h3.h3_status_string(42)


def _ws_expected(d, B, S):
    a = lambda n: (n + 255) // 256 * 256
    rows = B * S
    A = d.heads * d.head_dim
    one = a(rows * A * 2)
    return (a(rows * d.hidden * 2) + max(3 * one, a(rows * d.ffn * 2)) + a(rows * A * 2)
            + a(rows * d.hidden * 4))


@pytest.mark.parametrize("dims,B,S", [(FULL_DIMS, 1, 8192), (TINY_DIMS, 2, 256),
                                      (FULL_DIMS, 1, 0), (TINY_DIMS, 3, 333)])
def test_workspace_size(dims, B, S):
    assert h3.h3_workspace_size(h3.make_dims(dims), B, S) == _ws_expected(dims, B, S)


def _a256(n):
    return (n + 255) // 256 * 256


def _tmod_ws_expected(dims, n_t):
    base = _a256(n_t * (dims.freq_dim + dims.time_hidden + dims.time_embed_dim) * 4)
    if n_t < 65:
        return base
    stages = [(dims.freq_dim, dims.time_hidden), (dims.time_hidden, dims.time_embed_dim),
              (dims.time_embed_dim, 6 * dims.hidden)]
    return base + max(_a256(n_t * 6 * k * 2) + _a256(n * 6 * k * 2) for k, n in stages)


@pytest.mark.parametrize("dims", [TINY_DIMS, FULL_DIMS])
@pytest.mark.parametrize("n_t", [0, 1, 3, 64, 65, 126, 256, 8192])
def test_timestep_workspace_size(dims, n_t):
    """CUDA-core form below 65 timesteps (three fp32 activations); from 65 on
    also the bf16 split copies of the largest GEMM's two operands."""
    assert h3.h3_timestep_workspace_size(h3.make_dims(dims), n_t) == _tmod_ws_expected(dims, n_t)


@pytest.mark.parametrize("field,value", [("head_dim", 64), ("hidden", 500), ("heads", 5),
                                         ("ffn", 1000), ("rope_freq_dim", 8),
                                         ("freq_dim", 258), ("time_hidden", 5378),
                                         ("time_embed_dim", 2690)])
def test_unsupported_dims_are_rejected_on_the_host(field, value):
    kw = dict(FULL_DIMS.__dict__)
    kw[field] = value
    d = h3.make_dims(Dims(**kw))
    assert h3.h3_workspace_size(d, 1, 128) == 0
    out = ctypes.c_void_p()
    desc = h3.h3_layout_desc(S=0)
    assert h3.lib().h3_layout_prepare(ctypes.byref(d), ctypes.byref(desc), None,
                                      ctypes.byref(out)) == h3.H3_ERR_SHAPE
    assert out.value is None


def test_null_arguments_are_rejected_on_the_host():
    L = h3.lib()
    d = h3.make_dims(TINY_DIMS)
    out = ctypes.c_void_p()
    assert L.h3_layout_prepare(ctypes.byref(d), None, None, ctypes.byref(out)) == h3.H3_ERR_ARG
    desc = h3.h3_layout_desc(S=-1)
    assert L.h3_layout_prepare(ctypes.byref(d), ctypes.byref(desc), None,
                               ctypes.byref(out)) == h3.H3_ERR_ARG
    desc = h3.h3_layout_desc(S=10, n_t=10)  # null tags / positions
    assert L.h3_layout_prepare(ctypes.byref(d), ctypes.byref(desc), None,
                               ctypes.byref(out)) == h3.H3_ERR_ARG
    w = h3.h3_block_weights()
    assert L.h3_block_forward(ctypes.byref(d), ctypes.byref(w), None, None, None, 1, None, 0,
                              None) == h3.H3_ERR_ARG
    assert L.h3_pack_rows(None, 1, 8, None, None, None, None, None) == h3.H3_ERR_ARG
    assert L.h3_timestep_modulation(ctypes.byref(d), 4, None, None, None, None, None, None, 0,
                                    None) == h3.H3_ERR_ARG
    assert L.h3_timestep_modulation(ctypes.byref(d), 0, None, None, None, None, None, None, 0,
                                    None) == h3.H3_OK  # nothing to do
    assert L.h3_layout_error(None) == h3.H3_ERR_ARG


def test_binding_raises_typed_errors():
    with pytest.raises(h3.H3Error) as ei:
        h3._check(h3.H3_ERR_LAYOUT, "x")
    assert ei.value.status == h3.H3_ERR_LAYOUT


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(h3, "_lib", None)
    monkeypatch.setattr(h3, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        h3.lib()


def _imports(path):
    out = []
    for dp, _, fs in os.walk(path):
        for f in fs:
            if f.endswith(".py"):
                with open(os.path.join(dp, f)) as fh:
                    out += re.findall(r"^\s*(?:from|import)\s+([\w\.]+)", fh.read(), re.M)
    return out


def test_product_never_imports_the_oracle_and_vice_versa():
    assert not any(m.split(".")[0] == "oracle" for m in _imports(os.path.join(ROOT, "audio_generation_b200")))
    assert not any(m.split(".")[0] in ("audio_generation_b200",) for m in _imports(os.path.join(ROOT, "oracle")))
    assert not any(m.split(".")[0] in ("audio_generation_b200", "oracle")
                   for m in _imports(os.path.join(ROOT, "workloads")))


def test_row_limit_is_rejected_before_any_launch():
    """S above 524288 (128 x 4096 key tiles, the attention kernel's shared-memory
    key-tile list) is refused by h3_layout_prepare with H3_ERR_SHAPE; the check
    comes before any device call (the pointers here are not device memory)."""
    L = h3.lib()
    d = h3.make_dims(FULL_DIMS)
    out = ctypes.c_void_p()
    fake = 1 << 20  # never dereferenced: the shape check comes first
    for S, want in ((524289, h3.H3_ERR_SHAPE), (1 << 30, h3.H3_ERR_SHAPE)):
        desc = h3.h3_layout_desc(S=S, n_t=1, pos=fake, tags=fake, t_idx=fake)
        assert L.h3_layout_prepare(ctypes.byref(d), ctypes.byref(desc), None,
                                   ctypes.byref(out)) == want
        assert out.value is None


def test_noalloc_and_workspace_prologue_check_arguments_alike():
    """The no-allocation prologue returns the same status as the workspace form
    for the same bad input, including n_t = 0 (nothing to compute)."""
    L = h3.lib()
    bad_eps = dict(FULL_DIMS.__dict__, norm_eps=0.0)
    bad_shape = dict(FULL_DIMS.__dict__, hidden=500)
    for kw, want in ((bad_eps, h3.H3_ERR_ARG), (bad_shape, h3.H3_ERR_SHAPE)):
        d = h3.make_dims(Dims(**kw))
        for n_t in (0, 3):
            a = L.h3_timestep_modulation(ctypes.byref(d), n_t, None, None, None, None, None, None,
                                         0, None)
            b = L.h3_timestep_modulation_noalloc(ctypes.byref(d), n_t, None, None, None, None,
                                                 None, None)
            assert a == b == want, (kw, n_t, a, b)
    d = h3.make_dims(FULL_DIMS)
    assert L.h3_timestep_modulation(ctypes.byref(d), -1, None, None, None, None, None, None, 0,
                                    None) == h3.H3_ERR_ARG
    assert L.h3_timestep_modulation_noalloc(ctypes.byref(d), -1, None, None, None, None, None,
                                            None) == h3.H3_ERR_ARG
    assert L.h3_timestep_modulation_noalloc(ctypes.byref(d), 0, None, None, None, None, None,
                                            None) == h3.H3_OK


def test_new_entry_points_reject_bad_arguments_on_the_host():
    """The 8-bit steps and stack, and the sequence-parallel steps, return their
    status before any device work for missing or inconsistent arguments."""
    L = h3.lib()
    d = h3.make_dims(FULL_DIMS)
    fake = ctypes.c_void_p(256)  # never dereferenced: the checks fail first
    # 8-bit stack: no operands, negative block count
    w = h3.h3_block_weights()
    assert L.h3_stack_forward_e4m3(ctypes.byref(d), ctypes.byref(w), None, 1, fake, fake, fake, 1,
                                   fake, 1 << 30, None) == h3.H3_ERR_ARG
    assert L.h3_stack_forward_e4m3(ctypes.byref(d), None, None, -1, fake, fake, fake, 1, fake, 0,
                                   None) == h3.H3_ERR_ARG
    # 8-bit residual steps without a layout
    for fn in (L.h3_out_residual_e4m3, L.h3_ffn_down_residual_e4m3):
        assert fn(ctypes.byref(d), None, 1, fake, fake, fake, fake, fake, fake, fake,
                  None) == h3.H3_ERR_ARG
    # sequence-parallel steps: no layout, no peer table
    p = h3.make_peers(0, [256, 512], [256, 512], [256, 512], [256, 512])
    assert L.h3_qkv_rope_to_heads(ctypes.byref(d), None, fake, fake, fake, fake, ctypes.byref(p),
                                  None) == h3.H3_ERR_ARG
    assert L.h3_attention_to_rows(ctypes.byref(d), None, fake, fake, fake, None,
                                  None) == h3.H3_ERR_ARG
    assert h3.H3_MAX_RANKS == 8
