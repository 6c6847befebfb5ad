"""The checker that smoke() applies to the GPU block output, run on CPU
against oracle outputs: it accepts the oracle's own bf16-storage emulation and
rejects a block that leaves x unchanged or that drops its FFN branch."""

import numpy as np
import pytest

import __graft_entry__ as G
from oracle import h3_oracle as O
from workloads import TINY_DIMS, activations, block_weights, config_layout, prologue_weights


@pytest.fixture(scope="module")
def case():
    dims = TINY_DIMS
    L = config_layout(1)
    w = block_weights(dims, 1, 0)
    pw = prologue_weights(dims, 1)
    x0 = O.bf16_to_f64(activations(dims, 1, L.S)[0])
    tm = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim,
                               dims.hidden)
    ref = O.block_forward(x0[None], w, L, tm, dims)[0]
    emu = O.block_forward(x0[None], w, L, tm, dims, emulate=True)[0]
    return dims, L, w, tm, x0, ref, emu


def test_checker_accepts_the_emulated_block(case):
    dims, L, w, tm, x0, ref, emu = case
    G.check_block_output(emu, x0, ref, emu, L.tags < 0)


def test_checker_rejects_an_identity_block(case):
    dims, L, w, tm, x0, ref, emu = case
    # x_out alone would pass: the identity is within the x_out tolerance here
    assert np.linalg.norm(x0 - ref) / np.linalg.norm(ref) < 1e-2
    with pytest.raises(RuntimeError, match="update"):
        G.check_block_output(x0.copy(), x0, ref, emu, L.tags < 0)


def test_checker_rejects_a_block_without_its_ffn_branch(case):
    dims, L, w, tm, x0, ref, emu = case
    tm0 = tm.copy()
    tm0[:, 5] = 0.0
    w0 = block_weights(dims, 1, 0)
    w0.ada_table = w0.ada_table.copy()
    w0.ada_table[:, 5] = 0.0  # gate2 = 0: attention branch only
    half = O.block_forward(x0[None], w0, L, tm0, dims, emulate=True)[0]
    with pytest.raises(RuntimeError, match="update"):
        G.check_block_output(half, x0, ref, emu, L.tags < 0)
