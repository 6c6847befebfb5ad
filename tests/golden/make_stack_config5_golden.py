"""Writes tests/golden/stack_config5_golden.npz: the float64 oracle's output of
the full-width 50-block stack on the 16384-row padded layout, at sampled rows.

Source: "MiniMaxH3Transformer3DModel" (diffusers v0.43.0 docs), constructor
parameter ``num_layers`` (50 blocks) and the overview (one stack of blocks over
one packed 1-D sequence; padding rows in their own attention document).

This script calls only ``oracle/`` (the arithmetic) and ``workloads/`` (the
seeded inputs). Every block is ``oracle.h3_oracle.block_forward`` as it stands;
the one change is that its attention runs on pieces (a group of heads, a chunk
of query rows) in a thread pool. Heads are independent in the definition (each
head's softmax and value sum involve that head's q, k and v only), and so are
query rows (each row's softmax runs over that row's scores), so the pieces,
put back in place, give the same result.
``tests/test_golden_stack_script.py`` checks that on small cases.

With ``--emulate`` it writes tests/golden/stack_config5_golden_bf16.npz: the
same stack with the oracle's bf16 storage emulation at the block's operand
storage points (h, q, k, v, P, o, h2, g) and the residual stream in fp32, as the
stack holds it on the device: the result of an exactly rounded bf16 stack, which
separates the rounding every bf16 implementation carries from the device's own.

The stored file holds the sampled row indices, the rows' bf16 input and
float64 output (stored as float32), and a SHA-256 digest over every input the
stack reads (layout, timesteps, activations, the prologue weights and all 50
blocks' weights), so the GPU test can prove it regenerated the same inputs.

Run from the repository root (a few hours on 8 host cores, ~20 GB RAM):
    python -m tests.golden.make_stack_config5_golden
"""

from __future__ import annotations

import argparse
import hashlib
import os
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np
from threadpoolctl import threadpool_limits

from oracle import h3_oracle as O
from workloads import FULL_DIMS, activations, block_weights, config_layout, prologue_weights

HERE = os.path.dirname(os.path.abspath(__file__))
OUT = os.path.join(HERE, "stack_config5_golden.npz")
OUT_BF16 = os.path.join(HERE, "stack_config5_golden_bf16.npz")
N_BLOCKS = 50


def sample_rows(L, n: int = 64, seed: int = 5) -> np.ndarray:
    """Rows next to every padding run (both sides), rows of the two mixed
    128-row tiles, tile boundaries, some padding rows, then random rows of
    each modality until ``n`` rows are chosen."""
    S = L.S
    pad = L.tags < 0
    rows = {0, 127, 128, S // 2 - 1, S // 2, S - 1}
    edges = np.nonzero(np.diff(pad.astype(np.int8)))[0]
    for e in edges:
        rows.update({int(e), int(e) + 1})
    tiles = np.arange(S) // 128
    for t in np.unique(tiles[pad]):
        seg = np.nonzero(tiles == t)[0]
        if pad[seg].any() and not pad[seg].all():
            v = seg[~pad[seg]]
            rows.update({int(v[0]), int(v[len(v) // 2]), int(v[-1])})
    g = np.random.default_rng([S, seed])
    for tag in (1, 0, 2):
        cand = np.nonzero(L.tags == tag)[0]
        rows.update(int(r) for r in g.choice(cand, size=4, replace=False))
    valid = np.nonzero(~pad)[0]
    while len(rows) < n:
        rows.add(int(g.choice(valid)))
    return np.array(sorted(rows), np.int64)


def head_parallel_attention(workers: int, q_chunk: int = 128):
    """``oracle.h3_oracle.attention`` computed on (head group, query chunk) pieces
    in a thread pool. Heads are independent, and so are query rows (each row's
    softmax and value sum involve that row's scores only), so the pieces,
    reassembled, are the oracle's result. Small query chunks keep each piece's
    score arrays in cache."""
    base = O.attention

    def attention(q, doc_q, k, v, doc_k, emulate=False):
        n, NH, D = q.shape
        gs = max(1, min(NH, 8))
        groups = [list(range(i, min(NH, i + gs))) for i in range(0, NH, gs)]
        kc = [np.ascontiguousarray(k[:, hs]) for hs in groups]
        vc = [np.ascontiguousarray(v[:, hs]) for hs in groups]
        tasks = [(gi, r0) for gi in range(len(groups)) for r0 in range(0, n, q_chunk)]
        o = np.empty((n, NH, D), np.float64)

        def run(task):
            gi, r0 = task
            hs, r1 = groups[gi], min(n, r0 + q_chunk)
            part = base(np.ascontiguousarray(q[r0:r1, hs]), doc_q[r0:r1], kc[gi], vc[gi], doc_k,
                        emulate)
            o[r0:r1, hs] = part.reshape(r1 - r0, len(hs), D)

        with threadpool_limits(limits=1, user_api="blas"), \
                ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(run, tasks))
        return o.reshape(n, NH * D)

    return attention


class InputDigest:
    """SHA-256 over the stack's inputs, in a fixed order."""

    def __init__(self):
        self.h = hashlib.sha256()

    def add(self, *arrays) -> None:
        for a in arrays:
            a = np.ascontiguousarray(a)
            self.h.update(str(a.dtype).encode() + str(a.shape).encode())
            self.h.update(a.tobytes())

    def add_block(self, w) -> None:
        self.add(w.w_qkv, w.q_norm, w.k_norm, w.w_o, w.w13, w.w2, w.ada_table)

    def hexdigest(self) -> str:
        return self.h.hexdigest()


def layout_digest(d: InputDigest, L) -> None:
    d.add(L.tags, L.pos, L.t_idx, L.timestep, L.video_idx, L.audio_idx, L.text_idx)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workers", type=int, default=len(os.sched_getaffinity(0)),
                    help="attention pieces run at once")
    ap.add_argument("--blocks", type=int, default=N_BLOCKS)
    ap.add_argument("--out", default=None)
    ap.add_argument("--emulate", action="store_true",
                    help="bf16 at the device's operand storage points, fp32 residual stream")
    args = ap.parse_args()
    out = args.out or (OUT_BF16 if args.emulate else OUT)

    dims = FULL_DIMS
    L = config_layout(5)
    pw = prologue_weights(dims, 5)
    xb = activations(dims, 5, L.S)
    tmod = O.timestep_modulation(L.timestep, pw.w_t1, pw.w_t2, pw.w_proj, dims.freq_dim,
                                 dims.hidden)
    rows = sample_rows(L)
    dig = InputDigest()
    layout_digest(dig, L)
    dig.add(xb)
    dig.add(pw.w_t1, pw.w_t2, pw.w_proj)

    O.attention = head_parallel_attention(args.workers)
    y = O.bf16_to_f64(xb[0])[None]
    t0 = time.time()
    for i in range(args.blocks):
        w = block_weights(dims, 5, i)
        dig.add_block(w)
        y = O.block_forward(y, w, L, tmod, dims, emulate=args.emulate, stream_f32=args.emulate)
        print(f"block {i + 1}/{args.blocks}: {time.time() - t0:.0f} s", flush=True)
    np.savez(out, rows=rows, x_in_bits=xb[0, rows], x_out=y[0, rows].astype(np.float32),
             n_blocks=np.int64(args.blocks), input_sha256=np.array(dig.hexdigest()),
             seconds=np.float64(time.time() - t0), cores=np.int64(len(os.sched_getaffinity(0))))
    print("wrote", out, "digest", dig.hexdigest())


if __name__ == "__main__":
    main()
