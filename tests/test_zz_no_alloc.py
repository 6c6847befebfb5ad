"""h3_timestep_modulation_noalloc: the timestep-modulation prologue for callers
that cannot allocate device memory (a serving loop whose device memory is
reserved up front by its own pool, or a latency-critical frame callback where
allocation is forbidden). Its scratch is a fixed array inside the library, so
it must give the same result as h3_timestep_modulation, call after call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

from audio_generation_b200 import h3
from workloads import FULL_DIMS, TINY_DIMS, prologue_weights

# Same tolerance as the existing entry point's own test (fp32 outputs).
TMOD_REL = 1e-4


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _with_workspace(d, n_t, t, pw, hidden):
    ws_b = h3.h3_timestep_workspace_size(d, n_t)
    ws = torch.empty(ws_b, dtype=torch.uint8, device="cuda")
    out = torch.empty((n_t, 6, hidden), dtype=torch.float32, device="cuda")
    h3.h3_timestep_modulation(d, n_t, _dev(t), _dev(pw.w_t1), _dev(pw.w_t2), _dev(pw.w_proj),
                              out, ws, ws_b)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("dims,cfg", [(FULL_DIMS, 2), (TINY_DIMS, 1)])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(dims, cfg):
    d = h3.make_dims(dims)
    pw = prologue_weights(dims, cfg)
    g = np.random.default_rng([cfg, 404])
    for n_t in (126 if dims is FULL_DIMS else 200, 3):  # large call, then a small one
        t = g.random(n_t).astype(np.float32)
        out = torch.full((n_t, 6, dims.hidden), float("nan"), dtype=torch.float32,
                         device="cuda")
        h3.h3_timestep_modulation_noalloc(d, n_t, _dev(t), _dev(pw.w_t1), _dev(pw.w_t2),
                                          _dev(pw.w_proj), out)
        ref = _with_workspace(d, n_t, t, pw, dims.hidden)
        torch.cuda.synchronize()
        a, b = out.double().cpu().numpy(), ref.double().cpu().numpy()
        assert np.all(np.isfinite(a))
        assert np.linalg.norm(a - b) / np.linalg.norm(b) < TMOD_REL


@pytest.mark.gpu
def test_noalloc_rejects_requests_beyond_its_scratch():
    d = h3.make_dims(FULL_DIMS)
    assert h3.h3_timestep_workspace_size(d, 127) > 4 << 20
    with pytest.raises(h3.H3Error) as ei:
        h3.h3_timestep_modulation_noalloc(d, 127, 16, 16, 16, 16, 16)
    assert ei.value.status == h3.H3_ERR_WORKSPACE
