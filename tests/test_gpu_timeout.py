"""A bounded in-kernel wait that runs out is reported, and the library keeps
working afterwards.

Every wait inside the library's kernels is bounded; one that runs out records
H3_ERR_TIMEOUT in the layout's error word, the kernel drains what it issued and
returns. To make a wait run out without faulting anything, this test builds a
test-only variant of the library (50 ms wait limit, and an entry point that
makes the GEMM producer issue no loads, so the barrier the MMA warp waits on is
never completed), runs the tiny block once with the loads switched off and
checks the reported status, then runs it normally and checks the result against
the product library's. The variant runs in a child process.
"""

import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from audio_generation_b200 import build as B
from tests.h3_testlib import DevLayout, DevWeights, dev_bf16, host_bits
from workloads import TINY_DIMS, activations, block_weights, config_layout, prologue_weights

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_next_call_succeeds(tmp_path):
    from audio_generation_b200 import h3
    from tests.test_gpu_block import gpu_tmod
    lib = B.build_fault_injection(str(tmp_path / "libh3_fault_injection.so"))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "fault_injection_child.py"),
                        lib], cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, PYTHONPATH=ROOT))
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT ")]
    assert r.returncode == 0 and line, r.stderr[-3000:]
    res = json.loads(line[0][len("RESULT "):])
    assert res["faulted"] == h3.H3_ERR_TIMEOUT
    assert res["faulted_unchanged"]  # no GEMM epilogue ran: x was not written
    assert res["normal"] == h3.H3_OK
    # the product library on the same inputs gives the same bits
    dims = TINY_DIMS
    L = config_layout(1)
    dl = DevLayout(dims, L)
    w = DevWeights(block_weights(dims, 1, 0))
    tmod = gpu_tmod(dims, L.timestep, prologue_weights(dims, 1))
    xb = activations(dims, 1, L.S)
    x = dev_bf16(xb)
    ws_b = h3.h3_workspace_size(dl.dims, 1, L.S)
    ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
    h3.h3_block_forward(dl.dims, w.c, dl.handle, tmod, x, 1, ws, ws_b)
    torch.cuda.synchronize()
    assert h3.h3_layout_error(dl.handle) == h3.H3_OK
    np.testing.assert_array_equal(np.array(res["normal_x"], np.uint16), host_bits(x)[0])
    assert not np.array_equal(host_bits(x)[0], xb[0])
