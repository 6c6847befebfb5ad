"""Child process of tests/test_gpu_timeout.py (not collected by pytest).

Loads the test-only fault-injection build of the library given on the command
line, runs the tiny block once with the GEMM producer's loads switched off (its
bounded waits must run out and the layout's error word must report
H3_ERR_TIMEOUT), then once normally, and prints the status codes and the
normal run's output as JSON.
"""

import ctypes
import json
import sys

import numpy as np
import torch


def main(lib_path: str) -> None:
    from audio_generation_b200 import h3
    h3.LIB_PATH = lib_path
    h3._lib = None
    lib = h3.lib()
    lib.h3_test_gemm_skip_loads.restype = ctypes.c_int
    lib.h3_test_gemm_skip_loads.argtypes = [ctypes.c_int]
    from tests.h3_testlib import DevLayout, DevWeights, dev_bf16, host_bits
    from tests.test_gpu_block import gpu_tmod
    from workloads import TINY_DIMS, activations, block_weights, config_layout, prologue_weights

    dims = TINY_DIMS
    L = config_layout(1)
    dl = DevLayout(dims, L)
    w = DevWeights(block_weights(dims, 1, 0))
    tmod = gpu_tmod(dims, L.timestep, prologue_weights(dims, 1))
    xb = activations(dims, 1, L.S)
    ws_b = h3.h3_workspace_size(dl.dims, 1, L.S)
    ws = torch.zeros(ws_b, dtype=torch.uint8, device="cuda")
    out = {}
    for name, skip in (("faulted", 1), ("normal", 0)):
        assert lib.h3_test_gemm_skip_loads(skip) == 0
        x = dev_bf16(xb)
        h3.h3_block_forward(dl.dims, w.c, dl.handle, tmod, x, 1, ws, ws_b)
        torch.cuda.synchronize()
        out[name] = h3.h3_layout_error(dl.handle)
        out[name + "_x"] = host_bits(x)[0].tolist() if name == "normal" else None
        out[name + "_unchanged"] = bool(np.array_equal(host_bits(x)[0], xb[0]))
    print("RESULT " + json.dumps(out))


if __name__ == "__main__":
    main(sys.argv[1])
