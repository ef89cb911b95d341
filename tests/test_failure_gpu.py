"""Failure detection without a GPU fault: a bounded device wait that runs out
reports its site code through ret_device_error(), and the context stays
usable for the next call."""
import numpy as np
import pytest

import oracle
from linear_recurrent_sequence_scale_b200 import workloads as wl
from parity_check import worst_rel

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_scale_b200 as ret
    lib = ret.load_library()
    assert ret.device_error() == 0
    stream = torch.cuda.current_stream().cuda_stream
    import ctypes
    assert lib.ret_selftest_bounded_wait(50, ctypes.c_void_p(stream)) == ret.RET_OK
    torch.cuda.synchronize()
    assert ret.device_error() == 901
    assert ret.device_error() == 0          # read and cleared
    # the context still works: a normal call matches the oracle
    inp = wl.make_inputs(1, 2, 200, 64, 64, "bf16", seed=5)
    q, k, v = (wl.to_torch(inp[n], "cuda") for n in ("q", "k", "v"))
    g = torch.from_numpy(inp["gammas"]).cuda()
    o = ret.chunkwise(q, k, v, g, 128)
    torch.cuda.synchronize()
    o_ref, _ = oracle.chunkwise(inp["q"].exact, inp["k"].exact, inp["v"].exact, inp["gammas"], 128)
    assert worst_rel(wl.from_torch(o), o_ref) <= 2e-2
    assert ret.device_error() == 0
