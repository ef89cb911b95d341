"""ret_chunkwise_noalloc, the chunkwise entry point for callers that cannot
allocate device memory (a plugin whose host runtime owns all device memory,
or a loop that must not call cudaMalloc).  It takes its scratch from a fixed
array inside the library, so its results must equal those of ret_chunkwise
given a caller-allocated workspace, call after call, whatever the previous
call left in the shared array, and match the CPU oracle on their own (so a
fault shared by the two entry points does not pass unseen).

This file is collected last on purpose: a run that stops at the first
failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest

import oracle
from linear_recurrent_sequence_scale_b200 import workloads as wl
from parity_check import worst_rel

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}
STATE_TOL = 1e-4

# dtype, B, H, N, dk, dv, chunk, gn_eps, state_in
CASES = [
    ("bf16", 1, 3, 1000, 256, 512, 512, 1e-5, True),
    ("bf16", 2, 2, 700, 128, 128, 128, None, False),
    ("f32", 1, 2, 301, 64, 64, 37, None, True),
]


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_scale_b200 as ret
    lib = ret.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for dt, B, H, N, dk, dv, C, gn, with_s0 in CASES:
        inp = wl.make_inputs(B, H, N, dk, dv, dt, seed=500 + N, with_state=with_s0)
        q, k, v = (wl.to_torch(inp[x], "cuda") for x in ("q", "k", "v"))
        g = torch.from_numpy(inp["gammas"]).cuda()
        s0 = wl.to_torch(inp["state"], "cuda") if with_s0 else None
        o_ref, s_ref = ret.chunkwise(q, k, v, g, C, state_in=s0, return_state=True, gn_eps=gn)
        o = torch.empty_like(o_ref)
        s = torch.empty_like(s_ref)
        code = ret.RET_BF16 if dt == "bf16" else ret.RET_F32
        st = lib.ret_chunkwise_noalloc(_p(q), _p(k), _p(v), _p(g), C, _p(s0), _p(s), _p(o),
                                       B, H, N, dk, dv, code, -1.0 if gn is None else gn, stream)
        assert st == ret.RET_OK, ret.status_string(st)
        torch.cuda.synchronize()
        assert worst_rel(wl.from_torch(o), wl.from_torch(o_ref)) <= TOL[dt]
        assert worst_rel(wl.from_torch(s), wl.from_torch(s_ref)) <= STATE_TOL
        # and against the oracle directly
        o_or, s_or = oracle.chunkwise(inp["q"].exact, inp["k"].exact, inp["v"].exact,
                                      inp["gammas"], C, inp["state"].exact if with_s0 else None)
        if gn is not None:
            o_or = oracle.group_norm(o_or, gn)
        assert worst_rel(wl.from_torch(o), o_or) <= TOL[dt]
        assert worst_rel(wl.from_torch(s), s_or) <= STATE_TOL
        assert ret.device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_scale_b200 as ret
    lib = ret.load_library()
    B, H, N, dk, dv, C = 8, 16, 8192, 256, 512, 512   # needs 512 MiB of scratch
    assert lib.ret_chunkwise_workspace(B, H, N, dk, dv, C, ret.RET_BF16) > 64 << 20
    fake = ctypes.c_void_p(0x10000)   # never dereferenced: rejected before any launch
    st = lib.ret_chunkwise_noalloc(fake, fake, fake, fake, C, None, None, fake, B, H, N, dk, dv,
                                   ret.RET_BF16, -1.0, None)
    assert st == ret.RET_EWORKSPACE
