"""Full-size workloads, in the launch configuration bench.py times, checked on
sampled (batch, head) pairs against the CPU oracle.

The whole batch is drawn on the device (as bench.py does); the sampled heads
are then overwritten with their seeded per-head inputs, which the oracle
rebuilds on its own.  Heads are independent problems, so a kernel that mixed
heads up, or went wrong at a tile or chunk boundary anywhere in the sequence,
shows up in the sampled heads.  The chunkwise reference runs with a
different chunk size (256) than the kernel (512), relying on the pinned
agreement of the oracle's forms.
"""
import math

import numpy as np
import pytest

import oracle
from linear_recurrent_sequence_scale_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
STATE_TOL = 1e-4


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_scale_b200 as ret
    ret.load_library()
    yield torch, ret
    assert ret.device_error() == 0


def _device_batch(torch, w, seed, N=None):
    n = w.N if N is None else N
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    s = 1.0 / math.sqrt(w.dk)
    q = (torch.randn((w.B, w.H, n, w.dk), device="cuda", generator=g) * s).bfloat16()
    k = (torch.randn((w.B, w.H, n, w.dk), device="cuda", generator=g) * s).bfloat16()
    v = (torch.randn((w.B, w.H, n, w.dv), device="cuda", generator=g) * s).bfloat16()
    return q, k, v


def _plant(q, k, v, w, heads, N=None):
    exact = {}
    for b, h in heads:
        hq, hk, hv = wl.make_head_inputs(w, b, h, N)
        q[b, h] = wl.to_torch(hq, "cuda")
        k[b, h] = wl.to_torch(hk, "cuda")
        v[b, h] = wl.to_torch(hv, "cuda")
        exact[(b, h)] = (hq.exact, hk.exact, hv.exact)
    return exact


def _gammas(torch, H):
    return torch.from_numpy(wl.msr_gammas(H)).cuda()


def test_l6p7b_8k_chunkwise_groupnorm(env):
    torch, ret = env
    w = wl.WORKLOADS["l6p7b_8k_bf16"]
    q, k, v = _device_batch(torch, w, 11)
    heads = [(0, 0), (3, 7), (7, 15)]
    exact = _plant(q, k, v, w, heads)
    g = _gammas(torch, w.H)
    o = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(ret.chunkwise_workspace_bytes(w.B, w.H, w.N, w.dk, w.dv, w.chunk,
                                                   torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    ret.chunkwise(q, k, v, g, w.chunk, gn_eps=w.gn_eps, out=o, workspace=ws)
    torch.cuda.synchronize()
    gam = wl.msr_gammas(w.H)
    for (b, h), (qe, ke, ve) in exact.items():
        o_ref, _ = oracle.chunkwise(qe[None, None], ke[None, None], ve[None, None],
                                    [float(gam[h])], 256)
        o_ref = oracle.group_norm(o_ref, w.gn_eps)
        err = oracle.rel_frobenius(wl.from_torch(o[b, h]), o_ref[0, 0])
        assert err <= TOL_BF16, ((b, h), err)


def test_long_64k_chunkwise_with_state(env):
    torch, ret = env
    w = wl.WORKLOADS["long_64k_bf16"]
    q, k, v = _device_batch(torch, w, 12)
    heads = [(0, 0), (0, 15)]
    exact = _plant(q, k, v, w, heads)
    g = _gammas(torch, w.H)
    o, s = ret.chunkwise(q, k, v, g, w.chunk, return_state=True)
    torch.cuda.synchronize()
    gam = wl.msr_gammas(w.H)
    for (b, h), (qe, ke, ve) in exact.items():
        o_ref, s_ref = oracle.chunkwise(qe[None, None], ke[None, None], ve[None, None],
                                        [float(gam[h])], 256)
        assert oracle.rel_frobenius(wl.from_torch(o[b, h]), o_ref[0, 0]) <= TOL_BF16
        assert oracle.rel_frobenius(wl.from_torch(s[b, h]), s_ref[0, 0]) <= STATE_TOL


def test_l1p3b_parallel_and_chunkwise(env):
    torch, ret = env
    w = wl.WORKLOADS["l1p3b_bf16"]
    q, k, v = _device_batch(torch, w, 13)
    heads = [(0, 0), (5, 7)]
    exact = _plant(q, k, v, w, heads)
    g = _gammas(torch, w.H)
    op = ret.parallel(q, k, v, g)
    oc = ret.chunkwise(q, k, v, g, w.chunk)
    torch.cuda.synchronize()
    gam = wl.msr_gammas(w.H)
    for (b, h), (qe, ke, ve) in exact.items():
        o_ref, _ = oracle.parallel(qe[None, None], ke[None, None], ve[None, None],
                                   [float(gam[h])])
        assert oracle.rel_frobenius(wl.from_torch(op[b, h]), o_ref[0, 0]) <= TOL_BF16
        assert oracle.rel_frobenius(wl.from_torch(oc[b, h]), o_ref[0, 0]) <= TOL_BF16


def test_decode_after_prefill(env):
    """8192-token prefill with the chunkwise form, then all 1024 decode steps
    (the bench's loop, 4 rotating states reduced to the one being checked)."""
    torch, ret = env
    w = wl.WORKLOADS["decode_6p7b"]
    q, k, v = _device_batch(torch, w, 14)
    heads = [(1, 0), (6, 15)]
    exact = _plant(q, k, v, w, heads)
    g = _gammas(torch, w.H)
    state = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    ret.chunkwise(q, k, v, g, w.chunk, state_out=state)
    del q, k, v
    gam = wl.msr_gammas(w.H)
    S = {}
    for (b, h), (qe, ke, ve) in exact.items():
        _, s_ref = oracle.chunkwise(qe[None, None], ke[None, None], ve[None, None],
                                    [float(gam[h])], 256)
        S[(b, h)] = s_ref
    torch.cuda.synchronize()
    for (b, h) in heads:
        assert oracle.rel_frobenius(wl.from_torch(state[b, h]), S[(b, h)][0, 0]) <= STATE_TOL
    outs = {bh: [] for bh in heads}
    gpu_outs = {bh: [] for bh in heads}
    T = wl.DECODE_STEPS
    for t in range(T):
        tq, tk, tv = wl.make_decode_token(w, t)
        o = ret.step(wl.to_torch(tq, "cuda"), wl.to_torch(tk, "cuda"), wl.to_torch(tv, "cuda"),
                     g, state)
        if t % 128 == 127 or t == 0:
            for (b, h) in heads:
                gpu_outs[(b, h)].append(wl.from_torch(o[b, h]))
        for (b, h) in heads:
            o_ref, S[(b, h)] = oracle.step(tq.exact[b:b + 1, h:h + 1], tk.exact[b:b + 1, h:h + 1],
                                           tv.exact[b:b + 1, h:h + 1], [float(gam[h])],
                                           S[(b, h)])
            if t % 128 == 127 or t == 0:
                outs[(b, h)].append(o_ref[0, 0])
    torch.cuda.synchronize()
    for (b, h) in heads:
        assert oracle.rel_frobenius(np.array(gpu_outs[(b, h)]), np.array(outs[(b, h)])) <= TOL_BF16
        assert oracle.rel_frobenius(wl.from_torch(state[b, h]), S[(b, h)][0, 0]) <= STATE_TOL
