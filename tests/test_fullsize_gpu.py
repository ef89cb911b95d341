"""Full-size workloads, in the launch configuration bench.py times, checked
against the CPU oracle head by head.

Every (batch, head) pair of the 8k and 64k workloads and of the 1.3B-class
layer is drawn from its own seed (workloads.make_head_inputs), so the oracle
rebuilds each head on its own, in a pool of spawned processes.  Each head is
held to the tolerance over the whole head and over every 128-row tile, so a
kernel that mixed heads up, or went wrong at one tile, ring slot or chunk
boundary anywhere in the sequence, fails.  The chunkwise reference runs with
a different chunk size (256) than the kernel (512), relying on the pinned
agreement of the oracle's forms.
"""
import math
import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import pytest

import fullsize_workers as fw
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


@pytest.fixture(scope="module")
def pool():
    # spawned workers: safe after CUDA has been initialised in this process
    n = max(1, min(16, os.cpu_count() or 1))
    with ProcessPoolExecutor(n, mp_context=mp.get_context("spawn")) as ex:
        yield ex


def _bf16_bits(torch, x):
    """A bf16 device tensor's bit patterns as uint16 numpy (one copy to host)."""
    return x.view(torch.int16).cpu().numpy().view(np.uint16)


def _planted_batch(torch, pool, w, N=None):
    """The whole batch built head by head from the per-head seeds."""
    n = w.N if N is None else N
    q = torch.empty((w.B, w.H, n, w.dk), dtype=torch.bfloat16, device="cuda")
    k = torch.empty_like(q)
    v = torch.empty((w.B, w.H, n, w.dv), dtype=torch.bfloat16, device="cuda")
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    bits = pool.map(fw.head_bits, [w.name] * len(heads), *zip(*heads), [N] * len(heads))
    for (b, h), (qb, kb, vb) in zip(heads, bits):
        for dst, src in ((q, qb), (k, kb), (v, vb)):
            dst[b, h] = torch.from_numpy(src.view(np.int16)).view(torch.bfloat16).to("cuda")
    return q, k, v, heads


def _device_batch(torch, w, seed, N=None):
    n = w.N if N is None else N
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    s = 1.0 / math.sqrt(w.dk)
    q = (torch.randn((w.B, w.H, n, w.dk), device="cuda", generator=g) * s).bfloat16()
    k = (torch.randn((w.B, w.H, n, w.dk), device="cuda", generator=g) * s).bfloat16()
    v = (torch.randn((w.B, w.H, n, w.dv), device="cuda", generator=g) * s).bfloat16()
    return q, k, v


def _gammas(torch, H):
    return torch.from_numpy(wl.msr_gammas(H)).cuda()


def _assert_all(results, tol, what):
    bad = [(bh, r) for bh, r in results if not r[1] <= tol]
    assert not bad, f"{what}: {len(bad)} heads over {tol}, e.g. {bad[:3]}"


def test_l6p7b_8k_chunkwise_groupnorm_every_head(env, pool):
    torch, ret = env
    w = wl.WORKLOADS["l6p7b_8k_bf16"]
    q, k, v, heads = _planted_batch(torch, pool, w)
    g = _gammas(torch, w.H)
    o = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(ret.chunkwise_workspace_bytes(w.B, w.H, w.N, w.dk, w.dv, w.chunk,
                                                   torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    ret.chunkwise(q, k, v, g, w.chunk, gn_eps=w.gn_eps, out=o, workspace=ws)
    torch.cuda.synchronize()
    ob = _bf16_bits(torch, o)
    del q, k, v, ws
    res = pool.map(fw.check_chunkwise_head, [w.name] * len(heads), *zip(*heads),
                   [256] * len(heads), [ob[b, h] for b, h in heads])
    _assert_all([(bh, r[0]) for bh, r in zip(heads, res)], TOL_BF16, "8k output")


def test_long_64k_chunkwise_with_state_every_head(env, pool):
    torch, ret = env
    w = wl.WORKLOADS["long_64k_bf16"]
    q, k, v, heads = _planted_batch(torch, pool, w)
    g = _gammas(torch, w.H)
    o, s = ret.chunkwise(q, k, v, g, w.chunk, return_state=True)
    torch.cuda.synchronize()
    ob = _bf16_bits(torch, o)
    sn = s.cpu().numpy().astype(np.float64)
    del q, k, v, o
    res = list(pool.map(fw.check_chunkwise_head, [w.name] * len(heads), *zip(*heads),
                        [256] * len(heads), [ob[b, h] for b, h in heads],
                        [sn[b, h] for b, h in heads]))
    _assert_all([(bh, r[0]) for bh, r in zip(heads, res)], TOL_BF16, "64k output")
    _assert_all([(bh, r[1]) for bh, r in zip(heads, res)], STATE_TOL, "64k final state")


def test_l1p3b_parallel_and_chunkwise_every_head(env, pool):
    torch, ret = env
    w = wl.WORKLOADS["l1p3b_bf16"]
    q, k, v, heads = _planted_batch(torch, pool, w)
    g = _gammas(torch, w.H)
    op = ret.parallel(q, k, v, g)
    oc = ret.chunkwise(q, k, v, g, w.chunk)
    torch.cuda.synchronize()
    pb, cb = _bf16_bits(torch, op), _bf16_bits(torch, oc)
    res = list(pool.map(fw.check_parallel_head, [w.name] * len(heads), *zip(*heads),
                        [pb[b, h] for b, h in heads], [cb[b, h] for b, h in heads]))
    _assert_all([(bh, r[0]) for bh, r in zip(heads, res)], TOL_BF16, "parallel form")
    _assert_all([(bh, r[1]) for bh, r in zip(heads, res)], TOL_BF16, "chunkwise")


def test_decode_after_prefill(env, pool):
    """8192-token prefill with the chunkwise form, then all 1024 decode steps
    (the bench's loop on one state).  Sixteen heads, one per decay and spread
    over the batch, are rebuilt by the oracle from their own seeds, and every
    one of their 1024 outputs is checked, with the prefill and final states."""
    torch, ret = env
    w = wl.WORKLOADS["decode_6p7b"]
    q, k, v = _device_batch(torch, w, 14)
    heads = [(h % w.B, h) for h in range(w.H)]
    for (b, h), (qb, kb, vb) in zip(heads, pool.map(fw.head_bits, [w.name] * len(heads),
                                                     *zip(*heads))):
        for dst, src in ((q, qb), (k, kb), (v, vb)):
            dst[b, h] = torch.from_numpy(src.view(np.int16)).view(torch.bfloat16).to("cuda")
    g = _gammas(torch, w.H)
    state = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    ret.chunkwise(q, k, v, g, w.chunk, state_out=state)
    del q, k, v
    pre = state.cpu().numpy().astype(np.float64)
    T = wl.DECODE_STEPS
    outs = torch.empty((T, w.B, w.H, w.dv), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        tq, tk, tv = wl.make_decode_token(w, t)
        ret.step(wl.to_torch(tq, "cuda"), wl.to_torch(tk, "cuda"), wl.to_torch(tv, "cuda"),
                 g, state, out=outs[t])
    torch.cuda.synchronize()
    ob = _bf16_bits(torch, outs)
    fin = state.cpu().numpy().astype(np.float64)
    res = list(pool.map(fw.check_decode_head, [w.name] * len(heads), *zip(*heads),
                        [pre[b, h] for b, h in heads], [ob[:, b, h] for b, h in heads],
                        [fin[b, h] for b, h in heads]))
    _assert_all([(bh, r[0]) for bh, r in zip(heads, res)], STATE_TOL, "prefill state")
    _assert_all([(bh, r[1]) for bh, r in zip(heads, res)], TOL_BF16, "decode outputs")
    _assert_all([(bh, r[2]) for bh, r in zip(heads, res)], STATE_TOL, "final state")
