"""Sequence parallelism on CPU: the driver's exchange over torch.distributed
(gloo, 2 and 3 ranks) with the oracle standing in for the CUDA steps.  Each
rank's span output and the end state of the whole sequence must equal the
oracle run over the unsplit sequence; a wrong span combination or a wrong
exchange order fails it."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from linear_recurrent_sequence_scale_b200 import seqpar
from linear_recurrent_sequence_scale_b200 import workloads as wl


class OracleOps:
    """The driver's three steps in float64 on the CPU oracle."""

    def local_end_state(self, q, k, v, gammas, chunk):
        _, s = oracle.chunkwise(q.numpy(), k.numpy(), v.numpy(), gammas.numpy(), chunk)
        return torch.from_numpy(s)

    def rotate(self, x, theta, pos0):
        return torch.from_numpy(oracle.rotate(x.numpy(), theta.numpy(), pos0))

    def combine(self, locals_, spans, r, gammas, state0):
        # the chunk recurrence at span granularity: S <- gamma^N S + S_local
        g = gammas.numpy()[None, :, None, None]
        s = np.zeros(locals_.shape[1:]) if state0 is None else state0.numpy().copy()
        for i in range(r):
            s = g ** spans[i] * s + locals_[i].numpy()
        return torch.from_numpy(s)

    def chunkwise(self, q, k, v, gammas, chunk, state_in, gn_eps, gate, return_state):
        o, _ = oracle.chunkwise(q.numpy(), k.numpy(), v.numpy(), gammas.numpy(), chunk,
                                state_in.numpy())
        if gn_eps is not None:
            o = oracle.group_norm(o, gn_eps)
        if gate is not None:
            o = oracle.gated(o, gate.numpy())
        return torch.from_numpy(o)


SPANS = {2: [67, 83], 3: [50, 13, 87]}


def _inputs():
    N = 150
    inp = wl.make_inputs(1, 3, N, 8, 6, "f32", seed=81, with_state=True,
                         gammas=[0.9, 0.99, 0.5])
    gate = np.random.default_rng(82).standard_normal((1, 3, N, 6))
    return inp, gate


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out, rotated=False):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp, gate = _inputs()
        spans = SPANS[world]
        a = sum(spans[:rank])
        b = a + spans[rank]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, :, a:b]))
        o, s = seqpar.chunkwise_sequence_parallel(
            t(inp["q"].exact), t(inp["k"].exact), t(inp["v"].exact),
            torch.from_numpy(inp["gammas"].astype(np.float64)), 16,
            state0=torch.from_numpy(inp["state"].exact), gn_eps=1e-5, gate=t(gate),
            return_state=True, ops=OracleOps(),
            theta=torch.from_numpy(_theta()) if rotated else None, pos0=POS0)
        out[rank] = (a, b, o.numpy(), s.numpy())
    finally:
        dist.destroy_process_group()


POS0 = 1000


def _theta():
    return wl.rotation_angles(8, seed=4).astype(np.float64)


@pytest.mark.parametrize("world,rotated", [(2, False), (3, False), (2, True), (3, True)])
def test_spans_over_gloo_match_the_unsplit_sequence(world, rotated):
    """With rotated, q and k of each span are rotated from the span's start
    position (POS0 + the tokens before it) and must match the unsplit
    sequence rotated from POS0."""
    assert sum(SPANS[world]) == 150
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out, rotated))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    inp, gate = _inputs()
    q, k = inp["q"].exact, inp["k"].exact
    if rotated:
        q, k = oracle.rotate(q, _theta(), POS0), oracle.rotate(k, _theta(), POS0)
    o_ref, s_ref = oracle.chunkwise(q, k, inp["v"].exact, inp["gammas"], 16, inp["state"].exact)
    o_ref = oracle.gated(oracle.group_norm(o_ref, 1e-5), gate)
    for r in range(world):
        a, b, o, s = out[r]
        assert oracle.rel_frobenius(o, o_ref[:, :, a:b]) < 1e-12
        assert oracle.rel_frobenius(s, s_ref) < 1e-12
