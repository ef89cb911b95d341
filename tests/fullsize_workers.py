"""Oracle work of the full-size GPU tests, one (batch, head) per call, run in a
pool of spawned processes (test infrastructure: imports the oracle and the
seeded input recipe only).

Each worker rebuilds its head's inputs from the seed, so only storage bits
and results cross process boundaries.
"""
from __future__ import annotations

import numpy as np

import oracle
from linear_recurrent_sequence_scale_b200 import workloads as wl
from parity_check import worst


def _one_thread():
    from threadpoolctl import threadpool_limits
    return threadpool_limits(1)


def head_bits(wname: str, b: int, h: int, N=None):
    """Storage arrays (bf16 bit patterns) of one head's q, k, v."""
    w = wl.WORKLOADS[wname]
    q, k, v = wl.make_head_inputs(w, b, h, N)
    return q.store, k.store, v.store


def check_chunkwise_head(wname: str, b: int, h: int, ref_chunk: int, o_bits, s=None, N=None):
    """Worst-block errors (where, value) of one head's output (and final
    state) against the oracle's chunkwise form run with `ref_chunk`."""
    with _one_thread():
        w = wl.WORKLOADS[wname]
        q, k, v = wl.make_head_inputs(w, b, h, N)
        gam = float(wl.msr_gammas(w.H)[h])
        o_ref, s_ref = oracle.chunkwise(q.exact[None, None], k.exact[None, None],
                                        v.exact[None, None], [gam], ref_chunk)
        if w.gn_eps >= 0:
            o_ref = oracle.group_norm(o_ref, w.gn_eps)
        eo = worst(wl.bf16_bits_to_f64(o_bits), o_ref[0, 0])
        es = worst(s, s_ref[0, 0]) if s is not None else None
        return eo, es


def check_parallel_head(wname: str, b: int, h: int, o_bits_par, o_bits_chunk):
    """Worst-block errors of one head's parallel-form and chunkwise outputs
    against the oracle's parallel form."""
    with _one_thread():
        w = wl.WORKLOADS[wname]
        q, k, v = wl.make_head_inputs(w, b, h)
        gam = float(wl.msr_gammas(w.H)[h])
        o_ref, _ = oracle.parallel(q.exact[None, None], k.exact[None, None], v.exact[None, None],
                                   [gam])
        return (worst(wl.bf16_bits_to_f64(o_bits_par), o_ref[0, 0]),
                worst(wl.bf16_bits_to_f64(o_bits_chunk), o_ref[0, 0]))


def check_decode_head(wname: str, b: int, h: int, prefill_state, o_steps, final_state):
    """Prefill state, every decode output and the final state of one head
    against the oracle: the chunkwise form over the head's prefill, then one
    recurrent step per decode token."""
    with _one_thread():
        w = wl.WORKLOADS[wname]
        q, k, v = wl.make_head_inputs(w, b, h)
        gam = [float(wl.msr_gammas(w.H)[h])]
        _, S = oracle.chunkwise(q.exact[None, None], k.exact[None, None], v.exact[None, None],
                                gam, 256)
        e_pre = worst(prefill_state, S[0, 0])
        outs = []
        for t in range(o_steps.shape[0]):
            tq, tk, tv = wl.make_decode_token(w, t)
            o, S = oracle.step(tq.exact[b:b + 1, h:h + 1], tk.exact[b:b + 1, h:h + 1],
                               tv.exact[b:b + 1, h:h + 1], gam, S)
            outs.append(o[0, 0])
        # decode outputs as [steps, d_v]: tiles of 128 consecutive steps
        e_out = worst(wl.bf16_bits_to_f64(o_steps), np.array(outs))
        e_fin = worst(final_state, S[0, 0])
        return e_pre, e_out, e_fin
