"""Sequence-parallel chunkwise retention: one long sequence split into
contiguous spans, one per rank (GPU), in rank order.

"RetNet - Retentive Network - A Successor to Transformer for LLMs", Key
Equations, Chunkwise Recurrent: the state passed from chunk to chunk obeys
R_i = gamma^L R_{i-1} + (the chunk's own part), so the same holds between
spans.  Each rank
  1. computes its span's end state from a zero state (the states phase of
     the chunkwise form, on its GPU),
  2. exchanges it with all ranks (one all-gather of B*H*dk*dv floats per
     rank; over NCCL the states travel over NVLink), together with the span
     lengths,
  3. combines the gathered states into the state entering its span
     (ret_state_combine, on its GPU),
  4. runs the chunkwise form over its span from that state (outputs, fused
     GroupNorm / gate, and its end state).
Step 4 recomputes the chunk states of the span with the incoming state, so the
states phase runs twice; the exchange is the only communication.

With the xPos rotation (same page, core components, item 3: a complex
rotation of Q and K by position), q and k of a span are rotated from the
span's own start position before step 1, so the span lengths are gathered
first; every rank then holds the rows the unsplit sequence would have.

The steps are exposed separately (`local_end_state`, `span_output`) so that
callers can run them across processes themselves; `chunkwise_sequence_parallel`
runs all four with torch.distributed.  The arithmetic of every step is the
CUDA library's (`CudaOps`); another ops object with the same three methods can
stand in for it.
"""
from __future__ import annotations


class CudaOps:
    """The three steps on the CUDA library."""

    def local_end_state(self, q, k, v, gammas, chunk):
        import torch

        from . import chunkwise_states, chunkwise_workspace_bytes
        B, H, N, dk = k.shape
        dv = v.shape[-1]
        ws = torch.empty(chunkwise_workspace_bytes(B, H, N, dk, dv, chunk, k.dtype),
                         dtype=torch.uint8, device=k.device)
        s = torch.empty((B, H, dk, dv), dtype=torch.float32, device=k.device)
        chunkwise_states(k, v, gammas, chunk, ws, state_out=s)
        return s

    def rotate(self, x, theta, pos0):
        from . import rotate
        return rotate(x, theta, pos0)

    def combine(self, locals_, spans, r, gammas, state0):
        from . import state_combine
        return state_combine(locals_, spans, r, gammas, state0)

    def chunkwise(self, q, k, v, gammas, chunk, state_in, gn_eps, gate, return_state):
        from . import chunkwise
        return chunkwise(q, k, v, gammas, chunk, state_in=state_in, return_state=return_state,
                         gn_eps=gn_eps, gate=gate)


def local_end_state(q, k, v, gammas, chunk, ops=None):
    """Step 1: this span's end state from a zero state, [B,H,dk,dv] float32."""
    return (ops or CudaOps()).local_end_state(q, k, v, gammas, chunk)


def span_output(q, k, v, gammas, chunk, locals_, spans, rank, state0=None, gn_eps=None,
                gate=None, return_state=False, ops=None):
    """Steps 3 and 4 for span `rank`, given the end states of all spans
    (`locals_`, [R,B,H,dk,dv]) and their lengths.  Returns o, or
    (o, end state of the whole sequence) when return_state is set."""
    ops = ops or CudaOps()
    s_in = ops.combine(locals_, spans, rank, gammas, state0)
    o = ops.chunkwise(q, k, v, gammas, chunk, s_in, gn_eps, gate, False)
    if not return_state:
        return o
    return o, ops.combine(locals_, spans, len(spans), gammas, state0)


def chunkwise_sequence_parallel(q, k, v, gammas, chunk, group=None, state0=None, gn_eps=None,
                                gate=None, return_state=False, ops=None, theta=None, pos0=0):
    """All four steps over the ranks of `group` (torch.distributed): q, k, v
    (and gate) are this rank's span, [B,H,N_rank,d]; every rank passes the
    same gammas, chunk, state0 (the state entering the whole sequence, or
    None) and options.  With theta ([d_k/2] angles) q and k are rotated
    first, the first token of the whole sequence sitting at position pos0.
    Returns this span's o, and with return_state the end state of the whole
    sequence (the same on every rank)."""
    import torch
    import torch.distributed as dist

    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    n = torch.tensor([q.shape[2]], dtype=torch.int64, device=q.device)
    ns = [torch.empty_like(n) for _ in range(world)]
    dist.all_gather(ns, n, group=group)
    spans = [int(x.item()) for x in ns]
    if theta is not None:
        start = pos0 + sum(spans[:rank])
        q = ops.rotate(q, theta, start)
        k = ops.rotate(k, theta, start)
    s_loc = ops.local_end_state(q, k, v, gammas, chunk).contiguous()
    gathered = [torch.empty_like(s_loc) for _ in range(world)]
    dist.all_gather(gathered, s_loc, group=group)
    locals_ = torch.stack(gathered)
    return span_output(q, k, v, gammas, chunk, locals_, spans, rank, state0=state0,
                       gn_eps=gn_eps, gate=gate, return_state=return_state, ops=ops)
