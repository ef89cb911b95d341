"""CPU oracle for multi-scale retention, float64 numpy.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg use it.  It shares no code with the CUDA path;
its inputs come from the seeded generators in
linear_recurrent_sequence_scale_b200/workloads.py, which hold none of the
method's arithmetic.

Pages cited (by title; the web pages on retention this build follows):
  [RetNet blog]  "RetNet - Retentive Network - A Successor to Transformer for
                 LLMs" (irregular6612.github.io), sections Methods,
                 core components, Key Equations and the glossary.
  [glossary]     "RetNet" entry of the jisaku.com glossary (efficient-arch-
                 retnet): definition of D, the three modes, FAQ Q2.
  [Spiral.AI]    "RetNet入門" (Spiral.AI Tech Blog, news.ainew.jp digest),
                 sections Multi-Scale Retention (MSR) and the one on other
                 non-Transformer architectures (LEX Transformer, xPos).
  [Medium]       "What Is RetNet ? could it challenge the dominance of the
                 Transformer ?" (Medium, Publicis Sapient), section "How is
                 this dual representation achieved?".

Shapes: q, k [B,H,N,dk]; v [B,H,N,dv]; gammas [H]; state [B,H,dk,dv].
Every function returns float64 arrays.

Readings taken where the pages leave a step open (each one is also listed
in the design notes):
  * The chunk state printed on the RetNet blog (core components, item 1,
    R_i = K_i^T V_i + gamma^chunk R_{i-1}) leaves out the decay inside the
    chunk; it equals the recurrence only for gamma = 1.  The oracle uses
    R_i = gamma^L R_{i-1} + K_[i]^T (V_[i] * zeta), zeta_j = gamma^(L-1-j),
    which is what the recurrent form gives when it is summed over a chunk.
  * xi in the chunkwise equation (Key Equations) is not defined on the page;
    the oracle uses xi_j = gamma^(j+1) for in-chunk position j (0-based),
    since the recurrence updates S_n before reading it (o_n = Q_n S_n).
  * D is inclusive on the diagonal (n >= m), so D_nn = gamma^0 = 1, and
    0^0 = 1 when gamma = 0.
  * GroupNorm: one group is one head's d_v outputs at one token; biased
    variance; eps inside the square root; no affine parameters.  Parity
    unpinned beyond its invariants: the pages name GroupNorm per head but
    fix none of these conventions.
  * No scaling or normalising factors are applied to QK^T, D or their
    product (the Medium page mentions three such factors without formulas).
  * Gate: the block's "swish gating" is read as swish(G) (.) Y with the gate
    G supplied by the caller, swish(x) = x sigmoid(x).
  * xPos rotation: the pages call it a complex rotation of Q and K that
    carries relative position, and give no formula.  Read as: channels
    (2c, 2c+1) of a row are the real and imaginary parts of z_c, and the row
    at position n is multiplied by e^{i n theta_c}; the angles theta are
    supplied by the caller (the pages give no values); no length scaling
    (the decay gamma already plays that role in retention).
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def decay_mask(gamma: float, n: int) -> np.ndarray:
    """D[n, m] = gamma^(n-m) for n >= m, else 0 ([RetNet blog] Key Equations,
    Parallel Form; [glossary] definition of D)."""
    idx = np.arange(n)
    d = idx[:, None] - idx[None, :]
    return np.where(d >= 0, np.power(float(gamma), np.maximum(d, 0)), 0.0)


def step(q, k, v, gammas, state):
    """One recurrent step for every (batch, head) pair
    ([RetNet blog] Key Equations, Recurrent Form):
        S_n = gamma * S_{n-1} + k_n^T v_n,   o_n = q_n S_n.
    q, k: [B,H,dk]; v: [B,H,dv]; state: [B,H,dk,dv].  Returns (o, new state).
    """
    q, k, v, S = _f64(q), _f64(k), _f64(v), _f64(state)
    g = _f64(gammas)[None, :, None, None]
    S = g * S + k[..., :, None] * v[..., None, :]
    o = np.einsum("bhk,bhkv->bhv", q, S)
    return o, S


def recurrent(q, k, v, gammas, state_in=None):
    """Recurrent form over a whole sequence: repeated `step`, token by token.
    Returns (o [B,H,N,dv], final state [B,H,dk,dv])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if state_in is None else _f64(state_in).copy()
    o = np.zeros((B, H, N, dv))
    for n in range(N):
        o[:, :, n], S = step(q[:, :, n], k[:, :, n], v[:, :, n], gammas, S)
    return o, S


def parallel(q, k, v, gammas, state_in=None):
    """Parallel form ([RetNet blog] Key Equations, Parallel Form;
    [glossary] parallel mode): o = (Q K^T * D) V.

    With an initial state S_0 the recurrence adds gamma^(n+1) q_n S_0 to row n,
    and the final state is sum_m gamma^(N-1-m) k_m^T v_m + gamma^N S_0, the
    recurrence unrolled over the sequence.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, N, dv))
    S = np.zeros((B, H, dk, dv))
    n = np.arange(N)
    for h in range(H):
        g = float(gammas[h])
        D = decay_mask(g, N)
        for b in range(B):
            Q, K, V = q[b, h], k[b, h], v[b, h]
            o[b, h] = ((Q @ K.T) * D) @ V
            zeta = np.power(g, N - 1 - n)
            S[b, h] = K.T @ (V * zeta[:, None])
            if state_in is not None:
                S0 = _f64(state_in[b, h])
                xi = np.power(g, n + 1)
                o[b, h] += (Q * xi[:, None]) @ S0
                S[b, h] += g ** N * S0
    return o, S


def chunkwise(q, k, v, gammas, chunk: int, state_in=None):
    """Chunkwise-recurrent form ([RetNet blog] Key Equations, Chunkwise
    Recurrent; [glossary] chunkwise mode): inside chunk i (tokens
    [iC, iC+L), L = C except for a shorter last chunk)
        o_[i] = (Q_[i] K_[i]^T * D_L) V_[i] + (Q_[i] * xi) R_{i-1},
        xi_j  = gamma^(j+1),
        R_i   = gamma^L R_{i-1} + K_[i]^T (V_[i] * zeta),  zeta_j = gamma^(L-1-j),
    with R_{-1} the initial state (zero if none).  Returns (o, R_last).
    """
    if chunk < 1:
        raise ValueError("chunk must be >= 1")
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, N, dv))
    R = np.zeros((B, H, dk, dv)) if state_in is None else _f64(state_in).copy()
    for h in range(H):
        g = float(gammas[h])
        for s in range(0, N, chunk):
            L = min(chunk, N - s)
            j = np.arange(L)
            D = decay_mask(g, L)
            xi = np.power(g, j + 1)
            zeta = np.power(g, L - 1 - j)
            for b in range(B):
                Q, K, V = q[b, h, s:s + L], k[b, h, s:s + L], v[b, h, s:s + L]
                inner = ((Q @ K.T) * D) @ V
                cross = (Q * xi[:, None]) @ R[b, h]
                o[b, h, s:s + L] = inner + cross
                R[b, h] = g ** L * R[b, h] + K.T @ (V * zeta[:, None])
    return o, R


def group_norm(o, eps: float):
    """Per-head GroupNorm of retention outputs ([RetNet blog] Methods, block
    structure: MSR -> GroupNorm; [Medium] GroupNorm after the Hadamard
    product): for every (b, h, n), over the d_v values,
        mu = mean(o), var = mean((o - mu)^2), out = (o - mu) / sqrt(var + eps).
    """
    o = _f64(o)
    mu = o.mean(axis=-1, keepdims=True)
    var = ((o - mu) ** 2).mean(axis=-1, keepdims=True)
    return (o - mu) / np.sqrt(var + eps)


def backward(q, k, v, gammas, d_o, state_in=None, d_state_out=None):
    """Gradients of the retention outputs and the final state with respect to
    q, k, v and the initial state: the adjoint of the forms above ([RetNet
    blog] Key Equations; the pages call the parallel form the training form
    and give no gradient, so this is the chain rule written out).  Per
    (b, h), with A = Q K^T (.) D, xi_n = gamma^(n+1), z_m = gamma^(N-1-m),
    O = A V + (Q (.) xi) S_in and S_out = K^T (V (.) z) + gamma^N S_in:
        dA    = dO V^T (.) D
        dQ    = dA K + xi (.) (dO S_in^T)
        dK    = dA^T Q + z (.) (V dS_out^T)
        dV    = A^T dO + z (.) (K dS_out)
        dS_in = (Q (.) xi)^T dO + gamma^N dS_out.
    Returns (dq, dk, dv, d_state_in)."""
    q, k, v, d_o = _f64(q), _f64(k), _f64(v), _f64(d_o)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    s_in = np.zeros((B, H, dk, dv)) if state_in is None else _f64(state_in)
    d_s = np.zeros((B, H, dk, dv)) if d_state_out is None else _f64(d_state_out)
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    ds_in = np.zeros((B, H, dk, dv))
    n = np.arange(N)
    for h in range(H):
        g = float(gammas[h])
        D = decay_mask(g, N)
        xi = np.power(g, n + 1.0)
        z = np.power(g, N - 1.0 - n)
        for b in range(B):
            Q, K, V, dO = q[b, h], k[b, h], v[b, h], d_o[b, h]
            A = (Q @ K.T) * D
            dA = (dO @ V.T) * D
            dq[b, h] = dA @ K + xi[:, None] * (dO @ s_in[b, h].T)
            dkk[b, h] = dA.T @ Q + z[:, None] * (V @ d_s[b, h].T)
            dvv[b, h] = A.T @ dO + z[:, None] * (K @ d_s[b, h])
            ds_in[b, h] = (Q * xi[:, None]).T @ dO + g ** N * d_s[b, h]
    return dq, dkk, dvv, ds_in


def swish(x):
    """swish(x) = x * sigmoid(x) = x / (1 + exp(-x)), the gate activation of
    the retention block ([RetNet blog] core components, item 4: GroupNorm
    with swish gating).  The pages name the activation only; this is its
    standard definition, evaluated without overflow for large |x|."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    sig = np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return x * sig


def gated(y, g):
    """Gated multi-scale retention output swish(G) (.) Y ([RetNet blog] core
    components, item 4; abstract page, section 2.2 Gated Multi-Scale
    Retention): Y is the retention output (after the per-head GroupNorm when
    that is applied) and G a gate of the same shape.  Reading: G is an input
    of the operator; the projection that produces it and the output
    projection after the gate belong to the layer around it."""
    return swish(g) * _f64(y)


def rotate(x, theta, pos0: int = 0):
    """xPos-style rotation of q or k ([RetNet blog] core components, item 3:
    a complex rotation that puts relative position into Q and K; [Spiral.AI]
    LEX Transformer paragraph: the xPos term that links the recurrent and the
    parallel forms).

    x [..., N, d] with d even, theta [d/2]; the row at index j has position
    n = pos0 + j.  With phi = n theta_c, channel pair c turns by phi:
        y[2c]   = x[2c] cos(phi) - x[2c+1] sin(phi)
        y[2c+1] = x[2c] sin(phi) + x[2c+1] cos(phi)
    Rotating both q and k this way makes q'_n . k'_m = Re sum_c
    z_c(q_n) conj(z_c(k_m)) e^{i (n-m) theta_c}, a function of n - m only."""
    x = _f64(x)
    d = x.shape[-1]
    if d % 2:
        raise ValueError("rotate needs an even row length")
    n = pos0 + np.arange(x.shape[-2], dtype=np.float64)
    phi = n[:, None] * _f64(theta)[None, :]          # [N, d/2]
    c, s = np.cos(phi), np.sin(phi)
    re, im = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = re * c - im * s
    y[..., 1::2] = re * s + im * c
    return y


def rel_frobenius(x, ref) -> float:
    """||x - ref||_F / ||ref||_F (0 when both are zero)."""
    x, ref = _f64(x), _f64(ref)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)
