"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something it cannot agree with by
construction: hand-worked values, brute force, textbook special cases,
closed forms and the invariants the pages state (the three forms give the
same output; state passes exactly across chunk boundaries).  The mutation
tests at the end plant plausible mistakes in copies of the oracle's steps
and show that a pin catches each of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from linear_recurrent_sequence_scale_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _seq(a, d=None):
    """[N] or [N,d] list -> [1,1,N,d] float64."""
    x = np.asarray(a, dtype=np.float64)
    if x.ndim == 1:
        x = x[:, None]
    return x[None, None]


def _rand(rng, B, H, N, dk, dv, state=True):
    q = rng.standard_normal((B, H, N, dk))
    k = rng.standard_normal((B, H, N, dk))
    v = rng.standard_normal((B, H, N, dv))
    s = rng.standard_normal((B, H, dk, dv)) if state else None
    return q, k, v, s


# --- hand-worked values ------------------------------------------------------

@pytest.mark.parametrize("form", ["recurrent", "parallel", "chunk1", "chunk2", "chunk3"])
def test_hand_worked_scalar(form):
    g = _golden()["scalar"]
    q, k, v = _seq(g["q"]), _seq(g["k"]), _seq(g["v"])
    gam = [g["gamma"]]
    if form == "recurrent":
        o, s = oracle.recurrent(q, k, v, gam)
    elif form == "parallel":
        o, s = oracle.parallel(q, k, v, gam)
    else:
        o, s = oracle.chunkwise(q, k, v, gam, int(form[-1]))
    np.testing.assert_allclose(o[0, 0, :, 0], g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(s[0, 0, 0, 0], g["state"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("form", ["recurrent", "parallel", "chunk1", "chunk2"])
def test_hand_worked_matrix_with_state(form):
    g = _golden()["matrix_with_state"]
    q, k, v = _seq(g["q"]), _seq(g["k"]), _seq(g["v"])
    s0 = np.asarray(g["state_in"], dtype=np.float64)[None, None]
    gam = [g["gamma"]]
    if form == "recurrent":
        o, s = oracle.recurrent(q, k, v, gam, s0)
    elif form == "parallel":
        o, s = oracle.parallel(q, k, v, gam, s0)
    else:
        o, s = oracle.chunkwise(q, k, v, gam, int(form[-1]), s0)
    np.testing.assert_allclose(o[0, 0], g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(s[0, 0], g["state"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("form", ["recurrent", "parallel", "chunk2"])
def test_hand_worked_gamma_zero(form):
    g = _golden()["gamma_zero"]
    q, k, v = _seq(g["q"]), _seq(g["k"]), _seq(g["v"])
    gam = [g["gamma"]]
    if form == "recurrent":
        o, s = oracle.recurrent(q, k, v, gam)
    elif form == "parallel":
        o, s = oracle.parallel(q, k, v, gam)
    else:
        o, s = oracle.chunkwise(q, k, v, gam, 2)
    np.testing.assert_array_equal(o[0, 0], g["o"])
    np.testing.assert_array_equal(s[0, 0], g["state"])


def test_hand_worked_group_norm():
    g = _golden()["group_norm"]
    out = oracle.group_norm(np.asarray(g["o"], dtype=np.float64), g["eps"])
    np.testing.assert_allclose(out, g["out"], rtol=0, atol=1e-15)


def test_hand_worked_backward():
    g = _golden()["backward"]
    one = lambda x: np.asarray(x, dtype=np.float64).reshape(1, 1, 1, 1)
    dq, dk, dv, ds = oracle.backward(_seq(g["q"]), _seq(g["k"]), _seq(g["v"]), [g["gamma"]],
                                     _seq(g["d_o"]), one(g["state_in"]), one(g["d_state_out"]))
    np.testing.assert_allclose(dq[0, 0, :, 0], g["dq"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk[0, 0, :, 0], g["dk"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0, :, 0], g["dv"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(ds[0, 0, 0, 0], g["d_state_in"], rtol=0, atol=1e-14)


# --- P2: decay mask against brute force --------------------------------------

@pytest.mark.parametrize("gamma", [0.0, 0.3, 0.5, 0.96875, 1.0 - 2.0 ** -20, 1.0])
def test_decay_mask_brute_force(gamma):
    n = 16
    ref = np.zeros((n, n))
    for i in range(n):
        ref[i, i] = 1.0
        for j in range(i):
            # D[i, j] = gamma * D[i-1, j]: repeated multiplication
            ref[i, j] = gamma * ref[i - 1, j]
    np.testing.assert_allclose(oracle.decay_mask(gamma, n), ref, rtol=1e-14, atol=0)
    # lower-triangular, unit diagonal ([Medium]: D is lower triangular)
    assert np.all(np.triu(oracle.decay_mask(gamma, n), 1) == 0)


# --- P1 / P9: the three forms agree; state closed form -------------------------

@pytest.mark.parametrize("chunk", [1, 3, 7, 16, 37, 64])
@pytest.mark.parametrize("with_state", [False, True])
def test_three_forms_agree(chunk, with_state):
    rng = np.random.default_rng(11)
    q, k, v, s0 = _rand(rng, 2, 4, 37, 5, 6, state=with_state)
    gam = [0.9, 0.5, 0.999, 0.0]
    o_r, s_r = oracle.recurrent(q, k, v, gam, s0)
    o_p, s_p = oracle.parallel(q, k, v, gam, s0)
    o_c, s_c = oracle.chunkwise(q, k, v, gam, chunk, s0)
    assert oracle.rel_frobenius(o_p, o_r) < 1e-12
    assert oracle.rel_frobenius(o_c, o_r) < 1e-12
    assert oracle.rel_frobenius(s_p, s_r) < 1e-12
    assert oracle.rel_frobenius(s_c, s_r) < 1e-12


def test_state_closed_form_brute_force():
    """S_N = sum_m gamma^(N-1-m) k_m^T v_m + gamma^N S_0, summed term by term."""
    rng = np.random.default_rng(5)
    q, k, v, s0 = _rand(rng, 1, 1, 9, 3, 2)
    g = 0.7
    ref = g ** 9 * s0[0, 0].copy()
    for m in range(9):
        ref += g ** (8 - m) * np.outer(k[0, 0, m], v[0, 0, m])
    _, s = oracle.recurrent(q, k, v, [g], s0)
    np.testing.assert_allclose(s[0, 0], ref, rtol=1e-13)


# --- P3 / P4: textbook special cases ------------------------------------------

def test_gamma_zero_reduces_to_diagonal():
    rng = np.random.default_rng(3)
    q, k, v, _ = _rand(rng, 1, 1, 12, 4, 3, state=False)
    ref = np.einsum("nk,nk->n", q[0, 0], k[0, 0])[:, None] * v[0, 0]
    for form in ("recurrent", "parallel", "chunk"):
        if form == "recurrent":
            o, _ = oracle.recurrent(q, k, v, [0.0])
        elif form == "parallel":
            o, _ = oracle.parallel(q, k, v, [0.0])
        else:
            o, _ = oracle.chunkwise(q, k, v, [0.0], 5)
        np.testing.assert_allclose(o[0, 0], ref, rtol=1e-14, atol=1e-15)
    # a tiny gamma is a small perturbation of the same result
    o, _ = oracle.parallel(q, k, v, [1e-12])
    assert oracle.rel_frobenius(o[0, 0], ref) < 1e-10


def test_gamma_one_is_causal_linear_attention():
    """gamma = 1: o_n = q_n sum_{m<=n} k_m^T v_m (causal linear attention,
    the link to linear attention on the RetNet blog, Insights)."""
    rng = np.random.default_rng(4)
    q, k, v, _ = _rand(rng, 1, 1, 20, 4, 3, state=False)
    outer = k[0, 0][:, :, None] * v[0, 0][:, None, :]
    S = np.cumsum(outer, axis=0)
    ref = np.einsum("nk,nkv->nv", q[0, 0], S)
    for chunk in (1, 6, 20):
        o, s = oracle.chunkwise(q, k, v, [1.0], chunk)
        np.testing.assert_allclose(o[0, 0], ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(s[0, 0], S[-1], rtol=1e-12, atol=1e-12)


# --- P6: resume from a carried state ------------------------------------------

@pytest.mark.parametrize("split", [1, 13, 32, 49])
def test_split_sequence_resume(split):
    rng = np.random.default_rng(6)
    q, k, v, _ = _rand(rng, 2, 2, 50, 4, 5, state=False)
    gam = [0.95, 0.6]
    o_full, s_full = oracle.chunkwise(q, k, v, gam, 8)
    o1, s1 = oracle.chunkwise(q[:, :, :split], k[:, :, :split], v[:, :, :split], gam, 8)
    o2, s2 = oracle.chunkwise(q[:, :, split:], k[:, :, split:], v[:, :, split:], gam, 8, s1)
    assert oracle.rel_frobenius(np.concatenate([o1, o2], axis=2), o_full) < 1e-12
    assert oracle.rel_frobenius(s2, s_full) < 1e-12


def test_step_chain_equals_prefill():
    """A chunkwise prefill followed by single steps equals one long recurrence."""
    rng = np.random.default_rng(8)
    q, k, v, _ = _rand(rng, 2, 3, 30, 4, 4, state=False)
    gam = [0.9, 0.99, 0.3]
    o_ref, s_ref = oracle.recurrent(q, k, v, gam)
    _, s = oracle.chunkwise(q[:, :, :25], k[:, :, :25], v[:, :, :25], gam, 8)
    for n in range(25, 30):
        o, s = oracle.step(q[:, :, n], k[:, :, n], v[:, :, n], gam, s)
        np.testing.assert_allclose(o, o_ref[:, :, n], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s, s_ref, rtol=1e-12, atol=1e-12)


# --- P7: linearity --------------------------------------------------------------

def test_linearity():
    rng = np.random.default_rng(7)
    q, k, v, s0 = _rand(rng, 1, 2, 17, 3, 4)
    v2 = rng.standard_normal(v.shape)
    s02 = rng.standard_normal(s0.shape)
    gam = [0.8, 0.97]
    f = lambda qq, vv, ss: oracle.chunkwise(qq, k, vv, gam, 5, ss)
    o_a, s_a = f(q, v, s0)
    o_b, s_b = f(q, v2, s02)
    o_ab, s_ab = f(q, 2.0 * v - 3.0 * v2, 2.0 * s0 - 3.0 * s02)
    np.testing.assert_allclose(o_ab, 2 * o_a - 3 * o_b, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(s_ab, 2 * s_a - 3 * s_b, rtol=1e-11, atol=1e-11)
    o_q, _ = f(2.5 * q, v, s0)
    np.testing.assert_allclose(o_q, 2.5 * o_a, rtol=1e-12, atol=1e-12)


# --- P8: GroupNorm invariants ---------------------------------------------------

def test_group_norm_invariants():
    rng = np.random.default_rng(9)
    o = rng.standard_normal((2, 3, 11, 16)) * 3 + 1
    eps = 1e-5
    out = oracle.group_norm(o, eps)
    var = o.var(axis=-1, keepdims=True)
    np.testing.assert_allclose(out.mean(axis=-1), 0, atol=1e-13)
    np.testing.assert_allclose(out.var(axis=-1, keepdims=True), var / (var + eps), rtol=1e-12)
    # shift and positive-scale invariance of each group
    out2 = oracle.group_norm(4.0 * o + 7.0, 16 * eps)
    np.testing.assert_allclose(out2, out, rtol=1e-10, atol=1e-12)


# --- inputs: bf16 rounding and the decay schedule -------------------------------

def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 0.0],
                 dtype=np.float32)
    got = wl.bf16_bits_to_f64(wl.f32_to_bf16_bits(x))
    # 1+2^-8 is a tie -> 1 (even); 1+3*2^-8 is a tie -> 1+2^-6 (even); 1+2^-9 -> 1
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 0.0])


def test_msr_gammas_exact():
    g = wl.msr_gammas(16)
    assert g[0] == 0.96875 and g[1] == 0.984375
    assert float(g[15]) == 1.0 - 2.0 ** -20
    assert np.all((g > 0) & (g < 1))


# --- backward: the chain rule against finite differences ----------------------

@pytest.mark.parametrize("with_state", [False, True])
def test_backward_matches_finite_differences(with_state):
    """Directional derivatives of L = <dO, O> + <dS, S_out> (O, S_out from the
    parallel form with the closed-form state) by central differences, against
    <gradient, direction> from oracle.backward; also through the chunkwise
    form, whose agreement with the parallel form is pinned above."""
    rng = np.random.default_rng(31)
    B, H, N, dk, dv = 1, 2, 9, 3, 4
    q, k, v, s0 = _rand(rng, B, H, N, dk, dv, state=True)
    s0 = s0 if with_state else None
    gam = [0.8, 0.5]
    dO = rng.standard_normal((B, H, N, dv))
    dS = rng.standard_normal((B, H, dk, dv))
    gq, gk, gv, gs = oracle.backward(q, k, v, gam, dO, s0, dS)

    def loss(q_, k_, v_, s_, form):
        if form == "parallel":
            o, s = oracle.parallel(q_, k_, v_, gam, s_)
        else:
            o, s = oracle.chunkwise(q_, k_, v_, gam, 4, s_)
        return float((dO * o).sum() + (dS * s).sum())

    eps = 1e-6
    for form in ("parallel", "chunkwise"):
        for which in range(4 if with_state else 3):
            U = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v),
                 np.zeros((B, H, dk, dv))]
            U[which] = rng.standard_normal(U[which].shape)
            args_p = [q + eps * U[0], k + eps * U[1], v + eps * U[2]]
            args_m = [q - eps * U[0], k - eps * U[1], v - eps * U[2]]
            sp = None if s0 is None else s0 + eps * U[3]
            sm = None if s0 is None else s0 - eps * U[3]
            fd = (loss(*args_p, sp, form) - loss(*args_m, sm, form)) / (2 * eps)
            an = float((gq * U[0]).sum() + (gk * U[1]).sum() + (gv * U[2]).sum()
                       + (gs * U[3]).sum())
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (form, which, fd, an)


def test_backward_gamma_zero_and_one():
    """gamma = 0: O_n = (q_n . k_n) v_n, so dq_n = (dO_n . v_n) k_n; gamma = 1
    with dS = 0: dV_m = sum over n >= m of (q_n . k_m) dO_n (causal sums)."""
    rng = np.random.default_rng(32)
    q, k, v, _ = _rand(rng, 1, 1, 6, 3, 2, state=False)
    dO = rng.standard_normal((1, 1, 6, 2))
    gq, _, _, _ = oracle.backward(q, k, v, [0.0], dO)
    exp_q = np.einsum("nj,nj->n", dO[0, 0], v[0, 0])[:, None] * k[0, 0]
    np.testing.assert_allclose(gq[0, 0], exp_q, rtol=1e-12, atol=1e-12)
    _, _, gv, _ = oracle.backward(q, k, v, [1.0], dO)
    exp_v = np.stack([sum((q[0, 0, n] @ k[0, 0, m]) * dO[0, 0, n] for n in range(m, 6))
                      for m in range(6)])
    np.testing.assert_allclose(gv[0, 0], exp_v, rtol=1e-12, atol=1e-12)


# --- gate: swish(G) (.) Y ------------------------------------------------------

def test_swish_identities():
    """swish(x) - swish(-x) = x (sigmoid(x) + sigmoid(-x) = 1); swish(0) = 0;
    sigmoid(ln 3) = 3/4, so swish(ln 3) = (3/4) ln 3; swish(x) -> x and
    swish(-x) -> 0 as x grows; finite for |x| up to 1e4."""
    x = np.linspace(-30.0, 30.0, 121)
    np.testing.assert_allclose(oracle.swish(x) - oracle.swish(-x), x, rtol=0, atol=1e-12)
    assert oracle.swish(0.0) == 0.0
    assert abs(oracle.swish(np.log(3.0)) - 0.75 * np.log(3.0)) < 1e-15
    assert abs(oracle.swish(40.0) - 40.0) < 1e-12
    assert abs(oracle.swish(-40.0)) < 1e-14
    assert np.all(np.isfinite(oracle.swish(np.array([-1e4, 1e4]))))


def test_gated_pins():
    """The gate multiplies element by element: G = ln 3 everywhere scales Y by
    (3/4) ln 3; G = 0 gives 0; a gate of +40 on one column scales that column
    by 40 (swish(x) -> x) and leaves the others at 0."""
    rng = np.random.default_rng(21)
    y = rng.standard_normal((2, 3, 5, 4))
    np.testing.assert_allclose(oracle.gated(y, np.full_like(y, np.log(3.0))),
                               0.75 * np.log(3.0) * y, rtol=1e-14)
    assert np.all(oracle.gated(y, np.zeros_like(y)) == 0.0)
    g = np.zeros_like(y)
    g[..., 2] = 40.0
    out = oracle.gated(y, g)
    np.testing.assert_allclose(out[..., 2], 40.0 * y[..., 2], rtol=1e-12)
    assert np.all(out[..., [0, 1, 3]] == 0.0)


@pytest.mark.parametrize("mutation", ["sigmoid_only", "exp_sign", "tanh"])
def test_gate_pins_catch_planted_mistakes(mutation):
    x = np.linspace(-5.0, 5.0, 41)
    if mutation == "sigmoid_only":
        f = lambda t: 1.0 / (1.0 + np.exp(-t))
    elif mutation == "exp_sign":
        f = lambda t: t / (1.0 + np.exp(t))
    else:
        f = lambda t: t * np.tanh(t)
    caught = (np.max(np.abs(f(x) - f(-x) - x)) > 1e-6
              or abs(f(np.log(3.0)) - 0.75 * np.log(3.0)) > 1e-6)
    assert caught


# --- mutation tests: planted mistakes are caught by the pins --------------------

def _chunkwise_mutant(q, k, v, gammas, chunk, mutation):
    """A copy of the oracle's chunkwise steps with one planted mistake."""
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, N, dv))
    R = np.zeros((B, H, dk, dv))
    for h in range(H):
        g = gammas[h]
        for s in range(0, N, chunk):
            L = min(chunk, N - s)
            j = np.arange(L)
            D = oracle.decay_mask(g, L)
            xi = g ** (j + 1)
            zeta = g ** (L - 1 - j)
            if mutation == "xi_exponent":
                xi = g ** j
            if mutation == "diag_exclusive":
                D = D - np.eye(L)
            for b in range(B):
                Q, K, V = q[b, h, s:s + L], k[b, h, s:s + L], v[b, h, s:s + L]
                o[b, h, s:s + L] = ((Q @ K.T) * D) @ V + (Q * xi[:, None]) @ R[b, h]
                if mutation == "page_chunk_state":   # R_i = K^T V + gamma^chunk R_{i-1}
                    R[b, h] = g ** L * R[b, h] + K.T @ V
                elif mutation == "transposed_mask":
                    pass
                else:
                    R[b, h] = g ** L * R[b, h] + K.T @ (V * zeta[:, None])
            if mutation == "transposed_mask":
                for b in range(B):
                    Q, K, V = q[b, h, s:s + L], k[b, h, s:s + L], v[b, h, s:s + L]
                    o[b, h, s:s + L] = ((Q @ K.T) * D.T) @ V + (Q * xi[:, None]) @ R[b, h]
                    R[b, h] = g ** L * R[b, h] + K.T @ (V * zeta[:, None])
    return o, R


@pytest.mark.parametrize("mutation", ["xi_exponent", "diag_exclusive", "page_chunk_state",
                                      "transposed_mask"])
def test_pins_catch_planted_mistakes(mutation):
    rng = np.random.default_rng(12)
    q, k, v, _ = _rand(rng, 1, 2, 24, 3, 3, state=False)
    gam = [0.9, 0.5]
    o_ref, s_ref = oracle.recurrent(q, k, v, gam)
    o_m, s_m = _chunkwise_mutant(q, k, v, gam, 8, mutation)
    assert oracle.rel_frobenius(o_m, o_ref) > 1e-3 or oracle.rel_frobenius(s_m, s_ref) > 1e-3


def test_page_chunk_state_exact_only_for_gamma_one():
    """The chunk state as printed (no in-chunk decay) equals the recurrence
    only when gamma = 1; this is why the oracle carries zeta."""
    rng = np.random.default_rng(13)
    q, k, v, _ = _rand(rng, 1, 1, 16, 3, 3, state=False)
    o_ref, s_ref = oracle.recurrent(q, k, v, [1.0])
    o_m, s_m = _chunkwise_mutant(q, k, v, [1.0], 4, "page_chunk_state")
    assert oracle.rel_frobenius(o_m, o_ref) < 1e-12
    assert oracle.rel_frobenius(s_m, s_ref) < 1e-12


# --- xPos rotation ---------------------------------------------------------------

def test_hand_worked_rotation():
    g = _golden()["rotation"]
    theta = np.pi * np.asarray(g["theta_over_pi"])
    y = oracle.rotate(np.asarray(g["x"], dtype=np.float64), theta, g["pos0"])
    np.testing.assert_allclose(y, g["y"], rtol=0, atol=1e-14)


def _rotation_pins_hold(rot):
    """The rotation pins, for the oracle or a planted mutant: the hand-worked
    rows, complex multiplication by e^{i n theta} done with numpy's complex
    type, and q'_n . k'_m depending on n - m only."""
    g = _golden()["rotation"]
    theta = np.pi * np.asarray(g["theta_over_pi"])
    ok = np.allclose(rot(np.asarray(g["x"], dtype=np.float64), theta, g["pos0"]), g["y"],
                     rtol=0, atol=1e-12)
    rng = np.random.default_rng(31)
    x = rng.standard_normal((2, 3, 7, 10))
    th = rng.uniform(0.0, 2.0, 5)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * np.outer(np.arange(5, 12), th))
    want = np.stack([z.real, z.imag], axis=-1).reshape(x.shape)
    ok = ok and np.allclose(rot(x, th, 5), want, rtol=0, atol=1e-12)
    q, k = rng.standard_normal((1, 6)), rng.standard_normal((1, 6))
    th = rng.uniform(0.0, 2.0, 3)
    dots = [float(rot(q, th, n)[0] @ rot(k, th, m)[0]) for n, m in [(4, 1), (9, 6), (3, 0)]]
    ok = ok and np.allclose(dots, dots[0], rtol=1e-12)
    return ok


def test_rotation_pins():
    assert _rotation_pins_hold(oracle.rotate)


def test_rotation_invariants():
    """theta = 0 and position 0 leave rows unchanged; each channel pair keeps
    its length; turning by theta1 then theta2 is turning by theta1 + theta2;
    rotating q and k with the same offset leaves retention unchanged, since
    q'_n . k'_m depends on n - m only."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal((2, 2, 9, 8))
    t1, t2 = rng.uniform(-3, 3, 4), rng.uniform(-3, 3, 4)
    np.testing.assert_array_equal(oracle.rotate(x, np.zeros(4), 17), x)
    np.testing.assert_allclose(oracle.rotate(x[..., :1, :], t1, 0), x[..., :1, :], rtol=0,
                               atol=0)
    y = oracle.rotate(x, t1, 3)
    np.testing.assert_allclose(y[..., 0::2] ** 2 + y[..., 1::2] ** 2,
                               x[..., 0::2] ** 2 + x[..., 1::2] ** 2, rtol=1e-13)
    np.testing.assert_allclose(oracle.rotate(oracle.rotate(x, t1, 3), t2, 3),
                               oracle.rotate(x, t1 + t2, 3), rtol=0, atol=1e-12)
    q, k, v, _ = _rand(rng, 1, 2, 12, 8, 3, state=False)
    gam = [0.9, 0.6]
    o0, _ = oracle.parallel(oracle.rotate(q, t1, 0), oracle.rotate(k, t1, 0), v, gam)
    o1, _ = oracle.parallel(oracle.rotate(q, t1, 1000), oracle.rotate(k, t1, 1000), v, gam)
    assert oracle.rel_frobenius(o1, o0) < 1e-12
    with pytest.raises(ValueError):
        oracle.rotate(np.zeros((2, 3)), np.zeros(1))


def test_rotation_of_a_span_is_a_slice_of_the_whole():
    """A span that starts at position s, rotated with pos0 = s, gives the
    same rows as the whole sequence rotated from 0 (what a caller does when a
    sequence is split across GPUs, or when decoding token s)."""
    rng = np.random.default_rng(33)
    x = rng.standard_normal((2, 3, 40, 12))
    th = rng.uniform(0.0, 2.0, 6)
    whole = oracle.rotate(x, th, 0)
    for s0, s1 in ((0, 7), (7, 23), (23, 40), (39, 40)):
        np.testing.assert_allclose(oracle.rotate(x[..., s0:s1, :], th, s0), whole[..., s0:s1, :],
                                   rtol=0, atol=1e-13)


def _rotate_mutant(x, theta, pos0, mutation):
    """A copy of the oracle's rotation with one planted mistake."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    n = pos0 + np.arange(x.shape[-2], dtype=np.float64)
    if mutation == "position_off_by_one":
        n = n + 1
    phi = n[:, None] * np.asarray(theta, dtype=np.float64)[None, :]
    if mutation == "negative_angle":
        phi = -phi
    c, s = np.cos(phi), np.sin(phi)
    if mutation == "cos_sin_swapped":
        c, s = s, c
    if mutation == "half_split_pairs":
        re, im = x[..., :half], x[..., half:]
    else:
        re, im = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    if mutation == "half_split_pairs":
        y[..., :half], y[..., half:] = re * c - im * s, re * s + im * c
    else:
        y[..., 0::2], y[..., 1::2] = re * c - im * s, re * s + im * c
    if mutation == "rows_not_positions":       # every row turned by pos0 alone
        y[..., 0::2] = re * np.cos(pos0 * theta) - im * np.sin(pos0 * theta)
        y[..., 1::2] = re * np.sin(pos0 * theta) + im * np.cos(pos0 * theta)
    return y


@pytest.mark.parametrize("mutation", ["position_off_by_one", "negative_angle", "cos_sin_swapped",
                                      "half_split_pairs", "rows_not_positions"])
def test_rotation_pins_catch_planted_mistakes(mutation):
    assert not _rotation_pins_hold(lambda x, t, p: _rotate_mutant(x, t, p, mutation))


def _backward_mutant(q, k, v, gam, d_o, s_in, d_s, mutation):
    """A copy of the oracle's backward for one (b, h) with one planted mistake."""
    Q, K, V, dO = q[0, 0], k[0, 0], v[0, 0], d_o[0, 0]
    S, dS = s_in[0, 0], d_s[0, 0]
    N = Q.shape[0]
    n = np.arange(N)
    g = float(gam[0])
    D = oracle.decay_mask(g, N)
    xi = g ** (n + 1.0)
    z = g ** (N - 1.0 - n)
    if mutation == "xi_exponent":
        xi = g ** n
    if mutation == "zeta_exponent":
        z = g ** (N - n)
    A = (Q @ K.T) * D
    dA = (dO @ V.T) * (np.ones_like(D) if mutation == "mask_dropped" else D)
    dq = dA @ K + xi[:, None] * (dO @ S.T)
    dk = dA.T @ Q + z[:, None] * (V @ dS.T)
    dv = (A if mutation == "untransposed_a" else A.T) @ dO + z[:, None] * (K @ dS)
    ds = (Q * xi[:, None]).T @ dO + (0.0 if mutation == "no_state_carry" else g ** N * dS)
    return dq, dk, dv, ds


@pytest.mark.parametrize("mutation", ["xi_exponent", "zeta_exponent", "mask_dropped",
                                      "untransposed_a", "no_state_carry"])
def test_backward_pins_catch_planted_mistakes(mutation):
    g = _golden()["backward"]
    one = lambda x: np.asarray(x, dtype=np.float64).reshape(1, 1, 1, 1)
    got = _backward_mutant(_seq(g["q"]), _seq(g["k"]), _seq(g["v"]), [g["gamma"]],
                           _seq(g["d_o"]), one(g["state_in"]), one(g["d_state_out"]), mutation)
    want = (g["dq"], g["dk"], g["dv"], [g["d_state_in"]])
    clean = _backward_mutant(_seq(g["q"]), _seq(g["k"]), _seq(g["v"]), [g["gamma"]],
                             _seq(g["d_o"]), one(g["state_in"]), one(g["d_state_out"]), None)
    assert all(np.allclose(np.ravel(a), b, rtol=0, atol=1e-12) for a, b in zip(clean, want))
    assert any(not np.allclose(np.ravel(a), b, rtol=0, atol=1e-9) for a, b in zip(got, want))


# --- the parity checker ------------------------------------------------------
# Every parity assertion divides ||x - ref||_F by ||ref||_F.  The values below
# are worked by hand, and each planted mistake in a copy of the quotient
# (a difference of norms, no square root, the wrong denominator, zero for a
# zero reference, a max-norm) fails at least one of them.

REL_FROBENIUS_CASES = [
    # x, ref, value worked by hand
    ([0.0, 0.0], [3.0, 4.0], 1.0),                    # ||(-3,-4)|| / ||(3,4)|| = 5/5
    ([1.0, 1.0], [1.0, 2.0], 1.0 / np.sqrt(5.0)),     # ||(0,-1)|| / sqrt(1 + 4)
    ([1.0, 2.0], [1.0, 1.0], 1.0 / np.sqrt(2.0)),     # divided by the reference, not by x
    ([[1.0, 0.0], [0.0, 1.0]], [[2.0, 0.0], [0.0, 2.0]], 0.5),   # sqrt(2) / sqrt(8)
    ([-3.0, -4.0], [3.0, 4.0], 2.0),                  # ||(-6,-8)|| / 5: the sign counts
    ([3.0, 4.0], [3.0, 4.0], 0.0),
    ([0.0, 0.0], [0.0, 0.0], 0.0),                    # both zero
    ([0.5, 0.0], [0.0, 0.0], np.inf),                 # any error against a zero reference
]


def _rel_frobenius_pins_hold(fn):
    for x, ref, want in REL_FROBENIUS_CASES:
        got = fn(np.asarray(x), np.asarray(ref))
        if np.isinf(want):
            if not np.isinf(got):
                return False
        elif not np.isclose(got, want, rtol=1e-14, atol=0.0):
            return False
    return True


def _rel_frobenius_mutant(x, ref, mutation):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    num = np.linalg.norm((x - ref).ravel())
    den = np.linalg.norm(ref.ravel())
    if mutation == "difference_of_norms":
        num = abs(np.linalg.norm(x.ravel()) - den)
    if mutation == "no_square_root":
        num, den = num ** 2, den ** 2
    if mutation == "divided_by_x":
        den = np.linalg.norm(x.ravel())
    if mutation == "max_norm":
        num, den = np.abs(x - ref).max(), np.abs(ref).max()
    if den == 0.0:
        if mutation == "zero_reference_passes":
            return 0.0
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


def test_rel_frobenius_hand_worked():
    assert _rel_frobenius_pins_hold(oracle.rel_frobenius)


@pytest.mark.parametrize("mutation", ["difference_of_norms", "no_square_root", "divided_by_x",
                                      "max_norm", "zero_reference_passes"])
def test_rel_frobenius_pins_catch_planted_mistakes(mutation):
    assert _rel_frobenius_pins_hold(lambda x, r: _rel_frobenius_mutant(x, r, None))
    assert not _rel_frobenius_pins_hold(lambda x, r: _rel_frobenius_mutant(x, r, mutation))


def test_parity_blocks_find_a_local_error():
    """A defect confined to one 128-row tile of one head, diluted below the
    tolerance in the whole-output figure, is reported at full size by the
    per-tile check the GPU tests use."""
    from parity_check import worst, worst_rel
    rng = np.random.default_rng(5)
    ref = rng.standard_normal((2, 3, 8192, 64))
    x = ref.copy()
    x[1, 2, 1024:1152] *= 1.15                  # one tile 15% off
    assert oracle.rel_frobenius(x, ref) < 2e-2  # lost in the whole
    where, e = worst(x, ref)
    assert where == "(b,h)=(1, 2) rows 1024:1152" and np.isclose(e, 0.15, rtol=1e-12)
    assert worst_rel(ref, ref) == 0.0
    # a head that is wrong as a whole, and a decode row ([B,H,d] layout)
    y = ref.copy()
    y[0, 1] *= 1.01
    assert np.isclose(worst_rel(y, ref), 0.01, rtol=1e-12)
    d = rng.standard_normal((4, 16, 512))
    dd = d.copy()
    dd[3, 9] = 0.0
    assert worst(dd, d)[0] == "(b,h)=(3, 9)" and worst_rel(dd, d) == 1.0
    nan = ref.copy()
    nan[0, 0, 5, 5] = np.nan
    assert worst_rel(nan, ref) == np.inf
